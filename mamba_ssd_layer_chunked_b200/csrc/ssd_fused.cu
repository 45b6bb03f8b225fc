// ssd_fused.cu -- the fused tensor-core path of the SSD forward (bf16 in, fp32
// state): the block decomposition applied at two levels.
//
// The rows (batch row, head pair) are laid end to end, each cut into 128-token
// tiles, and the resulting line of tiles is cut into equal work ranges, one
// per CTA (about one per SM, so the ranges finish together). Within a range a
// CTA walks its tiles and carries the state on chip from tile to tile; a range
// may start or end inside a row, and only the states at those cuts go through
// HBM. Three kernels:
//
//   segment_state    per range ending inside a row: the end state of the
//                    range's last sequence piece from a zero start,
//                    accumulated over its tiles in TMEM (the right factors of
//                    the block algorithm at range level);
//   segment_passing  the short recurrence over the cuts of each row (centre
//                    factors), giving the state entering each range that
//                    starts inside a row;
//   fused_scan       per range: for each tile the masked quadratic term
//                    (L o C B^T) X, the carried state read out by C, D x, and
//                    the carried state update H <- a(tile) H + sum_l a(l..end) B_l x_l^T.
//
// Source: "Mamba-2: writing the recurrent state as a structured matrix"
// (wq-win.github.io/llm/088-mamba2.html), section 3 (block algorithm: local
// output, local end state, block decay, scan over blocks, incoming state read
// out by C) and section 2.3 (only independent-sample boundaries stop the
// state). The output equals the step recurrence regardless of the block sizes
// (section 1 of the same page: changing the order of computation need not
// change the output), so the tiles here are aligned to sequence starts: no tile
// mixes two sequences.
//
// fused_scan has 20 warps: 16 compute warps (warp w reaches the TMEM lane
// quarter w % 4) that run each tile's epilogue, L o G build and state update in
// turn; three issuing threads, one warp each (the L o G-side MMAs, the
// state-side MMAs and the Y store, the TMA loads); and one decay warp that walks
// the range ahead of the others and publishes, per tile, its coordinates and
// the within-tile cumsum of log a. The roles handshake through mbarriers.

#include <cuda.h>

#include <algorithm>
#include <atomic>

#include "ssd_tc.cuh"
#include "tc_ptx.cuh"

namespace ssd {

namespace {

using namespace tc;

constexpr int kP = 64;
constexpr uint32_t kBox = 128u * 128u;  // [128 rows][64 bf16] with 128-byte swizzle
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ int seq_clamped(const int32_t* seq_idx, int64_t row, int t, int nseq) {
    return seq_at(seq_idx, row, t, nseq);
}

// ---------------------------------------------------------------------------
// work ranges: rows r = b * npairs + hp, each of nt tiles of 128 tokens; the
// tiles of all rows in a line, cut into ranges of wt tiles (the last shorter)
// ---------------------------------------------------------------------------
struct Work {
    int npairs, nt, wt, nwork;
    int64_t total;  // rows * nt
};

__device__ __forceinline__ int64_t work_begin(const Work& w, int i) { return (int64_t)i * w.wt; }
__device__ __forceinline__ int64_t work_end(const Work& w, int i) {
    return min((int64_t)(i + 1) * w.wt, w.total);
}
// tokens [s0, s1) of row r that tiles [fb, fe) of the line cover
__device__ __forceinline__ void row_piece(const Work& w, int seqlen, int64_t fb, int64_t fe, int r, int& s0, int& s1) {
    const int64_t rb = (int64_t)r * w.nt;
    s0 = (int)(128 * max(fb - rb, (int64_t)0));
    s1 = (int)min((int64_t)128 * (fe - rb), (int64_t)seqlen);
}

// The two 64-column slots of pair row hp (rows r = b * npairs + hp): slot s
// carries head h from column p0 of that head's dimension. The heads of a group
// are paired in order; in a group with an odd number of heads the last pair's
// slot 1 has no head of its own (valid = false): it mirrors slot 0's head and
// nothing of it is written. With headdim 128 a row is one head, and its two
// slots are the two halves of the head dimension.
struct Slot {
    int h, p0;
    bool valid;
};
__device__ __forceinline__ Slot slot_of(const Dims& d, int hp, int s) {
    Slot o;
    if (d.headdim == 2 * kP) {
        o.h = hp;
        o.p0 = kP * s;
        o.valid = true;
        return o;
    }
    const int npg = (d.heads_per_group + 1) >> 1;  // pairs per group
    const int g = hp / npg, j = hp - g * npg;
    const int h0 = g * d.heads_per_group + 2 * j;
    o.valid = s == 0 || 2 * j + 1 < d.heads_per_group;
    o.h = o.valid ? h0 + s : h0;
    o.p0 = 0;
    return o;
}

// ===========================================================================
// segment_state
// ===========================================================================
constexpr float kSegCutLog = -40.f;           // walk cut: natural log of the decay product
constexpr int kSegScale = 256;                 // the warps that scale X and own the accumulator lanes
constexpr int kSegThreads = kSegScale + 32;    // + one warp that issues the MMAs

template <int N>
__global__ void __launch_bounds__(kSegThreads, 1)
    segment_state_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b, Dims d,
                         Work wk, const float* __restrict__ log_a, const int32_t* __restrict__ seq_idx,
                         float* __restrict__ work_local, float* __restrict__ work_decay, int whole_rows,
                         int32_t* __restrict__ row_ids, unsigned int* __restrict__ err) {
    constexpr uint32_t kXB = 2 * kBox, kBB = (N / 64) * kBox, kStage = kXB + kBB;
    // three stages: tile it scaled, tile it - 1 multiplied, tile it + 1 loading
    constexpr int kStages = 3;
    constexpr uint32_t kScaleBar = 1;  // named barrier of the scaling warps
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    __shared__ float wsum[8];
    __shared__ float tail_s[2];
    __shared__ int st_shared;
    __shared__ int probe_j;  // the last 128-token probe with the last sequence's id
    __shared__ int n_iter;  // iterations scaled (set when the scaling warps stop)
    __shared__ __align__(8) uint64_t bar_load[kStages], bar_mma[kStages], bar_scaled[kStages];
    __shared__ uint32_t tmem_base;

    wait_guard_init(err);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the scan that follows may start its setup and first tile now: it waits
    // for this grid before it reads the range states
    griddep_launch_dependents();
    // the last piece of range i, when it ends inside its row (or, with
    // whole_rows, one range per row: the whole row, its ids into row_ids)
    const int i_work = blockIdx.x;
    const int64_t fe = work_end(wk, i_work);
    const int r = (int)((fe - 1) / wk.nt);
    int s0, s1;
    row_piece(wk, d.seqlen, work_begin(wk, i_work), fe, r, s0, s1);
    if (s1 >= d.seqlen && !whole_rows) return;  // ends at the row end: nothing feeds a next range
    const int hp = r % wk.npairs, b = r / wk.npairs;
    const Slot sl0 = slot_of(d, hp, 0), sl1 = slot_of(d, hp, 1);
    const int g = sl0.h / d.heads_per_group;
    const int64_t row = (int64_t)b * d.seqlen;
    if (whole_rows && hp == 0 && tid == 0) {
        row_ids[2 * b] = seq_idx ? seq_clamped(seq_idx, row, 0, d.nseq) : 0;
        row_ids[2 * b + 1] = seq_idx ? seq_clamped(seq_idx, row, d.seqlen - 1, d.nseq) : 0;
    }

    if (tid == 0) {
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_b);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bar_load[s], 1);
            mbar_init(&bar_mma[s], 1);
            mbar_init(&bar_scaled[s], 1);
        }
        mbar_fence_init();
        st_shared = s0;
        probe_j = 0;
        n_iter = 1 << 30;
        tail_s[0] = tail_s[1] = 0.f;
    }
    // Start of the piece's last sequence: the first token of [s0, s1) with the
    // id of token s1 - 1 (ids never decrease), in two rounds of independent
    // loads. Round 1 probes every 128th token back from s1 - 1; the last probe
    // J that still has that id bounds the start to the 128 tokens ending at
    // probe J. Round 2 checks those tokens one per thread.
    if (seq_idx) {
        const int sl = seq_clamped(seq_idx, row, s1 - 1, d.nseq);
        const int nprobe = (s1 - s0 + 127) / 128;  // probes s1 - 1 - 128 j >= s0
        __syncthreads();
        int jb = 0;
        for (int j = tid; j < nprobe; j += kSegThreads)
            if (seq_clamped(seq_idx, row, s1 - 1 - 128 * j, d.nseq) == sl) jb = max(jb, j);
        if (jb > 0) atomicMax(&probe_j, jb);
        __syncthreads();
        const int qj = s1 - 1 - 128 * probe_j;
        const int lo = max(s0, qj - 127);
        if (tid == 0) st_shared = qj;
        __syncthreads();
        for (int u = tid; lo + u <= qj; u += kSegThreads)
            if (seq_clamped(seq_idx, row, lo + u, d.nseq) == sl) atomicMin(&st_shared, lo + u);
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, N);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tacc = tmem_base;
    const int st = st_shared;
    const int ntiles = (s1 - st + 127) / 128;
    bool cut = false;
    int lm = 0;  // the last iteration scaled (and multiplied)
    if (warp == kSegScale / 32) {
        // ---- MMA issue: S += (weighted X)^T B for every scaled tile, in order ----
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, N, true, true);
            for (int it = 0;; ++it) {
                const int sg = it % kStages;
                mbar_wait(&bar_scaled[sg], (it / kStages) & 1);
                if (it >= *reinterpret_cast<volatile int*>(&n_iter)) break;  // the scaling warps stopped
                tc_fence_after();
                const uint32_t xa = smem_u32(smem + sg * kStage), ba = xa + kXB;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_bf16_ss(tacc, smem_desc_sw128(xa + k * 2048, kBox, 1024),
                                smem_desc_sw128(ba + k * 2048, kBox, 1024), idesc, (it > 0 || k > 0) ? 1u : 0u);
                mma_commit(&bar_mma[sg]);
            }
        }
        __syncwarp();
    } else {
        const int rr = tid & 127, hh = tid >> 7;  // this thread's row and head in the transform
        float tail = 0.f;  // sum of log a after the current tile, this thread's head
        // log a of this thread's (row, head) in a tile; unconditional (clamped row)
        // so that the prefetch does not stall until the value is used
        auto load_la = [&](int i) -> float {
            const int ts = st + 128 * i;
            const int v = min(128, s1 - ts);
            return log_a[(row + ts + min(rr, v - 1)) * d.nheads + (hh ? sl1.h : sl0.h)];
        };
        // tile i's X (two heads) and B into stage sg
        auto issue_load = [&](int i, int sg) {
            const int ts = st + 128 * i;
            uint8_t* xs = smem + sg * kStage;
            uint8_t* bs = xs + kXB;
            mbar_arrive_expect_tx(&bar_load[sg], kStage);
            tma_load_4d(xs, &tm_x, &bar_load[sg], sl0.p0, sl0.h, ts, b);
            tma_load_4d(xs + kBox, &tm_x, &bar_load[sg], sl1.p0, sl1.h, ts, b);
#pragma unroll
            for (int q = 0; q < N / 64; ++q) tma_load_4d(bs + q * kBox, &tm_b, &bar_load[sg], 64 * q, g, ts, b);
        };
        float la_cur = load_la(ntiles - 1);
        if (tid == 0) issue_load(ntiles - 1, 0);
        // tiles from the end backwards; iteration it holds tile ntiles - 1 - it in
        // stage it % 3 (its use it / 3): while it is scaled, the MMAs of it - 1
        // run and tile it + 1 loads into the stage of it - 2
        int it = 0;
        for (int i = ntiles - 1; i >= 0; --i, ++it) {
            const int sg = it % kStages;
            const int ts = st + 128 * i;
            const int v = min(128, s1 - ts);
            const float la_nxt = i > 0 ? load_la(i - 1) : 0.f;
            if (tid == 0 && i > 0) {
                const int sn = (it + 1) % kStages;
                if (it >= 2) mbar_wait(&bar_mma[sn], ((it - 2) / kStages) & 1);  // read by the MMAs of it - 2
                issue_load(i - 1, sn);
            }
            // within-tile inclusive cumsum of log a (one row per thread, one head per 4 warps)
            float x = rr < v ? la_cur : 0.f;
            la_cur = la_nxt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (lane == 31) wsum[warp] = x;
            named_bar_sync(kScaleBar, kSegScale);
            float pre = 0.f, tot = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float sw = wsum[4 * hh + w];
                if (w < (warp & 3)) pre += sw;
                tot += sw;
            }
            const float cs = x + pre;
            // weight of row rr: prod of a over (rr, segment end] = exp(tail + tot - cs)
            const float wgt = rr < v ? ex2_approx((tail + tot - cs) * kLog2e) : 0.f;
            mbar_wait(&bar_load[sg], (it / kStages) & 1);
            // scale row rr of head hh in place; the chunk order is rotated by row so
            // that the 32 rows of a warp spread over all banks
            uint8_t* Xs = smem + sg * kStage;
            {
                uint8_t* rowp = Xs + hh * kBox + rr * 128;
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    const int c = (cc + rr) & 7;
                    uint4 vv = *reinterpret_cast<uint4*>(rowp + 16 * c);
                    uint32_t* u = reinterpret_cast<uint32_t*>(&vv);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u[k]));
                        u[k] = pack_bf16(f.x * wgt, f.y * wgt);
                    }
                    *reinterpret_cast<uint4*>(rowp + 16 * c) = vv;
                }
            }
            fence_async_shared();
            tail += tot;
            if (rr == 0) tail_s[hh] = tail;
            named_bar_sync(kScaleBar, kSegScale);
            if (tid == 0) mbar_arrive(&bar_scaled[sg]);  // the MMA warp may multiply tile it
            // the rest of the piece reaches the cut through a decay product below
            // e^kSegCutLog for both heads: its terms are below 1e-17 of the partial
            // state they come from, under the fp32 rounding of the kept sum
            if (tail_s[0] < kSegCutLog && tail_s[1] < kSegCutLog && i > 0) {
                cut = true;
                break;
            }
        }
        lm = cut ? it : it - 1;
        if (tid == 0) {
            // stop the MMA warp at iteration lm + 1
            n_iter = lm + 1;
            mbar_arrive(&bar_scaled[(lm + 1) % kStages]);
            // after a cut at tile i >= 1: the load issued for tile i - 1
            if (cut) mbar_wait(&bar_load[(lm + 1) % kStages], ((lm + 1) / kStages) & 1);
        }
        // the last MMAs (in order, so all of them)
        mbar_wait(&bar_mma[lm % kStages], (lm / kStages) & 1);
    }
    __syncthreads();
    tc_fence_after();
    if (warp < kSegScale / 32) {
        // epilogue: lane m = (head, p); warps w and w+4 split the N columns
        const int m = 32 * (warp & 3) + lane, half = warp >> 2;
        const int eh = m >> 6, p = m & 63;
        float* dst = work_local + ((int64_t)i_work * 2 + eh) * N * kP;
        const uint32_t lane_addr = tacc + ((uint32_t)(32 * (warp & 3)) << 16);
#pragma unroll
        for (int n0 = 0; n0 < N / 2; n0 += 32) {
            float vv[32];
            tmem_ld32(lane_addr + half * (N / 2) + n0, vv);
#pragma unroll
            for (int k = 0; k < 32; ++k) dst[(int64_t)(half * (N / 2) + n0 + k) * kP + p] = vv[k];
        }
        if (tid < 2) {
            const float t = tail_s[tid];
            work_decay[(int64_t)i_work * 2 + tid] = cut ? 0.f : ex2_approx(t * kLog2e);
        }
    }
    tc_fence_before();
    __syncthreads();
    wait_guard_finish();
    if (warp == 0) tmem_dealloc(tacc, N);
}

// ===========================================================================
// segment_passing: for every range i that starts inside its row r, the state
// entering it for the sequence of its first token. Over the pieces of row r
// before that cut (ranges i0 .. i-1 in order), H_end = decay * H_start + local,
// with H_start = H_end of the previous piece when the piece's last sequence
// continues from it, else that sequence's initial state (or zero); the entering
// state is H_end of the last piece when the first token continues the previous
// token's sequence, else its initial state (or zero). One block per (cut, head,
// slice of the state): the cuts are independent, each chain is a few pieces.
// ===========================================================================
constexpr int kPassMaxLinks = 64;  // pieces before a cut handled per block (longer chains loop)

__global__ void __launch_bounds__(256) segment_passing_kernel(Dims d, Work wk, const float* __restrict__ work_local,
                                                              const float* __restrict__ work_decay,
                                                              const float* __restrict__ init_states,
                                                              const int32_t* __restrict__ seq_idx,
                                                              float* __restrict__ work_in) {
    // per piece j of the chain: last id, last piece continues, and for the cut itself
    __shared__ int sl_s[kPassMaxLinks], cl_s[kPassMaxLinks];
    __shared__ int sf_s, cf_s;
    const int i = blockIdx.x >> 1, hh = blockIdx.x & 1;
    const int64_t fb = work_begin(wk, i);
    const int r = (int)(fb / wk.nt);
    const int64_t rb = (int64_t)r * wk.nt;
    if (fb == rb) return;  // the range starts at its row start: no entering state needed
    const int b = r / wk.npairs, h = 2 * (r % wk.npairs) + hh;
    const int NP = d.dstate * d.headdim;
    const int idx = (blockIdx.y * 256 + threadIdx.x) * 4;
    const bool active = idx < NP;
    const int64_t row = (int64_t)b * d.seqlen;
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    auto init_of = [&](int sq) -> float4 {
        if (!init_states) return zero;
        return *reinterpret_cast<const float4*>(init_states + seqst_off(d, b, sq, h) + idx);
    };
    const int i0 = (int)(rb / wk.wt);
    const int s_cut = (int)(128 * (fb - rb));  // first token of range i in row r
    float4 H = zero;
    for (int j0 = i0; j0 < i; j0 += kPassMaxLinks) {
        const int nl = min(kPassMaxLinks, i - j0);
        __syncthreads();
        // sequence information of the pieces [s0, s1) of ranges j0 .. j0+nl-1 in row r
        for (int l = threadIdx.x; l < nl; l += blockDim.x) {
            int s0, s1;
            row_piece(wk, d.seqlen, work_begin(wk, j0 + l), work_end(wk, j0 + l), r, s0, s1);
            int sl = 0, cont_last = (s0 > 0);
            if (seq_idx) {
                // the piece's last sequence starts at s0 when s0 already has its id
                // (ids never decrease), and continues when s0 - 1 has it too
                sl = seq_clamped(seq_idx, row, s1 - 1, d.nseq);
                const int prev = s0 > 0 ? seq_clamped(seq_idx, row, s0 - 1, d.nseq) : -1;
                cont_last = seq_clamped(seq_idx, row, s0, d.nseq) == sl && prev == sl;
            }
            sl_s[l] = sl;
            cl_s[l] = cont_last;
        }
        if (threadIdx.x == 0 && j0 + nl == i) {
            int sf = 0, cont_first = 1;
            if (seq_idx) {
                sf = seq_clamped(seq_idx, row, s_cut, d.nseq);
                cont_first = seq_clamped(seq_idx, row, s_cut - 1, d.nseq) == sf;
            }
            sf_s = sf;
            cf_s = cont_first;
        }
        __syncthreads();
        if (!active) continue;
#pragma unroll 4
        for (int l = 0; l < nl; ++l) {
            const int j = j0 + l;
            const int64_t o = ((int64_t)j * 2 + hh) * NP + idx;
            const float dec = work_decay[(int64_t)j * 2 + hh];
            const float4 sv = *reinterpret_cast<const float4*>(work_local + o);
            const float4 st = cl_s[l] ? H : init_of(sl_s[l]);
            H = make_float4(fmaf(dec, st.x, sv.x), fmaf(dec, st.y, sv.y), fmaf(dec, st.z, sv.z), fmaf(dec, st.w, sv.w));
        }
    }
    if (active)
        *reinterpret_cast<float4*>(work_in + ((int64_t)i * 2 + hh) * NP + idx) = cf_s ? H : init_of(sf_s);
}

// ===========================================================================
// fused_scan
// ===========================================================================
constexpr int kComputeWarps = 16;
constexpr int kComputeThreads = 32 * kComputeWarps;
// + two MMA-issue warps, the decay warp and the TMA warp: 5 warps on two of the
// four SM sub-partitions, which still fits 96 registers a thread
constexpr int kFusedThreads = kComputeThreads + 128;
constexpr int kCsBufs = 4;                           // decay buffers in flight
constexpr int kChainBatch = 64;                      // pieces resolved together in the scan prologue

template <int N>
struct FusedSmem {
    static constexpr uint32_t kC = (N / 64) * kBox;
    static constexpr uint32_t kB = (N / 64) * kBox;  // per stage
    static constexpr uint32_t kX = 2 * kBox;         // per stage, two heads
    static constexpr uint32_t kH = (N / 64) * kBox;  // carried state, bf16, rows (h,p), K = n
    static constexpr uint32_t kHY = kH > 2 * kBox ? kH : 2 * kBox;  // ... and the Y staging of a tile
    static constexpr uint32_t oC = 0, oB = kC, oX = oB + 2 * kB, oH = oX + 2 * kX, oTail = oH + kHY;
};

// One tile of a range, as the decay warp publishes it: batch row, head pair,
// first token, valid rows, the sequence id of its tokens, the id of the token
// before it in the row (-1 at the row start) and flags.
// Also the row's slot mapping (slot_of), worked out once per tile: the heads
// of slots 0 and 1, the first column of slot 1 in its head, the B/C group.
struct TileDesc {
    int b, hp, ts, v, sid, psid, flags;
    int h0, h1, p1, g;
};
enum : int {
    kTileLast = 1,       // last tile of its sequence piece in this range
    kTileSeqEnd = 2,     // ... and the sequence ends there (its final state is due)
    kTileRowEnd = 4,     // the tile ends its row
    kTileFinal = 8,      // last tile of the range
    kTileFromWork = 16,  // first tile of a range that starts inside its row
    kTileNoSlot1 = 32    // slot 1 has no head (odd heads per group): nothing of it is written
};

// 16-row block of the tokens held by lane half hi (lanes 16 hi .. 16 hi + 15)
// of TMEM lane quarter q: TMEM lane m holds token m of the tile in G, L o G
// and the Y accumulators.
__device__ __forceinline__ int row_block(int q, int hi) { return 2 * q + hi; }

// Per-tile data, written by the decay warp: c[h][k] = log2(e) * the
// within-tile inclusive cumsum of log a for head h, the whole-tile decays and
// the tile's descriptor.
struct __align__(16) CsBuf {
    float c[2][128];
    float dec[2];
    int pad[3];
    TileDesc td;
};
// every buffer's c rows are read and written as float4
static_assert(sizeof(CsBuf) % 16 == 0, "CsBuf must keep 16-byte alignment in an array");

// ---------------------------------------------------------------------------
// The decay warp of the scan kernels. Walks range i_work's pieces (one per row
// it covers) in tiles of at most 128 tokens that never cross a sequence start,
// one tile ahead of the buffers it fills: per tile its descriptor, the
// within-tile inclusive cumsum of log a (log2 units) for both heads, and the
// whole-tile decays. Lane j holds tokens 4j .. 4j+3 of a tile.
// ---------------------------------------------------------------------------
template <bool kGen>
__device__ __forceinline__ void decay_walk(const Dims d, const Work wk, const int i_work, const int lane,
                                        const float* __restrict__ log_a, const int32_t* __restrict__ seq_idx,
                                        CsBuf* csb, uint64_t* bar_csfull, uint64_t* bar_csfree) {
    const int64_t fb = work_begin(wk, i_work), fe = work_end(wk, i_work);
    int r = (int)(fb / wk.nt);
    int s0, s1;
    row_piece(wk, d.seqlen, fb, fe, r, s0, s1);
    int pos = s0;
    bool first = true;
    auto next_tile = [&](TileDesc& td) {
        const int b = r / wk.npairs, hp = r % wk.npairs;
        const int64_t row = (int64_t)b * d.seqlen;
        int v = min(128, s1 - pos);
        int sid = 0, psid = pos > 0 ? 0 : -1;
        bool change = false;  // the sequence changes right after the tile
        if (seq_idx) {
            sid = seq_clamped(seq_idx, row, pos, d.nseq);
            if (pos > 0) psid = seq_clamped(seq_idx, row, pos - 1, d.nseq);
            // first offset j in [1, min(128, s1 - pos - 1)] whose id differs
            const int jmax = min(128, s1 - pos - 1);
            int jm = 1 << 30;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int jj = 4 * lane + 1 + e;
                if (jj <= jmax && seq_clamped(seq_idx, row, pos + jj, d.nseq) != sid) jm = min(jm, jj);
            }
            jm = __reduce_min_sync(0xffffffffu, jm);
            if (jm <= jmax) {
                v = jm;
                change = true;
            }
        }
        const int pend = pos + v;
        const bool piece_end = pend == s1;
        const bool last_piece = (int64_t)(r + 1) * wk.nt >= fe;
        bool seq_end = false;
        if (pend == d.seqlen) seq_end = true;
        else if (change) seq_end = true;
        else if (piece_end && seq_idx) seq_end = seq_clamped(seq_idx, row, pend, d.nseq) != sid;
        int flags = 0;
        if (piece_end || change) flags |= kTileLast;
        if ((piece_end || change) && seq_end) flags |= kTileSeqEnd;
        if (pend == d.seqlen) flags |= kTileRowEnd;
        if (piece_end && last_piece) flags |= kTileFinal;
        if (first && s0 > 0) flags |= kTileFromWork;
        Slot q0, q1;
        if constexpr (kGen) {
            q0 = slot_of(d, hp, 0);
            q1 = slot_of(d, hp, 1);
            if (!q1.valid) flags |= kTileNoSlot1;
        } else {  // a plain head pair
            q0 = {2 * hp, 0, true};
            q1 = {2 * hp + 1, 0, true};
        }
        td.b = b;
        td.hp = hp;
        td.ts = pos;
        td.v = v;
        td.sid = sid;
        td.psid = psid;
        td.flags = flags;
        td.h0 = q0.h;
        td.h1 = q1.h;
        td.p1 = q1.p0;
        td.g = q0.h / d.heads_per_group;
        first = false;
        pos = pend;
        if (piece_end && !last_piece) {
            ++r;
            row_piece(wk, d.seqlen, fb, fe, r, s0, s1);
            pos = s0;
        }
    };
    auto load4 = [&](const TileDesc& td, float (&v)[2][4]) {
        const int64_t row = (int64_t)td.b * d.seqlen;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int tok = 4 * lane + e;
                v[hh][e] = tok < td.v ? log_a[(row + td.ts + tok) * d.nheads + (hh ? td.h1 : td.h0)] : 0.f;
            }
    };
    TileDesc cur;
    next_tile(cur);
    float lcur[2][4];
    load4(cur, lcur);
    for (int t = 0;; ++t) {
        const bool fin = (cur.flags & kTileFinal) != 0;
        TileDesc nxt = cur;
        float lnxt[2][4];
        if (!fin) {
            next_tile(nxt);
            load4(nxt, lnxt);
        }
        const int bi = t & (kCsBufs - 1);
        if (t >= kCsBufs) mbar_wait(&bar_csfree[bi], ((t / kCsBufs) - 1) & 1);
        const int last = cur.v - 1;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float x0 = lcur[hh][0] * kLog2e;
            float x1 = fmaf(lcur[hh][1], kLog2e, x0);
            float x2 = fmaf(lcur[hh][2], kLog2e, x1);
            float x3 = fmaf(lcur[hh][3], kLog2e, x2);
            float tot = x3;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, tot, o);
                if (lane >= o) tot += y;
            }
            const float pre = tot - x3;
            x0 += pre;
            x1 += pre;
            x2 += pre;
            x3 += pre;
            *reinterpret_cast<float4*>(&csb[bi].c[hh][4 * lane]) = make_float4(x0, x1, x2, x3);
            const int el = last & 3;
            const float mine = el == 0 ? x0 : el == 1 ? x1 : el == 2 ? x2 : x3;
            const float cend = __shfl_sync(0xffffffffu, mine, last >> 2);
            if (lane == 0) csb[bi].dec[hh] = ex2_approx(cend);
        }
        if (lane == 0) csb[bi].td = cur;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_csfull[bi]);
        if (fin) break;
        cur = nxt;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int e = 0; e < 4; ++e) lcur[hh][e] = lnxt[hh][e];
    }
}

// Thread layout of the 16 compute warps: warp w owns the TMEM lane quarter
// w % 4 and the column quarter w / 4 of every 128-column accumulator it
// touches; the four warps of a lane quarter split the columns.
//
// Per tile t the compute warps run, in this order,
//   epilogue(t):  Y = Y_diag + rscale Y_off (D x is on the diagonal of L o G, so
//                 it is part of Y_diag), staged (bf16) in the buffer
//                 of the carried state, which Y_off(t) has finished reading, for
//                 the TMA store; X' = w X in place in the tile's X buffer;
//   L o G(t+1):   the next tile's masked C B^T, written over G in TMEM (while
//                 the tile state MMA of tile t runs and Y(t) drains);
//   state(t):     the carried state H(t) (in TMEM: the tile state MMA adds
//                 X'^T B onto it) to bf16 for the next C H and to the final
//                 states, then pre-scaled by the next tile's decay.
// The decay warp runs ahead, filling the decay buffers. One thread each issues
// the MMAs of the L o G side (G, Y_diag), those of the state side (Y_off, the
// Y store, the tile state), and the TMA loads: an MMA issue blocks for about
// the MMA's run time, so one issuing thread would serialise work whose inputs
// are ready at different times.
// Tensor memory: G, then L o G in place [0,128); Y_diag [128,256);
// Y_off [256,384); the carried state H [384,512) (rows (head, p), N columns).
// kAcc: a later state slice, whose epilogue adds its Y to the Y already there
// (each thread reads the elements it then writes); a separate instantiation so
// that the common case keeps its epilogue unchanged. kSeq: sequence ids are
// given (the prologue's chain over the pieces before a cut then starts at the
// last piece in which a sequence starts); without them every branch on the ids
// folds away at compile time, which keeps the kernel's code (and so its
// instruction fetch) smaller.
template <int N, bool kAcc, bool kGen, bool kSeq>
__global__ void __launch_bounds__(kFusedThreads, 1)
    fused_scan_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                      const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y, Dims d,
                      Work wk, const float* __restrict__ log_a, const float* __restrict__ Dv,
                      const float* __restrict__ work_in, const float* __restrict__ init_states,
                      const int32_t* __restrict__ seq_idx_arg, __nv_bfloat16* __restrict__ Y,
                      float* __restrict__ final_states, const float* __restrict__ work_local,
                      const float* __restrict__ work_decay, unsigned int* __restrict__ err) {
    using S = FusedSmem<N>;
    // without sequence ids every branch on them folds away at compile time
    const int32_t* __restrict__ seq_idx = kSeq ? seq_idx_arg : nullptr;
    constexpr int NQ = N / 4;  // state columns per thread
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* Cs = smem + S::oC;
    uint8_t* Hs = smem + S::oH;
    __shared__ __align__(16) CsBuf csb[kCsBufs];
    // per-warp column factors of the full L o G blocks, [warp][head][row half][column]
    // (the second half's 32 entries XOR-swizzled by 4 so that both halves' float4
    // reads fall in different banks)
    __shared__ __align__(16) float colf[kComputeWarps][2][2][32];
    // per-warp factors exp2(c_{r+8} - c_{r+e}), e < 8, of the diagonal blocks [warp][row half][head][e]
    __shared__ __align__(16) float cf8[kComputeWarps][2][2][8];
    // per-thread row factors of the next tile: rf (head 0, 1), rg (head 0, 1)
    __shared__ float rowf_s[4][kComputeThreads];
    // the prologue's chain over the pieces before a cut: per piece its last
    // sequence id and whether that sequence continues from the piece before
    __shared__ int chain_sl[kChainBatch];
    __shared__ int chain_cont[kChainBatch];
    __shared__ __align__(8) uint64_t bar_c, bar_bx[2], bar_g, bar_yo, bar_yd, bar_s, bar_sfree[2], bar_lg, bar_epi,
        bar_st, bar_free, bar_csfull[kCsBufs], bar_csfree[kCsBufs];
    __shared__ uint32_t tmem_base;

    wait_guard_init(err);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int i_work = blockIdx.x;

    // ---- setup: barriers, TMEM ----
    if (tid == 0) {
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_b);
        prefetch_tmap(&tm_c);
        prefetch_tmap(&tm_y);
        mbar_init(&bar_c, 1);
        mbar_init(&bar_bx[0], 1);
        mbar_init(&bar_bx[1], 1);
        mbar_init(&bar_free, 1);
        mbar_init(&bar_g, 1);
        mbar_init(&bar_yo, 1);
        mbar_init(&bar_yd, 1);
        mbar_init(&bar_s, 1);
        mbar_init(&bar_sfree[0], 1);
        mbar_init(&bar_sfree[1], 1);
        mbar_init(&bar_lg, kComputeWarps);
        mbar_init(&bar_epi, kComputeWarps);
        mbar_init(&bar_st, kComputeWarps);
        for (int i = 0; i < kCsBufs; ++i) {
            mbar_init(&bar_csfull[i], 1);
            mbar_init(&bar_csfree[i], kComputeWarps);
        }
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm_g = tmem_base, tm_lg = tmem_base, tm_yd = tmem_base + 128, tm_yo = tmem_base + 256,
                   tm_h = tmem_base + 384;

    const uint32_t ca = smem_u32(Cs), ha = smem_u32(Hs);
    // slot s of a tile's row: its head, first column in that head, and whether it
    // has a head (kGen: the mapping the decay warp worked out; else a plain head
    // pair 2 hp, 2 hp + 1)
    auto head_of = [&](const TileDesc& td, int s) -> int {
        if constexpr (kGen) return s ? td.h1 : td.h0;
        else return 2 * td.hp + s;
    };
    auto p0_of = [&](const TileDesc& td, int s) -> int {
        if constexpr (kGen) return s ? td.p1 : 0;
        else return 0;
    };
    auto valid_of = [&](const TileDesc& td, int s) -> bool {
        if constexpr (kGen) return s == 0 || !(td.flags & kTileNoSlot1);
        else return true;
    };
    auto group_row = [&](const TileDesc& td) -> int {
        if constexpr (kGen) return td.g;
        else return 2 * td.hp / d.heads_per_group;
    };
    auto stage_x = [&](int t) { return smem_u32(smem + S::oX + (t & 1) * S::kX); };
    auto stage_b = [&](int t) { return smem_u32(smem + S::oB + (t & 1) * S::kB); };
    // tile t's descriptor, once the decay warp has published it
    auto desc = [&](int t) -> TileDesc {
        mbar_wait(&bar_csfull[t & (kCsBufs - 1)], (t / kCsBufs) & 1);
        return csb[t & (kCsBufs - 1)].td;
    };
    // Every wait below is for an event that cannot be followed by the barrier's
    // next phase before the waiting thread acts: the thread itself issues, or
    // loads an operand of, the work that completes that next phase.
    if (warp == kComputeWarps) {
        // =================== MMA issue, L o G side: G(t), Y_diag(t) ===================
        if (lane == 0) {
            const uint32_t idesc_nn = idesc_bf16(128, 128, false, false);  // K-major A and B
            const uint32_t idesc_ts = idesc_bf16(128, 64, false, true);    // TMEM A, MN-major B
            for (int t = 0;; ++t) {
                const bool fin = (desc(t).flags & kTileFinal) != 0;
                // G(t) = C(t) B(t)^T once both are in and Y_diag(t-1) has read
                // L o G(t-1) from the same tensor memory columns
                mbar_wait(&bar_c, t & 1);
                mbar_wait(&bar_bx[t & 1], (t >> 1) & 1);
                if (t > 0) mbar_wait(&bar_yd, (t - 1) & 1);
                tc_fence_after();
                const uint32_t ba = stage_b(t);
                // descriptors of later K steps: the start-address field plus the offset in 16-byte units
                const uint64_t dc = smem_desc_sw128(ca, 16, 1024), db = smem_desc_sw128(ba, 16, 1024);
#pragma unroll
                for (int k = 0; k < N / 16; ++k) {
                    const uint32_t off = ((k >> 2) * kBox + (k & 3) * 32) >> 4;
                    mma_bf16_ss(tm_g, dc + off, db + off, idesc_nn, k > 0 ? 1u : 0u);
                }
                mma_commit(&bar_g);
                // Y_diag(t) = (L o G)(t) X(t), A operand from TMEM, once L o G(t) is
                // built (the compute warps build it after epilogue(t-1) has read
                // Y_diag(t-1), and before state(t-1))
                mbar_wait(&bar_lg, t & 1);
                tc_fence_after();
                const uint64_t dx = smem_desc_sw128(stage_x(t), kBox, 1024);
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_bf16_ts(tm_yd + 64 * hh, tm_lg + 16 * k + 8 * hh, dx + ((hh * kBox + k * 2048) >> 4), idesc_ts,
                                    k > 0 ? 1u : 0u);
                mma_commit(&bar_yd);
                if (fin) break;
            }
        }
        __syncwarp();
    } else if (warp == kComputeWarps + 2) {
        // =================== MMA issue, state side: Y_off(t), Y store, tile state ===================
        if (lane == 0) {
            const uint32_t idesc_nn = idesc_bf16(128, 128, false, false);  // K-major A and B
            const uint32_t idesc_st = idesc_bf16(128, N, true, true);      // MN-major A and B
            for (int t = 0;; ++t) {
                const uint32_t par = t & 1;
                // Y_off(t) = C(t) Hs once the state before tile t is in Hs
                mbar_wait(&bar_c, par);
                mbar_wait(&bar_st, par);
                tc_fence_after();
                const uint64_t dc = smem_desc_sw128(ca, 16, 1024), dh = smem_desc_sw128(ha, 16, 1024);
#pragma unroll
                for (int k = 0; k < N / 16; ++k) {
                    const uint32_t off = ((k >> 2) * kBox + (k & 3) * 32) >> 4;
                    mma_bf16_ss(tm_yo, dc + off, dh + off, idesc_nn, k > 0 ? 1u : 0u);
                }
                mma_commit(&bar_yo);
                // epilogue(t) done: store Y(t) from the staging buffer; H += X'^T B
                mbar_wait(&bar_epi, par);
                // tile t's descriptor was published before epilogue(t) began; its
                // buffer is refilled only after state(t), which needs bar_free below,
                // so every field is read before that arrival
                const TileDesc& cur = csb[t & (kCsBufs - 1)].td;
                tc_fence_after();
                const bool full = cur.v == 128;
                const bool last = (cur.flags & kTileFinal) != 0;
                if (full) {
                    tma_store_4d(&tm_y, Hs, p0_of(cur, 0), head_of(cur, 0), cur.ts, cur.b);
                    if (valid_of(cur, 1)) tma_store_4d(&tm_y, Hs + kBox, p0_of(cur, 1), head_of(cur, 1), cur.ts, cur.b);
                    tma_store_commit();
                }
                const uint64_t dx = smem_desc_sw128(stage_x(t), kBox, 1024), db = smem_desc_sw128(stage_b(t), kBox, 1024);
#pragma unroll
                for (int k = 0; k < 8; ++k) mma_bf16_ss(tm_h, dx + k * (2048 >> 4), db + k * (2048 >> 4), idesc_st, 1u);
                mma_commit(&bar_s);
                mma_commit(&bar_sfree[t & 1]);  // the B/X stage of tile t is free
                if (full) tma_store_wait_read0();
                mbar_arrive(&bar_free);
                if (last) break;
            }
            tma_store_wait0();
        }
        __syncwarp();
    } else if (warp == kComputeWarps + 3) {
        // =================== TMA loads: C(t), B(t), X(t) ===================
        if (lane == 0) {
            auto load_bx = [&](const TileDesc& td, int st) {
                const int g = group_row(td);
                uint8_t* Bsg = smem + S::oB + st * S::kB;
                uint8_t* Xsg = smem + S::oX + st * S::kX;
                mbar_arrive_expect_tx(&bar_bx[st], S::kB + S::kX);
#pragma unroll
                for (int q = 0; q < N / 64; ++q)
                    tma_load_4d(Bsg + q * kBox, &tm_b, &bar_bx[st], 64 * q, g, td.ts, td.b);
                tma_load_4d(Xsg, &tm_x, &bar_bx[st], p0_of(td, 0), head_of(td, 0), td.ts, td.b);
                tma_load_4d(Xsg + kBox, &tm_x, &bar_bx[st], p0_of(td, 1), head_of(td, 1), td.ts, td.b);
            };
            auto load_c = [&](const TileDesc& td) {
                const int g = group_row(td);
                mbar_arrive_expect_tx(&bar_c, S::kC);
#pragma unroll
                for (int q = 0; q < N / 64; ++q) tma_load_4d(Cs + q * kBox, &tm_c, &bar_c, 64 * q, g, td.ts, td.b);
            };
            // in issue order: C(0), B X(0), B X(1), C(1), B X(2), C(2), ...: B, X of
            // tile u into stage u & 1 once the tile state MMA of tile u - 2 has
            // read it; C(u) once G(u-1) and Y_off(u-1) have read C(u-1) (at u = 1
            // the initial state can release Y_off(0) before G(0) has run)
            load_c(desc(0));
            for (int u = 0;; ++u) {
                const TileDesc td = desc(u);
                if (u >= 2) mbar_wait(&bar_sfree[u & 1], ((u - 2) >> 1) & 1);
                load_bx(td, u & 1);
                if (u >= 1) {
                    mbar_wait(&bar_g, (u - 1) & 1);
                    mbar_wait(&bar_yo, (u - 1) & 1);
                    load_c(td);
                }
                if (td.flags & kTileFinal) break;
            }
        }
        __syncwarp();
    } else if (warp == kComputeWarps + 1) {
        // =================== decay warp ===================
        decay_walk<kGen>(d, wk, i_work, lane, log_a, seq_idx, csb, bar_csfull, bar_csfree);
    } else {
        // =================== compute warps ===================
        const int q4 = warp & 3, cq = warp >> 2;
        const int m = 32 * q4 + lane;           // TMEM lane
        const int k = m;                        // its token in G, L o G and Y
        const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
        const int sh = m >> 6, sp = m & 63;     // state row (head, p) of lane m

        auto signal = [&](uint64_t* bar) {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar);
        };
        auto wait_cs = [&](int t) { mbar_wait(&bar_csfull[t & (kCsBufs - 1)], (t / kCsBufs) & 1); };
        // L o G of tile t into TMEM over G (bf16 pairs; the 16-token K block k of
        // head h in columns [16 k + 8 h, 16 k + 8 h + 8)), so that warp w reads its
        // 32 G columns [32 (w / 4), +32) and writes L o G back over the same columns.
        // Lane half hi holds the 16-row block rb of tokens; column block c (16
        // tokens) is zero above rb, exp2(c_k - c_l) masked on the diagonal block, and
        // below it exp2(c_k - c_{16 rb}) * exp2(c_{16 rb} - c_l), both factors <= 1.
        // this lane's row factors for one head: rf to its row block start, rg
        // to the middle of the row block, ck its cumsum, dd the head's D
        struct HeadF {
            float rf, rg, ck, dd;
        };
        // the per-warp column factor tables of tile t and this lane's row factors
        // rf, rg of tile t (before the wait for Y(t-1))
        auto lg_tables = [&](int t) {
            const CsBuf& cs = csb[t & (kCsBufs - 1)];
            const int l = 32 * cq + lane;
            {
                const int rb = row_block(q4, lane >> 4);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const float ck = cs.c[hh][k];
                    rowf_s[hh][tid] = ex2_approx(ck - cs.c[hh][16 * rb]);
                    rowf_s[2 + hh][tid] = ex2_approx(ck - cs.c[hh][16 * rb + 8]);
                }
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const float cl = cs.c[hh][l];
                // only columns l < 16 rb are read back (full blocks)
                colf[warp][hh][0][lane] = ex2_approx(cs.c[hh][16 * row_block(q4, 0)] - cl);
                colf[warp][hh][1][lane ^ 4] = ex2_approx(cs.c[hh][16 * row_block(q4, 1)] - cl);
            }
            {
                const int hf = lane >> 4, hh = (lane >> 3) & 1, e = lane & 7;
                const int r = 16 * row_block(q4, hf);
                cf8[warp][hf][hh][e] = ex2_approx(cs.c[hh][r + 8] - cs.c[hh][r + e]);
            }
        };
        // The diagonal 16x16 block of row block rb for head hh, this lane's 16
        // columns as 8 packed words: 8x8 quadrants, row i < 8 has columns [0, 8)
        // direct (masked); row i >= 8 has [8, 16) direct and [0, 8) as
        // exp2(c_k - c_{r+8}) exp2(c_{r+8} - c_l) (both factors <= 1); the
        // diagonal element also carries D_h, so that Y_diag includes D x.
        // g(j) = (selb ? gb : ga)[j] are the block's 16 G values of this lane.
        auto diag_block = [&](const CsBuf& cs, const HeadF& f, int hh, int rb, const uint32_t* ga, const uint32_t* gb,
                              bool selb, uint32_t* w) {
            const int hi = lane >> 4, i = lane & 15;
            const bool lo = i < 8;
            const int own = lo ? 0 : 8;
            const float* cr = &cs.c[hh][16 * rb + own];
            const float4 ca = *reinterpret_cast<const float4*>(cr);
            const float4 cb = *reinterpret_cast<const float4*>(cr + 4);
            const float cv[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
            const float4 fa = *reinterpret_cast<const float4*>(&cf8[warp][hi][hh][0]);
            const float4 fb = *reinterpret_cast<const float4*>(&cf8[warp][hi][hh][4]);
            const float fv[8] = {fa.x, fa.y, fa.z, fa.w, fb.x, fb.y, fb.z, fb.w};
            float dv[8], lv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const uint32_t g0 = selb ? gb[e] : ga[e], g8 = selb ? gb[8 + e] : ga[8 + e];
                const float v = __uint_as_float(lo ? g0 : g8) * ex2_approx(f.ck - cv[e]);
                dv[e] = own + e < i ? v : (own + e == i ? v + f.dd : 0.f);
                lv[e] = lo ? dv[e] : __uint_as_float(g0) * f.rg * fv[e];
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                w[e] = pack_bf16(lv[2 * e], lv[2 * e + 1]);
                w[4 + e] = lo ? 0u : pack_bf16(dv[2 * e], dv[2 * e + 1]);
            }
        };
        // a full block (all columns below the row block) for head hh: 8 packed words
        auto full_block = [&](const HeadF& f, int hh, int cc, const uint32_t* g, uint32_t* w) {
            const int hi = lane >> 4;
            const float* cf = &colf[warp][hh][hi][0];
            const float2 r2 = make_float2(f.rf, f.rf);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
                const float4 fq = *reinterpret_cast<const float4*>(cf + ((16 * cc + 4 * v4) ^ (4 * hi)));
                const uint32_t* g4 = g + 4 * v4;
                const float2 a = __fmul2_rn(__fmul2_rn(make_float2(__uint_as_float(g4[0]), __uint_as_float(g4[1])), r2),
                                            make_float2(fq.x, fq.y));
                const float2 c = __fmul2_rn(__fmul2_rn(make_float2(__uint_as_float(g4[2]), __uint_as_float(g4[3])), r2),
                                            make_float2(fq.z, fq.w));
                w[2 * v4] = pack_bf16(a.x, a.y);
                w[2 * v4 + 1] = pack_bf16(c.x, c.y);
            }
        };
        // L o G(t) over G(t) in TMEM. Warp (q4, cq) covers row blocks 2 q4,
        // 2 q4 + 1 and column blocks 2 cq, 2 cq + 1: all zero for cq > q4, all
        // full for cq < q4, the diagonal pair for cq == q4. G stays in registers
        // while each head's two 8-column groups go back to TMEM, so the head
        // loop needs no staging and is not unrolled (code size).
        auto build_lg = [&](int t) {
            const CsBuf& cs = csb[t & (kCsBufs - 1)];
            const int hi = lane >> 4;
            const int rb = row_block(q4, hi);
            const uint32_t tcol = tm_lg + lane_off + 32 * cq;  // this warp's 32 columns
            __syncwarp();
            mbar_wait(&bar_g, t & 1);
            tc_fence_after();
            if (cq > q4) {
                const uint32_t z[32] = {};
                tmem_st32(tcol, z);
            } else {
                uint32_t gw[32];  // G columns [32 cq, 32 cq + 32)
                tmem_ld32_async(tcol, gw);
                tmem_wait_ld();
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    const HeadF f = {rowf_s[hh][tid], rowf_s[2 + hh][tid], cs.c[hh][k],
                                     Dv ? Dv[head_of(cs.td, hh)] : 0.f};
                    uint32_t w0[8], w1[8];
                    full_block(f, hh, 0, gw, w0);  // column block 0: full below the diagonal pair
                    if (cq == q4) {
                        // lane half hi's diagonal block is column block hi; block 0
                        // is full for half 1, block 1 zero for half 0: one pass for
                        // both halves, no divergence
                        uint32_t dw[8];
                        diag_block(cs, f, hh, rb, gw, gw + 16, hi != 0, dw);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            w1[e] = hi ? dw[e] : 0u;
                            w0[e] = hi ? w0[e] : dw[e];
                        }
                    } else {
                        full_block(f, hh, 1, gw + 16, w1);
                    }
                    tmem_st8(tcol + 8 * hh, w0);       // column block 2 cq, head hh
                    tmem_st8(tcol + 16 + 8 * hh, w1);  // column block 2 cq + 1, head hh
                }
            }
            tmem_wait_st();
            tc_fence_before();
            signal(&bar_lg);
        };
        // the state columns [NQ cq, NQ cq + NQ) of lane m, to/from TMEM
        auto ld_state = [&](float (&v)[NQ]) {
            if constexpr (NQ == 32) {
                uint32_t r[32];
                tmem_ld32_async(tm_h + lane_off + NQ * cq, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
            } else {
                uint32_t r[16];
                tmem_ld16_async(tm_h + lane_off + NQ * cq, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
            }
        };
        // scales v in place, then stores it
        auto st_state_scaled = [&](float (&v)[NQ], float a) {
#pragma unroll
            for (int i = 0; i < NQ; i += 2) {
                const float2 sc = __fmul2_rn(make_float2(v[i], v[i + 1]), make_float2(a, a));
                v[i] = sc.x;
                v[i + 1] = sc.y;
            }
            if constexpr (NQ == 32) tmem_st32(tm_h + lane_off + NQ * cq, reinterpret_cast<const uint32_t(&)[32]>(v));
            else tmem_st16(tm_h + lane_off + NQ * cq, reinterpret_cast<const uint32_t(&)[16]>(v));
        };
        // src: this slot's columns of an [N][stride] state (stride = headdim for the
        // caller's states, 64 for the range buffers), or null for zero
        auto load_state = [&](float (&v)[NQ], const float* src, int stride) {
#pragma unroll
            for (int i = 0; i < NQ; ++i) v[i] = src ? src[(int64_t)(cq * NQ + i) * stride + sp] : 0.f;
        };
        const int P = kGen ? d.headdim : kP;  // row stride of the caller's states
        auto write_hs = [&](const float (&v)[NQ]) {  // bf16 state, row m, K-major over n
#pragma unroll
            for (int c8 = 0; c8 < NQ / 8; ++c8) {
                const int n = cq * NQ + 8 * c8;
                const uint4 u = make_uint4(pack_bf16(v[8 * c8], v[8 * c8 + 1]), pack_bf16(v[8 * c8 + 2], v[8 * c8 + 3]),
                                           pack_bf16(v[8 * c8 + 4], v[8 * c8 + 5]), pack_bf16(v[8 * c8 + 6], v[8 * c8 + 7]));
                *reinterpret_cast<uint4*>(Hs + (n >> 6) * kBox + sw128_off(m, (n & 63) >> 3)) = u;
            }
        };

        // this slot's columns of the initial state of sequence sid of batch row b
        // in pair row hp, or null (zero) without initial states or for a slot
        // without a head
        auto init_src = [&](int b, int hp, int sid) -> const float* {
            if constexpr (kGen) {
                const Slot o = slot_of(d, hp, sh);
                return init_states && o.valid ? init_states + seqst_off(d, b, sid, o.h) + o.p0 : nullptr;
            } else {
                return init_states ? init_states + seqst_off(d, b, sid, 2 * hp + sh) : nullptr;
            }
        };
        // this slot's columns of the final state of sequence sid, or null for a
        // slot without a head
        auto final_dst = [&](int b, int hp, int sid) -> float* {
            if constexpr (kGen) {
                const Slot o = slot_of(d, hp, sh);
                return o.valid ? final_states + seqst_off(d, b, sid, o.h) + o.p0 : nullptr;
            } else {
                return final_states + seqst_off(d, b, sid, 2 * hp + sh);
            }
        };

        // ids that never occur between the sequence before tile td and its own
        // keep their initial state (or zero) as final state
        auto fill_gap = [&](const TileDesc& td) {
            if (!final_states || !seq_idx) return;
            for (int sq = td.psid + 1; sq < td.sid; ++sq) {
                float* f = final_dst(td.b, td.hp, sq);
                if (!f) continue;
                const float* src = init_src(td.b, td.hp, sq);
#pragma unroll 1
                for (int i = 0; i < NQ; ++i) {
                    const int64_t o = (int64_t)(cq * NQ + i) * P + sp;
                    f[o] = src ? src[o] : 0.f;
                }
            }
        };

        // ---- prologue: tile 0's L o G and the first piece's state ----
        wait_cs(0);
        fill_gap(csb[0].td);
        lg_tables(0);
        build_lg(0);
        {
            const TileDesc& td0 = csb[0].td;
            float hv[NQ];
            if (!(td0.flags & kTileFromWork)) {
                load_state(hv, init_src(td0.b, td0.hp, td0.sid), P);
            } else if (work_in) {
                load_state(hv, work_in + ((int64_t)i_work * 2 + sh) * N * kP, kP);
            } else {
                // The range starts inside its row: the state entering its first
                // token from the pieces of the row before the cut (ranges i0 ..
                // i_work - 1, each E = dec * start + loc from segment_state), with
                // start = the previous piece's E when the piece's last sequence
                // continues from it, else that sequence's initial state (or zero);
                // the entering state is the last E when the first token
                // continues the previous token's sequence, else its initial state.
                const int64_t fb = work_begin(wk, i_work);
                const int r = (int)(fb / wk.nt);
                const int64_t rb = (int64_t)r * wk.nt;
                const int b = r / wk.npairs, hp = r % wk.npairs;
                const int64_t row = (int64_t)b * d.seqlen;
                const int s_cut = (int)(128 * (fb - rb));
#pragma unroll
                for (int i = 0; i < NQ; ++i) hv[i] = 0.f;
                // Pieces are taken kChainBatch at a time: first every piece's last
                // sequence id and whether that sequence continues from the piece
                // before (its first token seq(s0) has that id, and so does the token
                // before s0: ids never decrease), one piece per thread; then the
                // chain itself, element by element. The ids come from seq_idx alone,
                // so they are read before the wait for the range states.
                const int jbeg = (int)(rb / wk.wt);
                bool waited = false;
                for (int j0 = jbeg; j0 < i_work; j0 += kChainBatch) {
                    const int nl = min(kChainBatch, i_work - j0);
                    named_bar_sync(1, kComputeThreads);  // the previous batch is consumed
                    if (tid < nl) {
                        int s0, s1;
                        row_piece(wk, d.seqlen, work_begin(wk, j0 + tid), work_end(wk, j0 + tid), r, s0, s1);
                        int sl = 0, cont = s0 > 0;
                        if (seq_idx) {
                            sl = seq_clamped(seq_idx, row, s1 - 1, d.nseq);
                            cont = s0 > 0 && seq_clamped(seq_idx, row, s0, d.nseq) == sl &&
                                   seq_clamped(seq_idx, row, s0 - 1, d.nseq) == sl;
                        }
                        chain_sl[tid] = sl;
                        chain_cont[tid] = cont;
                    }
                    named_bar_sync(1, kComputeThreads);
                    if (!waited) {
                        griddep_wait();  // the range states come from the kernel before this one
                        waited = true;
                    }
                    int l0 = 0;
                    if constexpr (kSeq) {  // the pieces before the last sequence start drop out
                        l0 = nl - 1;
                        while (l0 > 0 && chain_cont[l0]) --l0;
                    }
                    for (int l = l0; l < nl; ++l) {
                        const int j = j0 + l;
                        const bool cont = chain_cont[l] != 0;
                        const float a = work_decay[(int64_t)j * 2 + sh];
                        const float* loc = work_local + ((int64_t)j * 2 + sh) * N * kP;
                        const float* is = cont ? nullptr : init_src(b, hp, chain_sl[l]);
#pragma unroll
                        for (int i = 0; i < NQ; ++i) {
                            const int64_t n = cq * NQ + i;
                            const float start = cont ? hv[i] : (is ? is[n * P + sp] : 0.f);
                            hv[i] = fmaf(a, start, loc[n * kP + sp]);
                        }
                    }
                }
                if (seq_idx) {
                    const int sf = seq_clamped(seq_idx, row, s_cut, d.nseq);
                    if (seq_clamped(seq_idx, row, s_cut - 1, d.nseq) != sf) load_state(hv, init_src(b, hp, sf), P);
                }
            }
            write_hs(hv);
            st_state_scaled(hv, csb[0].dec[sh]);
            tmem_wait_st();
        }
        fence_async_shared();
        tc_fence_before();
        signal(&bar_st);

        const int eh = cq >> 1, p0 = 32 * (cq & 1);  // epilogue: head and first p of this thread
        for (int t = 0;; ++t) {
            const uint32_t par = t & 1;
            const int st = t & 1;
            // the descriptors are read from the decay buffers where they are used:
            // held in registers across the loop they spill at the register cap
            const TileDesc& cur = csb[t & (kCsBufs - 1)].td;
            const bool fin = (cur.flags & kTileFinal) != 0;
            const float* ct = csb[t & (kCsBufs - 1)].c[eh];
            uint8_t* Xst = smem + S::oX + st * S::kX + eh * kBox;
            const int64_t rowt = (int64_t)cur.b * d.seqlen;

            // the next tile's column factor tables while Y(t) is computed
            const TileDesc& nx = csb[(t + 1) & (kCsBufs - 1)].td;  // read only when !fin
            if (!fin) {
                wait_cs(t + 1);
                lg_tables(t + 1);
            }
            // ---- epilogue(t): Y staged in Hs (or stored), X' = w X in place ----
            const float ck_e = ct[k], cend_e = ct[cur.v - 1];
            const float rs = ex2_approx(ck_e);                               // decay from the tile start
            const float wx = k < cur.v ? ex2_approx(cend_e - ck_e) : 0.f;  // decay to the tile end
            mbar_wait(&bar_yd, par);
            mbar_wait(&bar_yo, par);
            tc_fence_after();
            {
                const __nv_bfloat162 wx2 = __floats2bfloat162_rn(wx, wx);
                const bool yvalid = valid_of(cur, eh);
                const int64_t yoff = ((rowt + cur.ts + k) * d.nheads + head_of(cur, eh)) * (int64_t)P +
                                     p0_of(cur, eh) + p0;
                __nv_bfloat16* yrow = Y + yoff;
#pragma unroll 1
                for (int hf = 0; hf < 2; ++hf) {
                    // a later state slice: the Y this thread's outputs add to
                    uint4 ya[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
                    if (kAcc && k < cur.v && yvalid) {
#pragma unroll
                        for (int c = 0; c < 2; ++c) ya[c] = *reinterpret_cast<const uint4*>(Y + yoff + 8 * (2 * hf + c));
                    }
                    uint32_t yd[16], yo[16];
                    tmem_ld16_async(tm_yd + lane_off + 32 * cq + 16 * hf, yd);
                    tmem_ld16_async(tm_yo + lane_off + 32 * cq + 16 * hf, yo);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const int c16 = (p0 >> 3) + 2 * hf + c;
                        const uint32_t off = sw128_off(k, c16);
                        uint4 xv = *reinterpret_cast<const uint4*>(Xst + off);
                        uint32_t* xu = reinterpret_cast<uint32_t*>(&xv);
                        uint32_t out[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const __nv_bfloat162 xb = *reinterpret_cast<const __nv_bfloat162*>(&xu[i]);
                            const int e0 = 8 * c + 2 * i;  // of this half; D x is in Y_diag (L o G diagonal)
                            float2 yy = __ffma2_rn(make_float2(rs, rs),
                                                   make_float2(__uint_as_float(yo[e0]), __uint_as_float(yo[e0 + 1])),
                                                   make_float2(__uint_as_float(yd[e0]), __uint_as_float(yd[e0 + 1])));
                            if (kAcc) {
                                const float2 pv = __bfloat1622float2(
                                    *reinterpret_cast<const __nv_bfloat162*>(reinterpret_cast<const uint32_t*>(&ya[c]) + i));
                                yy.x += pv.x;
                                yy.y += pv.y;
                            }
                            out[i] = pack_bf16(yy.x, yy.y);
                            const __nv_bfloat162 xs = __hmul2(xb, wx2);
                            xu[i] = *reinterpret_cast<const uint32_t*>(&xs);
                        }
                        const uint4 ov = make_uint4(out[0], out[1], out[2], out[3]);
                        if (cur.v == 128) *reinterpret_cast<uint4*>(Hs + eh * kBox + off) = ov;  // Y_off(t) has read Hs
                        else if (k < cur.v && yvalid) *reinterpret_cast<uint4*>(yrow + 8 * (c16 - (p0 >> 3))) = ov;
                        *reinterpret_cast<uint4*>(Xst + off) = xv;
                    }
                }
            }
            fence_async_shared();
            tc_fence_before();
            signal(&bar_epi);

            // ---- L o G(t+1) while H += X'^T B runs ----
            if (!fin) build_lg(t + 1);

            // ---- state(t): H(t) to Hs (bf16) and to the final states; pre-scale for t+1 ----
            mbar_wait(&bar_s, par);
            mbar_wait(&bar_free, par);
            tc_fence_after();
            {
                float hv[NQ];
                ld_state(hv);
                if (cur.flags & kTileLast) {
                    float* f = final_states && (cur.flags & kTileSeqEnd) ? final_dst(cur.b, cur.hp, cur.sid) : nullptr;
                    if (f) {
#pragma unroll
                        for (int i = 0; i < NQ; ++i) f[(int64_t)(cq * NQ + i) * P + sp] = hv[i];
                    }
                    // the next tile starts a new sequence or a new row
                    if (!fin) {
                        load_state(hv, init_src(nx.b, nx.hp, nx.sid), P);
                        fill_gap(nx);
                    }
                }
                // ids after the row's last sequence never occur: they keep their initial state
                if ((cur.flags & kTileRowEnd) && final_states && seq_idx) {
                    for (int sq = cur.sid + 1; sq < d.nseq; ++sq) {
                        float* f = final_dst(cur.b, cur.hp, sq);
                        if (!f) continue;
                        const float* src = init_src(cur.b, cur.hp, sq);
#pragma unroll 1
                        for (int i = 0; i < NQ; ++i) {
                            const int64_t o = (int64_t)(cq * NQ + i) * P + sp;
                            f[o] = src ? src[o] : 0.f;
                        }
                    }
                }
                if (!fin) {
                    write_hs(hv);
                    st_state_scaled(hv, csb[(t + 1) & (kCsBufs - 1)].dec[sh]);
                    tmem_wait_st();
                }
            }
            fence_async_shared();
            tc_fence_before();
            signal(&bar_st);
            signal(&bar_csfree[t & (kCsBufs - 1)]);  // done with tile t's decay data
            if (fin) break;
        }
    }
    tc_fence_before();
    __syncthreads();
    wait_guard_finish();
    if (warp == 0) tmem_dealloc(tmem_base, 512);
}

}  // namespace

// ---------------------------------------------------------------------------
// host
// ---------------------------------------------------------------------------
namespace {

template <typename K>
cudaError_t set_smem_attr(K kernel, int bytes, int slot) {
    return ensure_smem_attr(reinterpret_cast<const void*>(kernel), bytes, slot);
}

// the scan instantiation for (accumulate into Y, general slot mapping, sequence ids)
template <int N>
auto scan_instance(bool acc, bool gen, bool sq) {
    decltype(&fused_scan_kernel<N, false, false, false>) const k[2][2][2] = {
        {{fused_scan_kernel<N, false, false, false>, fused_scan_kernel<N, false, false, true>},
         {fused_scan_kernel<N, false, true, false>, fused_scan_kernel<N, false, true, true>}},
        {{fused_scan_kernel<N, true, false, false>, fused_scan_kernel<N, true, false, true>},
         {fused_scan_kernel<N, true, true, false>, fused_scan_kernel<N, true, true, true>}}};
    return k[acc][gen][sq];
}

template <int N>
int fused_smem_bytes() {
    return (int)FusedSmem<N>::oTail + 1024;
}

// SM count of the current device, cached per device (host threads may call
// concurrently: the cache is atomic, and a race only repeats the query)
int num_sms() {
    static std::atomic<int> n[16];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) {
        cudaGetLastError();
        return 148;
    }
    int v = n[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
        cudaGetLastError();
        v = 148;
    }
    n[dev].store(v, std::memory_order_relaxed);
    return v;
}

// pair rows per batch row: head pairs of each group (the last one half empty
// when a group has an odd number of heads), or single heads with headdim 128
int pair_rows(const Dims& d) {
    if (d.headdim == 2 * kP) return d.nheads;
    return d.ngroups * ((d.heads_per_group + 1) / 2);
}

Work make_work(const Dims& d, int64_t work_tiles) {
    Work w;
    w.npairs = pair_rows(d);
    w.nt = (d.seqlen + 127) / 128;
    w.total = (int64_t)d.batch * w.npairs * w.nt;
    w.wt = (int)work_tiles;
    w.nwork = (int)((w.total + work_tiles - 1) / work_tiles);
    return w;
}

}  // namespace

bool fused_supported(const ssd_problem* p) {
    if (p->dtype != SSD_DTYPE_BF16 || p->headdim != kP) return false;
    if (p->dstate != 64 && p->dstate != 128) return false;
    if ((p->nheads / p->ngroups) % 2 != 0) return false;
    return true;
}

bool fused_fwd_supported(const ssd_problem* p) {
    if (p->dtype != SSD_DTYPE_BF16) return false;
    if (p->headdim != kP && p->headdim != 2 * kP) return false;  // pairs of 64-column slots
    if (p->dstate % 16 != 0 || p->dstate > 256) return false;
    return true;
}

bool fused_work_ok(const Dims& d, int64_t work_tiles) {
    const int64_t total = (int64_t)d.batch * pair_rows(d) * ((d.seqlen + 127) / 128);
    if (work_tiles < 1 || work_tiles > total) return false;
    return (total + work_tiles - 1) / work_tiles <= (int64_t)1 << 30;
}

int64_t fused_work_count(const Dims& d, int64_t work_tiles) { return make_work(d, work_tiles).nwork; }

bool fused_needs_cut_states(const Dims& d, int64_t work_tiles) {
    const Work w = make_work(d, work_tiles);
    return w.nwork > 1 && work_tiles % w.nt != 0;
}

// Tiles per work range: the line of tiles split evenly over the SMs (one CTA
// per SM), so that every CTA has the same number of tiles to walk. (Whole rows
// per CTA, which need no cut states, measured slower on the 130M-shaped layer:
// 72.4 against 69.5 us with 96 of 148 SMs busy.)
int fused_default_work_tiles(const Dims& d) {
    const int64_t total = (int64_t)d.batch * pair_rows(d) * ((d.seqlen + 127) / 128);
    const int64_t g = std::min<int64_t>(num_sms(), total);
    return (int)((total + g - 1) / g);
}

size_t fused_workspace_bytes(const Dims& d, int64_t work_tiles) {
    const size_t nwork = (size_t)make_work(d, work_tiles).nwork;
    const size_t st = nwork * 2 * d.dstate * d.headdim * sizeof(float);
    const size_t dec = nwork * 2 * sizeof(float);
    const auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    return 2 * al(st) + al(dec);
}

cudaError_t launch_segment_state(const Dims& d, int64_t work_tiles, const void* X, const float* log_a, const void* B,
                                 const int32_t* seq_idx, float* work_local, float* work_decay, cudaStream_t st,
                                 int32_t* row_ids) {
    CUtensorMap mx, mb;
    cudaError_t e;
    unsigned int* err = nullptr;
    if ((e = device_error_word(&err)) != cudaSuccess) return e;
    if ((e = x_map(&mx, d, X, 128)) != cudaSuccess) return e;
    if ((e = bc_map(&mb, d, B, 128)) != cudaSuccess) return e;
    const Work w = make_work(d, work_tiles);
    const dim3 grid(w.nwork);
    const int smem = 3 * (2 * (int)kBox + (d.dstate / 64) * (int)kBox) + 1024;
    if (d.dstate == 64) {
        auto k = segment_state_kernel<64>;
        if ((e = set_smem_attr(k, smem, 30)) != cudaSuccess) return e;
        k<<<grid, kSegThreads, smem, st>>>(mx, mb, d, w, log_a, seq_idx, work_local, work_decay, row_ids != nullptr,
                                           row_ids, err);
    } else if (d.dstate == 128) {
        auto k = segment_state_kernel<128>;
        if ((e = set_smem_attr(k, smem, 31)) != cudaSuccess) return e;
        k<<<grid, kSegThreads, smem, st>>>(mx, mb, d, w, log_a, seq_idx, work_local, work_decay, row_ids != nullptr,
                                           row_ids, err);
    } else {
        return cudaErrorNotSupported;
    }
    return cudaGetLastError();
}

cudaError_t launch_segment_passing(const Dims& d, int64_t work_tiles, const float* work_local, const float* work_decay,
                                   const float* init_states, const int32_t* seq_idx, float* work_in, cudaStream_t st) {
    const Work w = make_work(d, work_tiles);
    const dim3 grid(2 * w.nwork, (d.dstate * d.headdim + 1023) / 1024);
    segment_passing_kernel<<<grid, 256, 0, st>>>(d, w, work_local, work_decay, init_states, seq_idx, work_in);
    return cudaGetLastError();
}

cudaError_t launch_fused_scan(const Dims& d, int64_t work_tiles, const void* X, const float* log_a, const void* B,
                              const void* C, const float* D, const float* work_in, const float* init_states,
                              const int32_t* seq_idx, void* Y, float* final_states, cudaStream_t st,
                              const float* work_local, const float* work_decay, bool after_segment_state,
                              const void* Yacc) {
    if (Yacc && Yacc != Y) return cudaErrorInvalidValue;  // the slices accumulate in place
    CUtensorMap mx, mb, mc, my;
    cudaError_t e;
    unsigned int* err = nullptr;
    if ((e = device_error_word(&err)) != cudaSuccess) return e;
    if ((e = x_map(&mx, d, X, 128)) != cudaSuccess) return e;
    if ((e = bc_map(&mb, d, B, 128)) != cudaSuccess) return e;
    if ((e = bc_map(&mc, d, C, 128)) != cudaSuccess) return e;
    if ((e = x_map(&my, d, Y, 128)) != cudaSuccess) return e;
    const Work w = make_work(d, work_tiles);
    // Right after segment_state in the same stream, the scan is launched as its
    // programmatic dependent: its CTAs start as segment_state's leave the SMs and
    // wait for that grid only before reading the range states. Everything the
    // scan reads before that wait was complete before segment_state started.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(w.nwork);
    cfg.blockDim = dim3(kFusedThreads);
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = after_segment_state ? 1 : 0;
    __nv_bfloat16* Yb = (__nv_bfloat16*)Y;
    // the general slot mapping (headdim 128, or an odd number of heads per group) is
    // its own instantiation, so that the plain head pairs keep their code
    const bool gen = d.headdim != kP || d.heads_per_group % 2 != 0;
    const bool sq = seq_idx != nullptr;
    const int slot = (Yacc ? 2 : 0) + (gen ? 4 : 0) + (sq ? 8 : 0);
    if (d.dstate == 64) {
        auto k = scan_instance<64>(Yacc != nullptr, gen, sq);
        cfg.dynamicSmemBytes = fused_smem_bytes<64>();
        if ((e = set_smem_attr(k, (int)cfg.dynamicSmemBytes, 40 + slot)) != cudaSuccess) return e;
        e = cudaLaunchKernelEx(&cfg, k, mx, mb, mc, my, d, w, log_a, D, work_in, init_states, seq_idx, Yb,
                               final_states, work_local, work_decay, err);
    } else if (d.dstate == 128) {
        auto k = scan_instance<128>(Yacc != nullptr, gen, sq);
        cfg.dynamicSmemBytes = fused_smem_bytes<128>();
        if ((e = set_smem_attr(k, (int)cfg.dynamicSmemBytes, 41 + slot)) != cudaSuccess) return e;
        e = cudaLaunchKernelEx(&cfg, k, mx, mb, mc, my, d, w, log_a, D, work_in, init_states, seq_idx, Yb,
                               final_states, work_local, work_decay, err);
    } else {
        return cudaErrorNotSupported;
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace ssd
