// ssd_fused.cu -- the fused tensor-core path of the SSD forward (bf16 in, fp32
// state): the block decomposition applied at two levels.
//
// The sequence is cut into segments of L tokens (a multiple of 128). Within a
// segment a CTA walks 128-token tiles and carries the state on chip from tile
// to tile; only one state per segment goes through HBM. Three kernels:
//
//   segment_state    per (batch row, head pair, segment): the end state of the
//                    segment's last sequence piece from a zero start,
//                    accumulated over its tiles in TMEM (the right factors of
//                    the block algorithm at segment level);
//   segment_passing  the short recurrence over segments (centre factors);
//   fused_scan       per (batch row, head pair, segment): for each tile the
//                    masked quadratic term (L o C B^T) X, the carried state read
//                    out by C, D x, and the carried state update
//                    H <- a(tile) H + sum_l a(l..end) B_l x_l^T.
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
// fused_scan is warp-specialised: 8 compute warps (the TMEM lane quarters are
// shared by warps w and w+4, which split the columns) and one control warp that
// issues TMA loads/stores and tcgen05.mma, handshaking through mbarriers.
// Tensor memory (512 columns): G = C B^T [0,128), L o G (bf16, the A operand of
// a TS-MMA) and later the tile state S [128,256), Y_diag [256,384), Y_off [384,512).

#include <cuda.h>

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

// first index in [lo, hi) of the row whose id is >= v (ids non-decreasing)
__device__ int lower_bound_global(const int32_t* seq_idx, int64_t row, int lo, int hi, int v, int nseq) {
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (seq_clamped(seq_idx, row, mid, nseq) < v) lo = mid + 1;
        else hi = mid;
    }
    return lo;
}

// ===========================================================================
// segment_state
// ===========================================================================
constexpr int kSegThreads = 256;

template <int N>
__global__ void __launch_bounds__(kSegThreads, 1)
    segment_state_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b, Dims d,
                         int seglen, int nseg, const float* __restrict__ log_a, const int32_t* __restrict__ seq_idx,
                         float* __restrict__ seg_states, float* __restrict__ seg_decay) {
    constexpr uint32_t kXB = 2 * kBox, kBB = (N / 64) * kBox;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* Xs = smem;
    uint8_t* Bs = smem + kXB;
    __shared__ float wsum[8];
    __shared__ float tail_s[2];
    __shared__ int st_shared;
    __shared__ __align__(8) uint64_t bar_load, bar_mma;
    __shared__ uint32_t tmem_base;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int npairs = d.nheads / 2;
    int r = blockIdx.x;
    const int j = r % nseg;
    r /= nseg;
    const int hp = r % npairs, b = r / npairs;
    const int h0 = 2 * hp, g = h0 / d.heads_per_group;
    const int s0 = j * seglen, s1 = min(d.seqlen, s0 + seglen);
    const int64_t row = (int64_t)b * d.seqlen;

    if (tid == 0) {
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_b);
        mbar_init(&bar_load, 1);
        mbar_init(&bar_mma, 1);
        mbar_fence_init();
        // start of the segment's last sequence piece
        int st = s0;
        if (seq_idx) {
            const int sl = seq_clamped(seq_idx, row, s1 - 1, d.nseq);
            st = lower_bound_global(seq_idx, row, s0, s1 - 1, sl, d.nseq);
        }
        st_shared = st;
        tail_s[0] = tail_s[1] = 0.f;
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
    const int rr = tid & 127, hh = tid >> 7;  // this thread's row and head in the transform
    const uint32_t idesc = idesc_bf16(128, N, true, true);
    float tail = 0.f;  // sum of log a after the current tile, this thread's head
    bool cut = false;
    int done = 0;
    // log a of this thread's (row, head) in a tile; unconditional (clamped row)
    // so that the prefetch does not stall until the value is used
    auto load_la = [&](int i) -> float {
        const int ts = st + 128 * i;
        const int v = min(128, s1 - ts);
        return log_a[(row + ts + min(rr, v - 1)) * d.nheads + h0 + hh];
    };
    float la_cur = load_la(ntiles - 1);
    for (int i = ntiles - 1; i >= 0; --i) {
        const int ts = st + 128 * i;
        const int v = min(128, s1 - ts);
        const float la_nxt = i > 0 ? load_la(i - 1) : 0.f;
        if (tid == 0) {
            mbar_arrive_expect_tx(&bar_load, kXB + kBB);
            tma_load_4d(Xs, &tm_x, &bar_load, 0, h0, ts, b);
            tma_load_4d(Xs + kBox, &tm_x, &bar_load, 0, h0 + 1, ts, b);
#pragma unroll
            for (int q = 0; q < N / 64; ++q) tma_load_4d(Bs + q * kBox, &tm_b, &bar_load, 64 * q, g, ts, b);
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
        __syncthreads();
        float pre = 0.f, tot = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const float s = wsum[4 * hh + w];
            if (w < (warp & 3)) pre += s;
            tot += s;
        }
        const float cs = x + pre;
        // weight of row rr: prod of a over (rr, segment end] = exp(tail + tot - cs)
        const float wgt = rr < v ? ex2_approx((tail + tot - cs) * kLog2e) : 0.f;
        mbar_wait(&bar_load, done & 1);
        // scale row rr of head hh in place; the chunk order is rotated by row so
        // that the 32 rows of a warp spread over all banks
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
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t xa = smem_u32(Xs), ba = smem_u32(Bs);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_bf16_ss(tacc, smem_desc_sw128(xa + k * 2048, kBox, 1024), smem_desc_sw128(ba + k * 2048, kBox, 1024),
                            idesc, (done > 0 || k > 0) ? 1u : 0u);
            mma_commit(&bar_mma);
        }
        mbar_wait(&bar_mma, done & 1);
        ++done;
        tail += tot;
        if (rr == 0) tail_s[hh] = tail;
        __syncthreads();
        // everything further back decays below fp32 range for both heads
        if (tail_s[0] < -104.f && tail_s[1] < -104.f && i > 0) {
            cut = true;
            break;
        }
    }
    tc_fence_after();
    // epilogue: lane m = (head, p); warps w and w+4 split the N columns
    const int m = 32 * (warp & 3) + lane, half = warp >> 2;
    const int eh = m >> 6, p = m & 63;
    float* dst = seg_states + (((int64_t)b * nseg + j) * d.nheads + h0 + eh) * (int64_t)N * kP;
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
        seg_decay[((int64_t)b * nseg + j) * d.nheads + h0 + tid] = cut ? 0.f : ex2_approx(t * kLog2e);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tacc, N);
}

// ===========================================================================
// segment_passing: H_end(j) = decay(j) * H_start(j) + S(j) over segments, and
// over S(j), in place, the state entering segment j for the sequence of its
// first token: H_end(j-1) when that sequence continues from segment j-1, else
// its initial state (or zero).
// ===========================================================================
__global__ void __launch_bounds__(256) segment_passing_kernel(Dims d, int seglen, int nseg, float* seg_states,
                                                              const float* __restrict__ seg_decay,
                                                              const float* __restrict__ init_states,
                                                              const int32_t* __restrict__ seq_idx) {
    __shared__ int info[4];  // last id, last piece continues, first id, first token continues
    const int bh = blockIdx.x;
    const int h = bh % d.nheads, b = bh / d.nheads;
    const int NP = d.dstate * d.headdim;
    const int idx = (blockIdx.y * 256 + threadIdx.x) * 4;
    const bool active = idx < NP;
    const int64_t row = (int64_t)b * d.seqlen;
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    auto init_of = [&](int sq) -> float4 {
        if (!init_states) return zero;
        return *reinterpret_cast<const float4*>(init_states + seqst_off(d, b, sq, h) + idx);
    };
    float4 H = zero;
    for (int j = 0; j < nseg; ++j) {
        const int s0 = j * seglen, s1 = min(d.seqlen, s0 + seglen);
        __syncthreads();
        if (threadIdx.x == 0) {
            int sl = 0, cont_last = (j > 0), sf = 0, cont_first = (j > 0);
            if (seq_idx) {
                sl = seq_clamped(seq_idx, row, s1 - 1, d.nseq);
                sf = seq_clamped(seq_idx, row, s0, d.nseq);
                const int st = lower_bound_global(seq_idx, row, s0, s1 - 1, sl, d.nseq);
                const int prev = s0 > 0 ? seq_clamped(seq_idx, row, s0 - 1, d.nseq) : -1;
                cont_last = (st == s0) && prev == sl;
                cont_first = prev == sf;
            }
            info[0] = sl;
            info[1] = cont_last;
            info[2] = sf;
            info[3] = cont_first;
        }
        __syncthreads();
        float* S = seg_states + ((int64_t)b * nseg + j) * d.nheads * (int64_t)NP + (int64_t)h * NP;
        const float dec = seg_decay[((int64_t)b * nseg + j) * d.nheads + h];
        if (!active) continue;
        const float4 s = *reinterpret_cast<const float4*>(S + idx);
        *reinterpret_cast<float4*>(S + idx) = info[3] ? H : init_of(info[2]);
        const float4 st = info[1] ? H : init_of(info[0]);
        H = make_float4(fmaf(dec, st.x, s.x), fmaf(dec, st.y, s.y), fmaf(dec, st.z, s.z), fmaf(dec, st.w, s.w));
    }
}

// ===========================================================================
// fused_scan
// ===========================================================================
constexpr int kComputeWarps = 16;
constexpr int kComputeThreads = 32 * kComputeWarps;
constexpr int kFusedThreads = kComputeThreads + 32;  // + one control warp

template <int N>
struct FusedSmem {
    static constexpr uint32_t kC = (N / 64) * kBox;
    static constexpr uint32_t kB = (N / 64) * kBox;  // per stage
    static constexpr uint32_t kX = 2 * kBox;         // per stage, two heads
    static constexpr uint32_t kH = (N / 64) * kBox;  // carried state, bf16, rows (h,p), K = n
    static constexpr uint32_t kHY = kH > 2 * kBox ? kH : 2 * kBox;  // ... and the Y staging of a tile
    static constexpr uint32_t oC = 0, oB = kC, oX = oB + 2 * kB, oH = oX + 2 * kX, oTail = oH + kHY;
};

// One tile: first token, valid rows, and flags.
struct Tile {
    int ts, v;
    int first;     // first tile of its sequence piece
    int last;      // last tile of its sequence piece
};

__device__ __forceinline__ Tile unpack_tile(int2 e) {
    Tile t;
    t.ts = e.x;
    t.v = e.y & 0xFF;
    if (t.v == 0) t.v = 128;
    t.first = (e.y >> 8) & 1;
    t.last = (e.y >> 9) & 1;
    return t;
}

// Thread layout of the 16 compute warps: warp w owns the TMEM lane quarter
// w % 4 (rows 32 (w % 4) .. +31) and the column quarter w / 4 of every
// 128-column accumulator it touches; the four warps of a lane quarter split
// the columns.
//
// Per tile t the compute warps run, in this order,
//   epilogue(t):  Y = Y_diag + rscale Y_off + D x, staged (bf16) in the buffer
//                 of the carried state, which Y_off(t) has finished reading, for
//                 the TMA store; X' = w X in place in the tile's X buffer;
//   L o G(t+1):   the next tile's masked C B^T, written over G in TMEM (while
//                 the tile state MMA of tile t runs and Y(t) drains);
//   state(t):     the carried state H(t) (in TMEM: the tile state MMA adds
//                 X'^T B onto it) to bf16 for the next C H and to the final
//                 states, then pre-scaled by the next tile's decay.
// Tensor memory: G, then L o G in place [0,128); Y_diag [128,256);
// Y_off [256,384); the carried state H [384,512) (rows (head, p), N columns).
template <int N>
__global__ void __launch_bounds__(kFusedThreads, 1)
    fused_scan_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                      const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y, Dims d,
                      int seglen, int nseg, const float* __restrict__ log_a, const float* __restrict__ Dv,
                      const float* __restrict__ seg_incoming, const float* __restrict__ init_states,
                      const int32_t* __restrict__ seq_idx, __nv_bfloat16* __restrict__ Y,
                      float* __restrict__ final_states) {
    using S = FusedSmem<N>;
    constexpr int NQ = N / 4;  // state columns per thread
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* Cs = smem + S::oC;
    uint8_t* Hs = smem + S::oH;
    int* seq_s = reinterpret_cast<int*>(smem + S::oTail);  // [seglen] ids of the segment (varlen only)
    int2* tiles = reinterpret_cast<int2*>(seq_s + (seq_idx ? seglen : 0));  // tile list
    __shared__ __align__(16) float cs2[2][2][128];  // [buffer][head][row]: log2-scaled within-tile cumsum
    __shared__ __align__(16) float colf[kComputeWarps][2][32];  // per-warp column factors
    __shared__ float wsum[8];
    __shared__ int ntiles_s, lastid_s;
    __shared__ __align__(8) uint64_t bar_c, bar_bx[2], bar_g, bar_yo, bar_yd, bar_s, bar_lg, bar_epi, bar_st,
        bar_free;
    __shared__ uint32_t tmem_base;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int npairs = d.nheads / 2;
    int r = blockIdx.x;
    const int j = r % nseg;
    r /= nseg;
    const int hp = r % npairs, b = r / npairs;
    const int h0 = 2 * hp, g = h0 / d.heads_per_group;
    const int s0 = j * seglen, s1 = min(d.seqlen, s0 + seglen);
    const int64_t row = (int64_t)b * d.seqlen;
    const int L = s1 - s0;

    // ---- setup: barriers, TMEM, the segment's ids and tile list ----
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
        mbar_init(&bar_lg, kComputeWarps);
        mbar_init(&bar_epi, kComputeWarps);
        mbar_init(&bar_st, kComputeWarps);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, 512);
        tmem_relinquish();
    }
    if (seq_idx)
        for (int k = tid; k < L; k += kFusedThreads) seq_s[k] = seq_clamped(seq_idx, row, s0 + k, d.nseq);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        // tiles aligned to the starts of the sequence pieces of [s0, s1)
        int n = 0, pos = s0;
        while (pos < s1) {
            int pend = s1;
            if (seq_idx) {  // end of the piece containing pos
                const int v = seq_s[pos - s0];
                int lo = pos - s0, hi = L;
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if (seq_s[mid] <= v) lo = mid + 1;
                    else hi = mid;
                }
                pend = s0 + lo;
            }
            for (int ts = pos; ts < pend; ts += 128) {
                const int v = min(128, pend - ts);
                tiles[n++] = make_int2(ts, (v & 0xFF) | ((ts == pos) << 8) | ((ts + v == pend) << 9));
            }
            pos = pend;
        }
        ntiles_s = n;
        lastid_s = seq_idx ? seq_s[L - 1] : 0;
    }
    __syncthreads();
    const int ntiles = ntiles_s;
    const uint32_t tm_g = tmem_base, tm_lg = tmem_base, tm_yd = tmem_base + 128, tm_yo = tmem_base + 256,
                   tm_h = tmem_base + 384;

    if (warp == kComputeWarps) {
        // =================== control warp: TMA and MMA issue ===================
        if (lane == 0) {
            const uint32_t idesc_nn = idesc_bf16(128, 128, false, false);   // K-major A and B
            const uint32_t idesc_ts = idesc_bf16(128, 64, false, true);     // TMEM A, MN-major B
            const uint32_t idesc_st = idesc_bf16(128, N, true, true);       // MN-major A and B
            auto load_bx = [&](int t) {
                const Tile tl = unpack_tile(tiles[t]);
                const int st = t & 1;
                uint8_t* Bsg = smem + S::oB + st * S::kB;
                uint8_t* Xsg = smem + S::oX + st * S::kX;
                mbar_arrive_expect_tx(&bar_bx[st], S::kB + S::kX);
#pragma unroll
                for (int q = 0; q < N / 64; ++q) tma_load_4d(Bsg + q * kBox, &tm_b, &bar_bx[st], 64 * q, g, tl.ts, b);
                tma_load_4d(Xsg, &tm_x, &bar_bx[st], 0, h0, tl.ts, b);
                tma_load_4d(Xsg + kBox, &tm_x, &bar_bx[st], 0, h0 + 1, tl.ts, b);
            };
            auto load_c = [&](int t) {
                const Tile tl = unpack_tile(tiles[t]);
                mbar_arrive_expect_tx(&bar_c, S::kC);
#pragma unroll
                for (int q = 0; q < N / 64; ++q) tma_load_4d(Cs + q * kBox, &tm_c, &bar_c, 64 * q, g, tl.ts, b);
            };
            const uint32_t ca = smem_u32(Cs), ha = smem_u32(Hs);
            auto issue_g = [&](int t) {
                const uint32_t ba = smem_u32(smem + S::oB + (t & 1) * S::kB);
#pragma unroll
                for (int k = 0; k < N / 16; ++k) {
                    const uint32_t off = (k >> 2) * kBox + (k & 3) * 32;
                    mma_bf16_ss(tm_g, smem_desc_sw128(ca + off, 16, 1024), smem_desc_sw128(ba + off, 16, 1024),
                                idesc_nn, k > 0 ? 1u : 0u);
                }
                mma_commit(&bar_g);
            };
            load_c(0);
            load_bx(0);
            if (ntiles > 1) load_bx(1);
            mbar_wait(&bar_c, 0);
            mbar_wait(&bar_bx[0], 0);
            tc_fence_after();
            issue_g(0);
            for (int t = 0; t < ntiles; ++t) {
                const int st = t & 1;
                const uint32_t par = t & 1;
                const Tile tl = unpack_tile(tiles[t]);
                const uint32_t xa = smem_u32(smem + S::oX + st * S::kX);
                const uint32_t ba = smem_u32(smem + S::oB + st * S::kB);
                // Y_diag = (L o G) X, A operand from TMEM: L o G(t) is built before
                // state(t-1), so this runs while the state update does
                mbar_wait(&bar_lg, par);
                tc_fence_after();
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_bf16_ts(tm_yd + 64 * hh, tm_lg + 64 * hh + 8 * k,
                                    smem_desc_sw128(xa + hh * kBox + k * 2048, kBox, 1024), idesc_ts, k > 0 ? 1u : 0u);
                mma_commit(&bar_yd);
                // Y_off = C Hs once the state before this tile is in Hs
                mbar_wait(&bar_st, par);
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < N / 16; ++k) {
                    const uint32_t off = (k >> 2) * kBox + (k & 3) * 32;
                    mma_bf16_ss(tm_yo, smem_desc_sw128(ca + off, 16, 1024), smem_desc_sw128(ha + off, 16, 1024),
                                idesc_nn, k > 0 ? 1u : 0u);
                }
                mma_commit(&bar_yo);
                // C is free once G(t) and Y_off(t) have read it; G(t+1) once its
                // operands are in and Y_diag(t) has read L o G(t) from the same columns
                if (t + 1 < ntiles) {
                    mbar_wait(&bar_yo, par);
                    load_c(t + 1);
                    mbar_wait(&bar_c, (t + 1) & 1);
                    mbar_wait(&bar_bx[st ^ 1], ((t + 1) >> 1) & 1);
                    mbar_wait(&bar_yd, par);
                    tc_fence_after();
                    issue_g(t + 1);
                }
                // epilogue done: store Y(t) from the staging buffer; H += X'^T B
                mbar_wait(&bar_epi, par);
                tc_fence_after();
                const bool full = tl.v == 128;
                if (full) {
                    tma_store_4d(&tm_y, Hs, 0, h0, tl.ts, b);
                    tma_store_4d(&tm_y, Hs + kBox, 0, h0 + 1, tl.ts, b);
                    tma_store_commit();
                }
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_bf16_ss(tm_h, smem_desc_sw128(xa + k * 2048, kBox, 1024), smem_desc_sw128(ba + k * 2048, kBox, 1024),
                                idesc_st, 1u);
                mma_commit(&bar_s);
                if (full) tma_store_wait_read0();
                mbar_arrive(&bar_free);
                // this stage is free once the tile state has been added
                if (t + 2 < ntiles) {
                    mbar_wait(&bar_s, par);
                    load_bx(t + 2);
                }
            }
        }
        __syncwarp();
    } else {
        // =================== compute warps ===================
        const int q4 = warp & 3, cq = warp >> 2;
        const int m = 32 * q4 + lane;           // TMEM lane: token row, or (head, p) for states
        const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
        const int sh = m >> 6, sp = m & 63;     // state row (head, p) of lane m

        auto signal = [&](uint64_t* bar) {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar);
        };
        // log a of tile t for (head warp/4, row 32 (warp%4) + lane), warps 0..7; the
        // load is unconditional (clamped row) so that it does not stall until used
        auto load_la = [&](int t) -> float {
            if (warp >= 8 || t >= ntiles) return 0.f;
            const Tile tl = unpack_tile(tiles[t]);
            const int hh = warp >> 2, rr = min(32 * (warp & 3) + lane, tl.v - 1);
            return log_a[(row + tl.ts + rr) * d.nheads + h0 + hh];
        };
        // within-tile cumsum of log a * log2(e) for tile t into buffer t & 1
        auto tile_cumsum = [&](int t, float la_raw) {
            const int hh = (warp >> 2) & 1, rr = 32 * (warp & 3) + lane;
            float x = 0.f;
            if (warp < 8) {
                const Tile tl = unpack_tile(tiles[t]);
                x = rr < tl.v ? la_raw * kLog2e : 0.f;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x, o);
                    if (lane >= o) x += y;
                }
                if (lane == 31) wsum[warp] = x;
            }
            named_bar_sync(1, kComputeThreads);
            if (warp < 8) {
                float pre = 0.f;
#pragma unroll
                for (int w = 0; w < 3; ++w)
                    if (w < (warp & 3)) pre += wsum[4 * hh + w];
                cs2[t & 1][hh][rr] = x + pre;
            }
            named_bar_sync(1, kComputeThreads);
        };
        // L o G of tile t into TMEM (bf16): row m, columns [32 cq, 32 cq + 32), both heads.
        // Above the diagonal block 0; on it exp(c_m - c_l) for l <= m; below it
        // exp(c_m - c_r0) * exp(c_r0 - c_l) with r0 = 32 q4 (both factors <= 1).
        auto build_lg = [&](int t) {
            const float* c2 = &cs2[t & 1][0][0];
            const int r0 = 32 * q4, cb = 32 * cq;
            const float ck0 = c2[m], ck1 = c2[128 + m];
            float rf0 = 0.f, rf1 = 0.f;
            if (cq < q4) {  // below the diagonal: ref r0, column factors of this warp's 32 columns
                const float cr0 = c2[r0], cr1 = c2[128 + r0];
                rf0 = ex2_approx(ck0 - cr0);
                rf1 = ex2_approx(ck1 - cr1);
                colf[warp][0][lane] = ex2_approx(cr0 - c2[cb + lane]);
                colf[warp][1][lane] = ex2_approx(cr1 - c2[128 + cb + lane]);
                __syncwarp();
            } else if (cq == q4) {  // diagonal: lower-left 16x16 quarter, ref = r0 + 15
                const float cref0 = c2[r0 + 15], cref1 = c2[128 + r0 + 15];
                rf0 = lane >= 16 ? ex2_approx(ck0 - cref0) : 0.f;
                rf1 = lane >= 16 ? ex2_approx(ck1 - cref1) : 0.f;
                if (lane < 16) {
                    colf[warp][0][lane] = ex2_approx(cref0 - c2[r0 + lane]);
                    colf[warp][1][lane] = ex2_approx(cref1 - c2[128 + r0 + lane]);
                }
                __syncwarp();
            }
            mbar_wait(&bar_g, t & 1);
            tc_fence_after();
            // this warp's 32 G columns, read by all warps of the lane quarter before
            // any of them writes L o G over the same columns
            uint32_t ga[16], gb[16];
            if (cq <= q4) {
                tmem_ld16_async(tm_g + lane_off + cb, ga);
                tmem_ld16_async(tm_g + lane_off + cb + 16, gb);
                tmem_wait_ld();
            }
            named_bar_sync(2 + q4, 128);
            if (cq > q4) {
                uint32_t z[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) z[i] = 0u;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    tmem_st8(tm_lg + lane_off + 16 * cq + 8 * hf, z);
                    tmem_st8(tm_lg + lane_off + 64 + 16 * cq + 8 * hf, z);
                }
            } else if (cq < q4) {
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {  // 16 columns at a time
                    uint32_t w0[8], w1[8];
                    const uint32_t* gr = hf ? gb : ga;
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        const float4 a = *reinterpret_cast<const float4*>(&colf[warp][0][16 * hf + 4 * v4]);
                        const float4 bq = *reinterpret_cast<const float4*>(&colf[warp][1][16 * hf + 4 * v4]);
                        const float g0 = __uint_as_float(gr[4 * v4]), g1 = __uint_as_float(gr[4 * v4 + 1]);
                        const float g2 = __uint_as_float(gr[4 * v4 + 2]), g3 = __uint_as_float(gr[4 * v4 + 3]);
                        w0[2 * v4] = pack_bf16(g0 * rf0 * a.x, g1 * rf0 * a.y);
                        w0[2 * v4 + 1] = pack_bf16(g2 * rf0 * a.z, g3 * rf0 * a.w);
                        w1[2 * v4] = pack_bf16(g0 * rf1 * bq.x, g1 * rf1 * bq.y);
                        w1[2 * v4 + 1] = pack_bf16(g2 * rf1 * bq.z, g3 * rf1 * bq.w);
                    }
                    // head h's packed L o G occupies columns [64 h, 64 h + 64) of the region
                    tmem_st8(tm_lg + lane_off + 16 * cq + 8 * hf, w0);
                    tmem_st8(tm_lg + lane_off + 64 + 16 * cq + 8 * hf, w1);
                }
            } else {
                // Diagonal block. Lanes 0..15 (rows r0..r0+15) own columns r0..r0+15,
                // lanes 16..31 own r0+16..r0+31: direct exps there (16 per lane and
                // head, issued as 16 instructions for the whole warp). Lanes 16..31
                // x columns r0..r0+15: exp(c_m - c_ref) exp(c_ref - c_l); lanes 0..15
                // x columns r0+16..: above the diagonal.
                const bool upper = lane < 16;
                const int own0 = cb + (upper ? 0 : 16);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const float ck = hh ? ck1 : ck0, rf = hh ? rf1 : rf0;
                    const float* crow = c2 + 128 * hh;
                    uint32_t o0[8], o1[8];
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        const float4 cv = *reinterpret_cast<const float4*>(crow + own0 + 4 * v4);
                        const float4 fv = *reinterpret_cast<const float4*>(&colf[warp][hh][4 * v4]);
                        const float cvs[4] = {cv.x, cv.y, cv.z, cv.w};
                        const float fvs[4] = {fv.x, fv.y, fv.z, fv.w};
                        float lo[4], hi[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int jj = 4 * v4 + e;
                            const float gown = __uint_as_float(upper ? ga[jj] : gb[jj]);
                            const float a = (own0 + jj <= m) ? gown * ex2_approx(ck - cvs[e]) : 0.f;
                            const float bq = upper ? 0.f : __uint_as_float(ga[jj]) * rf * fvs[e];
                            lo[e] = upper ? a : bq;  // column cb + jj
                            hi[e] = upper ? 0.f : a;  // column cb + 16 + jj
                        }
                        o0[2 * v4] = pack_bf16(lo[0], lo[1]);
                        o0[2 * v4 + 1] = pack_bf16(lo[2], lo[3]);
                        o1[2 * v4] = pack_bf16(hi[0], hi[1]);
                        o1[2 * v4 + 1] = pack_bf16(hi[2], hi[3]);
                    }
                    tmem_st8(tm_lg + lane_off + 64 * hh + 16 * cq, o0);
                    tmem_st8(tm_lg + lane_off + 64 * hh + 16 * cq + 8, o1);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            signal(&bar_lg);
        };
        auto piece_id = [&](int ts) -> int { return seq_idx ? seq_s[ts - s0] : 0; };
        auto seq_ends_at = [&](int pend) -> bool {  // does the sequence of token pend-1 end there?
            if (pend < s1) return true;
            if (pend >= d.seqlen) return true;
            return seq_idx ? seq_clamped(seq_idx, row, pend, d.nseq) != seq_s[pend - 1 - s0] : false;
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
        auto st_state_scaled = [&](const float (&v)[NQ], float a) {
#pragma unroll
            for (int h16 = 0; h16 < NQ / 16; ++h16) {
                float w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) w[i] = a * v[16 * h16 + i];
                tmem_st16f(tm_h + lane_off + NQ * cq + 16 * h16, w);
            }
        };
        auto load_state = [&](float (&v)[NQ], const float* src) {  // src: [N][P] of head sh, or null
#pragma unroll
            for (int i = 0; i < NQ; ++i) v[i] = src ? src[(int64_t)(cq * NQ + i) * kP + sp] : 0.f;
        };
        auto write_hs = [&](const float (&v)[NQ]) {  // bf16 state, row m, K-major over n
#pragma unroll
            for (int c8 = 0; c8 < NQ / 8; ++c8) {
                const int n = cq * NQ + 8 * c8;
                const uint4 u = make_uint4(pack_bf16(v[8 * c8], v[8 * c8 + 1]), pack_bf16(v[8 * c8 + 2], v[8 * c8 + 3]),
                                           pack_bf16(v[8 * c8 + 4], v[8 * c8 + 5]), pack_bf16(v[8 * c8 + 6], v[8 * c8 + 7]));
                *reinterpret_cast<uint4*>(Hs + (n >> 6) * kBox + sw128_off(m, (n & 63) >> 3)) = u;
            }
        };
        // decay of a whole tile for the head of state lane m (cs2 of that tile must be in)
        auto tile_decay = [&](int t) -> float {
            const Tile tl = unpack_tile(tiles[t]);
            return ex2_approx(cs2[t & 1][sh][tl.v - 1]);
        };

        // ---- prologue: the first piece's state, tile 0's cumsum and L o G ----
        {
            const Tile t0 = unpack_tile(tiles[0]);
            const int sid = piece_id(t0.ts);
            const float* src = nullptr;
            if (seg_incoming) src = seg_incoming + (((int64_t)b * nseg + j) * d.nheads + h0 + sh) * (int64_t)N * kP;
            else if (init_states) src = init_states + seqst_off(d, b, sid, h0 + sh);
            float hv[NQ];
            load_state(hv, src);
            write_hs(hv);
            tile_cumsum(0, load_la(0));
            st_state_scaled(hv, tile_decay(0));
            tmem_wait_st();
        }
        float la_next = load_la(1);
        fence_async_shared();
        tc_fence_before();
        signal(&bar_st);
        build_lg(0);

        const int eh = cq >> 1, p0 = 32 * (cq & 1);  // epilogue: head and first p of this thread
        const float dh = Dv ? Dv[h0 + eh] : 0.f;
        for (int t = 0; t < ntiles; ++t) {
            const uint32_t par = t & 1;
            const int st = t & 1;
            const Tile tl = unpack_tile(tiles[t]);
            const float* c2 = &cs2[t & 1][0][0];
            uint8_t* Xst = smem + S::oX + st * S::kX + eh * kBox;

            // the next tile's cumsum while Y(t) is computed
            if (t + 1 < ntiles) {
                tile_cumsum(t + 1, la_next);
                la_next = load_la(t + 2);
            }
            // ---- epilogue(t): Y staged in Hs (or stored), X' = w X in place ----
            mbar_wait(&bar_yd, par);
            mbar_wait(&bar_yo, par);
            tc_fence_after();
            {
                const float ck = c2[128 * eh + m];
                const float cend = c2[128 * eh + tl.v - 1];
                const float rs = ex2_approx(ck);                           // decay from the tile start
                const float wx = m < tl.v ? ex2_approx(cend - ck) : 0.f;  // decay to the tile end
                const __nv_bfloat162 wx2 = __floats2bfloat162_rn(wx, wx);
                __nv_bfloat16* yrow = Y + ((row + tl.ts + m) * d.nheads + h0 + eh) * (int64_t)kP + p0;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {  // 16 columns at a time
                    uint32_t yd[16], yo[16];
                    tmem_ld16_async(tm_yd + lane_off + 32 * cq + 16 * hf, yd);
                    tmem_ld16_async(tm_yo + lane_off + 32 * cq + 16 * hf, yo);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const int c16 = (p0 >> 3) + 2 * hf + c;
                        const uint32_t off = sw128_off(m, c16);
                        uint4 xv = *reinterpret_cast<const uint4*>(Xst + off);
                        uint32_t* xu = reinterpret_cast<uint32_t*>(&xv);
                        uint32_t out[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const __nv_bfloat162 xb = *reinterpret_cast<const __nv_bfloat162*>(&xu[i]);
                            const float2 xf = __bfloat1622float2(xb);
                            const int e0 = 8 * c + 2 * i;
                            out[i] = pack_bf16(fmaf(dh, xf.x, fmaf(rs, __uint_as_float(yo[e0]), __uint_as_float(yd[e0]))),
                                               fmaf(dh, xf.y, fmaf(rs, __uint_as_float(yo[e0 + 1]), __uint_as_float(yd[e0 + 1]))));
                            const __nv_bfloat162 xs = __hmul2(xb, wx2);
                            xu[i] = *reinterpret_cast<const uint32_t*>(&xs);
                        }
                        const uint4 ov = make_uint4(out[0], out[1], out[2], out[3]);
                        if (tl.v == 128) *reinterpret_cast<uint4*>(Hs + eh * kBox + off) = ov;  // Y_off(t) has read Hs
                        else if (m < tl.v) *reinterpret_cast<uint4*>(yrow + 8 * (c16 - (p0 >> 3))) = ov;
                        *reinterpret_cast<uint4*>(Xst + off) = xv;
                    }
                }
            }
            fence_async_shared();
            tc_fence_before();
            signal(&bar_epi);

            // ---- L o G(t+1) while H += X'^T B runs ----
            if (t + 1 < ntiles) build_lg(t + 1);

            // ---- state(t): H(t) to Hs (bf16) and to the final states; pre-scale for t+1 ----
            mbar_wait(&bar_s, par);
            mbar_wait(&bar_free, par);
            tc_fence_after();
            {
                float hv[NQ];
                ld_state(hv);
                if (tl.last) {
                    const int pend = tl.ts + tl.v;
                    const int sid = piece_id(tl.ts);
                    if (final_states && seq_ends_at(pend)) {
                        float* f = final_states + seqst_off(d, b, sid, h0 + sh);
#pragma unroll
                        for (int i = 0; i < NQ; ++i) f[(int64_t)(cq * NQ + i) * kP + sp] = hv[i];
                    }
                    if (t + 1 < ntiles) {  // the next piece starts a new sequence
                        const Tile tn = unpack_tile(tiles[t + 1]);
                        load_state(hv, init_states ? init_states + seqst_off(d, b, piece_id(tn.ts), h0 + sh) : nullptr);
                    }
                }
                if (t + 1 < ntiles) {
                    write_hs(hv);
                    st_state_scaled(hv, tile_decay(t + 1));
                    tmem_wait_st();
                }
            }
            fence_async_shared();
            tc_fence_before();
            signal(&bar_st);
        }
        // ids after the row's last sequence never occur: they keep their initial state
        if (final_states && s1 == d.seqlen && seq_idx) {
            for (int sq = lastid_s + 1; sq < d.nseq; ++sq) {
                float* f = final_states + seqst_off(d, b, sq, h0 + sh);
                const float* src = init_states ? init_states + seqst_off(d, b, sq, h0 + sh) : nullptr;
#pragma unroll
                for (int i = 0; i < NQ; ++i) {
                    const int64_t o = (int64_t)(cq * NQ + i) * kP + sp;
                    f[o] = src ? src[o] : 0.f;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
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

int max_tiles(int seglen, bool varlen) { return varlen ? seglen + seglen / 128 + 2 : seglen / 128 + 2; }

template <int N>
int fused_smem_bytes(int seglen, bool varlen) {
    return (int)FusedSmem<N>::oTail + (varlen ? seglen * 4 : 0) + max_tiles(seglen, varlen) * 8 + 1024;
}

int num_sms() {
    static int n[16] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) {
        cudaGetLastError();
        return 148;
    }
    if (!n[dev]) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
            cudaGetLastError();
            v = 148;
        }
        n[dev] = v;
    }
    return n[dev];
}

}  // namespace

bool fused_supported(const ssd_problem* p) {
    if (p->dtype != SSD_DTYPE_BF16 || p->headdim != kP) return false;
    if (p->dstate != 64 && p->dstate != 128) return false;
    if ((p->nheads / p->ngroups) % 2 != 0) return false;
    return true;
}

bool fused_seglen_ok(const Dims& d, int64_t seglen) {
    (void)d;
    return seglen >= 128 && seglen <= 2048 && seglen % 128 == 0;
}

// Segment length: balance the waves of fused_scan (one CTA per SM, time per
// wave proportional to the tiles of a segment) against the per-segment state
// traffic (about four tiles' worth of bytes per segment, spread over the SMs).
int fused_default_seglen(const Dims& d) {
    const int nsm = num_sms();
    const int64_t pairs = (int64_t)d.batch * (d.nheads / 2);
    int best = 128;
    double best_cost = 1e300;
    for (int L = 128; L <= 2048; L *= 2) {
        const int64_t nseg = (d.seqlen + L - 1) / L;
        const int64_t items = pairs * nseg;
        const double waves = (double)((items + nsm - 1) / nsm);
        const double tiles = (double)(L < d.seqlen ? L : ((d.seqlen + 127) / 128) * 128) / 128.0;
        const double cost = waves * tiles + (nseg > 1 ? 4.0 * (double)items / nsm : 0.0);
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best = L;
        }
        if (L >= d.seqlen) break;
    }
    return best;
}

size_t fused_workspace_bytes(const Dims& d, int seglen) {
    const size_t nseg = (d.seqlen + seglen - 1) / seglen;
    const size_t st = (size_t)d.batch * nseg * d.nheads * d.dstate * d.headdim * sizeof(float);
    const size_t dec = (size_t)d.batch * nseg * d.nheads * sizeof(float);
    return ((st + 255) & ~size_t(255)) + ((dec + 255) & ~size_t(255));
}

cudaError_t launch_segment_state(const Dims& d, int seglen, const void* X, const float* log_a, const void* B,
                                 const int32_t* seq_idx, float* seg_states, float* seg_decay, cudaStream_t st) {
    CUtensorMap mx, mb;
    cudaError_t e;
    if ((e = x_map(&mx, d, X, 128)) != cudaSuccess) return e;
    if ((e = bc_map(&mb, d, B, 128)) != cudaSuccess) return e;
    const int nseg = (d.seqlen + seglen - 1) / seglen;
    const dim3 grid(d.batch * (d.nheads / 2) * nseg);
    const int smem = 2 * (int)kBox + (d.dstate / 64) * (int)kBox + 1024;
    if (d.dstate == 64) {
        auto k = segment_state_kernel<64>;
        if ((e = set_smem_attr(k, smem, 30)) != cudaSuccess) return e;
        k<<<grid, kSegThreads, smem, st>>>(mx, mb, d, seglen, nseg, log_a, seq_idx, seg_states, seg_decay);
    } else if (d.dstate == 128) {
        auto k = segment_state_kernel<128>;
        if ((e = set_smem_attr(k, smem, 31)) != cudaSuccess) return e;
        k<<<grid, kSegThreads, smem, st>>>(mx, mb, d, seglen, nseg, log_a, seq_idx, seg_states, seg_decay);
    } else {
        return cudaErrorNotSupported;
    }
    return cudaGetLastError();
}

cudaError_t launch_segment_passing(const Dims& d, int seglen, float* seg_states, const float* seg_decay,
                                   const float* init_states, const int32_t* seq_idx, cudaStream_t st) {
    const int nseg = (d.seqlen + seglen - 1) / seglen;
    const dim3 grid(d.batch * d.nheads, (d.dstate * d.headdim + 1023) / 1024);
    segment_passing_kernel<<<grid, 256, 0, st>>>(d, seglen, nseg, seg_states, seg_decay, init_states, seq_idx);
    return cudaGetLastError();
}

cudaError_t launch_fused_scan(const Dims& d, int seglen, const void* X, const float* log_a, const void* B,
                              const void* C, const float* D, const float* seg_incoming, const float* init_states,
                              const int32_t* seq_idx, void* Y, float* final_states, cudaStream_t st) {
    CUtensorMap mx, mb, mc, my;
    cudaError_t e;
    if ((e = x_map(&mx, d, X, 128)) != cudaSuccess) return e;
    if ((e = bc_map(&mb, d, B, 128)) != cudaSuccess) return e;
    if ((e = bc_map(&mc, d, C, 128)) != cudaSuccess) return e;
    if ((e = x_map(&my, d, Y, 128)) != cudaSuccess) return e;
    const int nseg = (d.seqlen + seglen - 1) / seglen;
    const dim3 grid(d.batch * (d.nheads / 2) * nseg);
    const bool varlen = seq_idx != nullptr;
    if (d.dstate == 64) {
        auto k = fused_scan_kernel<64>;
        const int smem = fused_smem_bytes<64>(seglen, varlen);
        if ((e = set_smem_attr(k, smem, 32)) != cudaSuccess) return e;
        k<<<grid, kFusedThreads, smem, st>>>(mx, mb, mc, my, d, seglen, nseg, log_a, D, seg_incoming, init_states,
                                             seq_idx, (__nv_bfloat16*)Y, final_states);
    } else if (d.dstate == 128) {
        auto k = fused_scan_kernel<128>;
        const int smem = fused_smem_bytes<128>(seglen, varlen);
        if ((e = set_smem_attr(k, smem, 33)) != cudaSuccess) return e;
        k<<<grid, kFusedThreads, smem, st>>>(mx, mb, mc, my, d, seglen, nseg, log_a, D, seg_incoming, init_states,
                                             seq_idx, (__nv_bfloat16*)Y, final_states);
    } else {
        return cudaErrorNotSupported;
    }
    return cudaGetLastError();
}

}  // namespace ssd
