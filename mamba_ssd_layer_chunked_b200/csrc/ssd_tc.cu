// ssd_tc.cu -- tensor-core kernels of the SSD chunked scan for sm_100a (bf16
// inputs, fp32 accumulation in TMEM): chunk_state and chunk_scan.
//
// Both kernels give one CTA (4 warps) a pair of heads of one batch row, so
// that the two heads' 64-wide head dimensions fill the 128 rows of a
// tcgen05.mma (M = 128) and the group's B and C tiles, shared by the heads
// ("Mamba-2 - Transformer and SSM share one algebra", design 3: B and C shared
// across the input heads), are read once per pair. Tiles arrive by TMA with
// 128-byte swizzle; thread 0 issues the MMAs; the accumulators are read back
// with tcgen05.ld by the warp that owns each TMEM lane quarter.
//
// Block algorithm: "Mamba-2: writing the recurrent state as a structured
// matrix" (wq-win.github.io/llm/088-mamba2.html), section 3: per chunk the
// local end state (zero incoming state), the local output (L o C B^T) X, and
// the incoming state decayed to each position and read out by C.

#include <cuda.h>

#include <mutex>

#include "ssd_tc.cuh"
#include "tc_ptx.cuh"

namespace ssd {

namespace {

using namespace tc;

constexpr int kTcThreads = 128;
constexpr int kP = 64;  // head dim covered by the tensor-core kernels

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// scale the 64 bf16 of a 128-byte row by w (in place; chunk order is irrelevant)
__device__ __forceinline__ void scale_row_bf16(uint8_t* row, float w) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4 v = *reinterpret_cast<uint4*>(row + 16 * c);
        uint32_t* u = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 b2 = *reinterpret_cast<__nv_bfloat162*>(&u[i]);
            float2 f = __bfloat1622float2(b2);
            u[i] = pack_bf16(f.x * w, f.y * w);
        }
        *reinterpret_cast<uint4*>(row + 16 * c) = v;
    }
}

// ---------------------------------------------------------------------------
// chunk_state: S^T[(h,p), n] = sum_l w_h(l) X_h[l, p] B[l, n]   (M=128: 2 heads x P)
//   A = decay-scaled X tile, MN-major (rows l, 64 p per head, heads LBO apart)
//   B = B tile, MN-major (rows l, 64 n per 128-byte box, boxes LBO apart)
// grid.x = (b, head pair, chunk), chunk fastest.
// ---------------------------------------------------------------------------
template <int Q, int N>
__global__ void __launch_bounds__(kTcThreads, 1)
    chunk_state_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b, Dims d,
                          const float* __restrict__ cs, const int32_t* __restrict__ seq_idx,
                          float* __restrict__ states, float* __restrict__ final_states) {
    constexpr uint32_t kXBytes = 2u * Q * 128u;        // two heads, [Q][64] bf16 each
    constexpr uint32_t kBBytes = (N / 64) * Q * 128u;  // N/64 boxes of [Q][64]
    constexpr uint32_t kCols = N;                      // fp32 accumulator columns
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* Xs = smem;
    uint8_t* Bs = smem + kXBytes;
    __shared__ float cs_s[2][Q];
    __shared__ int seq_s[Q];
    __shared__ int pst_s[Q];
    __shared__ __align__(8) uint64_t bar_load, bar_mma;
    __shared__ uint32_t tmem_base;

    const int tid = threadIdx.x, warp = tid >> 5;
    const int npairs = d.nheads / 2;
    int r = blockIdx.x;
    const int c = r % d.nchunks;
    r /= d.nchunks;
    const int hp = r % npairs, b = r / npairs;
    const int h0 = 2 * hp, g = h0 / d.heads_per_group;

    if (tid == 0) {
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_b);
        mbar_init(&bar_load, 1);
        mbar_init(&bar_mma, 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, kCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t taddr = tmem_base;

    if (tid == 0) {
        mbar_arrive_expect_tx(&bar_load, kXBytes + kBBytes);
        tma_load_4d(Xs, &tm_x, &bar_load, 0, h0, c * Q, b);
        tma_load_4d(Xs + Q * 128, &tm_x, &bar_load, 0, h0 + 1, c * Q, b);
#pragma unroll
        for (int j = 0; j < N / 64; ++j) tma_load_4d(Bs + j * Q * 128, &tm_b, &bar_load, 64 * j, g, c * Q, b);
    }
    const int64_t row = (int64_t)b * d.seqlen;
    for (int i = tid; i < 2 * Q; i += kTcThreads) cs_s[i / Q][i % Q] = cs[cs_off(d, b, h0 + i / Q, c) + i % Q];
    for (int k = tid; k < Q; k += kTcThreads) seq_s[k] = seq_at_padded(seq_idx, row, c * Q + k, d.seqlen, d.nseq);
    __syncthreads();
    for (int k = tid; k < Q; k += kTcThreads) {
        const int v = seq_s[k];
        int lo = 0, hi = k;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (seq_s[mid] < v) lo = mid + 1;
            else hi = mid;
        }
        pst_s[k] = lo;
    }
    __syncthreads();
    mbar_wait(&bar_load, 0);

    uint32_t load_phase = 1, mma_phase = 0;
    const uint32_t idesc = idesc_bf16(128, N, true, true);
    const uint32_t xs_addr = smem_u32(Xs), bs_addr = smem_u32(Bs);
    int e = Q - 1;
    while (e >= 0) {
        const int st = pst_s[e];
        const bool last = (e == Q - 1);
        if (!last && (final_states == nullptr || seq_idx == nullptr)) break;
        if (!last) {  // the X tile was scaled in place: fetch it again
            if (tid == 0) {
                mbar_arrive_expect_tx(&bar_load, kXBytes);
                tma_load_4d(Xs, &tm_x, &bar_load, 0, h0, c * Q, b);
                tma_load_4d(Xs + Q * 128, &tm_x, &bar_load, 0, h0 + 1, c * Q, b);
            }
            mbar_wait(&bar_load, load_phase);
            load_phase ^= 1;
        }
        // X' = exp(cs[e] - cs[l]) X for l in [st, e], 0 elsewhere
        for (int R = tid; R < 2 * Q; R += kTcThreads) {
            const int hh = R / Q, l = R % Q;
            const float w = (l >= st && l <= e) ? __expf(cs_s[hh][e] - cs_s[hh][l]) : 0.f;
            scale_row_bf16(Xs + hh * Q * 128 + l * 128, w);
        }
        fence_async_shared();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const int j0 = st / 16, j1 = e / 16;
            for (int j = j0; j <= j1; ++j) {
                const uint64_t ad = smem_desc_sw128(xs_addr + j * 2048, Q * 128, 1024);
                const uint64_t bd = smem_desc_sw128(bs_addr + j * 2048, Q * 128, 1024);
                mma_bf16_ss(taddr, ad, bd, idesc, j > j0 ? 1u : 0u);
            }
            mma_commit(&bar_mma);
        }
        mbar_wait(&bar_mma, mma_phase);
        mma_phase ^= 1;
        tc_fence_after();
        // epilogue: lane tid holds S^T row (head tid/64, p = tid%64), N columns
        const int hh = tid >> 6, p = tid & 63;
        float* dst = last ? states + st_off(d, b, c, h0 + hh) : final_states + seqst_off(d, b, seq_s[e], h0 + hh);
        const uint32_t lane_addr = taddr + ((uint32_t)(warp * 32) << 16);
#pragma unroll
        for (int n0 = 0; n0 < N; n0 += 32) {
            float v[32];
            tmem_ld32(lane_addr + n0, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) dst[(int64_t)(n0 + i) * kP + p] = v[i];
        }
        tc_fence_before();
        __syncthreads();
        e = st - 1;
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(taddr, kCols);
}

// ---------------------------------------------------------------------------
// chunk_scan: for the 128 rows [128 r, 128 r + 128) of chunk c and two heads
//   Yo[k, (h,p)] = C_k . Hs[h][:, p]                        (M=128, N=128, K=N)
//   G[k, l]      = C_k . B_l  for each column block c' <= r (M=128, N=128, K=N)
//   Yd_h[k, p]  += (L_h o G)[k, l] X_h[l, p]                 (M=128, N=64,  K=128)
//   Y = Yd + rscale_h(k) Yo + D_h x
// C, B, L o G and Hs are K-major operands, X is MN-major.
// grid.x = (b, head pair, chunk, row block), row block fastest.
// ---------------------------------------------------------------------------
template <int Q, int N>
struct ScanSmem {
    static constexpr uint32_t kBox = 128u * 128u;          // [128 rows][64 bf16]
    static constexpr uint32_t kC = (N / 64) * kBox;       // C rows of the block, K = n
    static constexpr uint32_t kB = (N / 64) * kBox;       // B rows of a column block
    static constexpr uint32_t kX = 2u * kBox;             // X of a column block, two heads
    static constexpr uint32_t kLG = 2u * 2u * kBox;       // L o G, two heads x two K blocks
    static constexpr uint32_t kH = (N / 64) * kBox;       // Hs^T, rows (h,p), K = n
    static constexpr uint32_t kHX = kH > kX ? kH : kX;    // Hs^T, then the diagonal X block
    static constexpr uint32_t oC = 0, oB = oC + kC, oX = oB + kB, oLG = oX + kX, oHX = oLG + kLG;
    static constexpr uint32_t kBytes = oHX + kHX;
};

template <int Q, int N>
__global__ void __launch_bounds__(kTcThreads, 1)
    chunk_scan_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                         const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y, Dims d,
                         const float* __restrict__ cs, const float* __restrict__ Dv,
                         const float* __restrict__ incoming, const float* __restrict__ init_states,
                         const int32_t* __restrict__ seq_idx) {
    using S = ScanSmem<Q, N>;
    constexpr int NR = Q / 128;  // row blocks per chunk
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* Cs = smem + S::oC;
    uint8_t* Bs = smem + S::oB;
    uint8_t* Xa = smem + S::oX;
    uint8_t* LG = smem + S::oLG;
    uint8_t* HX = smem + S::oHX;
    __shared__ float cs_s[2][Q];
    __shared__ float colf[2][128];
    __shared__ int seq_s[Q];
    __shared__ int pst_s[Q];
    __shared__ int multi_piece;
    __shared__ __align__(8) uint64_t bar_ld0, bar_ldb, bar_ldx, bar_yo, bar_g, bar_yd;
    __shared__ uint32_t tmem_base;

    const int tid = threadIdx.x, warp = tid >> 5;
    const int npairs = d.nheads / 2;
    int rr = blockIdx.x;
    const int rb = rr % NR;
    rr /= NR;
    const int c = rr % d.nchunks;
    rr /= d.nchunks;
    const int hp = rr % npairs, b = rr / npairs;
    const int h0 = 2 * hp, g = h0 / d.heads_per_group;
    const int t0 = c * Q;  // first token of the chunk
    const int k0 = 128 * rb;  // first row of this block inside the chunk
    // a row block wholly past the end of a partial last chunk has no output:
    // leave before any setup, so that no TMA copy starts past the row end
    if (t0 + k0 >= d.seqlen) return;

    if (tid == 0) {
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_b);
        prefetch_tmap(&tm_c);
        prefetch_tmap(&tm_y);
        mbar_init(&bar_ld0, 1);
        mbar_init(&bar_ldb, 1);
        mbar_init(&bar_ldx, 1);
        mbar_init(&bar_yo, 1);
        mbar_init(&bar_g, 1);
        mbar_init(&bar_yd, 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm_g = tmem_base, tm_yd = tmem_base + 128, tm_yo = tmem_base + 256;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

    // column block 0 (C of this row block, B and X of column block 0)
    if (tid == 0) {
        mbar_arrive_expect_tx(&bar_ld0, S::kC + S::kB + S::kX);
#pragma unroll
        for (int j = 0; j < N / 64; ++j) {
            tma_load_4d(Cs + j * S::kBox, &tm_c, &bar_ld0, 64 * j, g, t0 + k0, b);
            tma_load_4d(Bs + j * S::kBox, &tm_b, &bar_ld0, 64 * j, g, t0, b);
        }
        tma_load_4d(Xa, &tm_x, &bar_ld0, 0, h0, t0, b);
        tma_load_4d(Xa + S::kBox, &tm_x, &bar_ld0, 0, h0 + 1, t0, b);
    }
    const int64_t row = (int64_t)b * d.seqlen;
    for (int i = tid; i < 2 * Q; i += kTcThreads) cs_s[i / Q][i % Q] = cs[cs_off(d, b, h0 + i / Q, c) + i % Q];
    for (int k = tid; k < Q; k += kTcThreads) seq_s[k] = seq_at_padded(seq_idx, row, t0 + k, d.seqlen, d.nseq);
    if (tid == 0) multi_piece = 0;
    __syncthreads();
    for (int k = tid; k < Q; k += kTcThreads) {
        const int v = seq_s[k];
        int lo = 0, hi = k;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (seq_s[mid] < v) lo = mid + 1;
            else hi = mid;
        }
        pst_s[k] = lo;
    }
    __syncthreads();
    const int kk = k0 + tid;  // this thread's row inside the chunk
    const int my_pst = pst_s[kk];
    if (my_pst != 0 && init_states != nullptr) multi_piece = 1;
    __syncthreads();

    // ---- left factor: Yo = C Hs, rows grouped by their sequence piece ----
    // thread tid builds row (h, p) = (tid/64, tid%64) of Hs^T (K-major, K = n)
    auto build_hs = [&](const float* src_h0, const float* src_h1) {
        const int hh = tid >> 6, p = tid & 63;
        const float* src = hh ? src_h1 : src_h0;
#pragma unroll 4
        for (int n8 = 0; n8 < N / 8; ++n8) {
            uint32_t u[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float a = src ? src[(int64_t)(8 * n8 + 2 * i) * kP + p] : 0.f;
                const float bb = src ? src[(int64_t)(8 * n8 + 2 * i + 1) * kP + p] : 0.f;
                u[i] = pack_bf16(a, bb);
            }
            const int kb = n8 >> 3, ch = n8 & 7;
            *reinterpret_cast<uint4*>(HX + kb * S::kBox + sw128_off(tid, ch)) = make_uint4(u[0], u[1], u[2], u[3]);
        }
    };
    const uint32_t idesc_128x128 = idesc_bf16(128, 128, false, false);
    const uint32_t idesc_128x64_mn = idesc_bf16(128, 64, false, true);
    auto issue_yo = [&](const uint8_t* A, uint32_t accumulate) {
        const uint32_t a_addr = smem_u32(A), h_addr = smem_u32(HX);
#pragma unroll
        for (int j = 0; j < N / 16; ++j) {
            const uint32_t off = (j >> 2) * S::kBox + (j & 3) * 32;
            mma_bf16_ss(tm_yo, smem_desc_sw128(a_addr + off, 16, 1024), smem_desc_sw128(h_addr + off, 16, 1024),
                        idesc_128x128, (j > 0 || accumulate) ? 1u : 0u);
        }
    };
    uint32_t yo_phase = 0;
    if (!multi_piece) {
        build_hs(incoming + st_off(d, b, c, h0), incoming + st_off(d, b, c, h0 + 1));
        fence_async_shared();
        __syncthreads();
        if (tid == 0) {
            mbar_wait(&bar_ld0, 0);
            tc_fence_after();
            issue_yo(Cs, 0);
            mma_commit(&bar_yo);
        }
    } else {
        // rare: sequences with initial states start inside this row block; one
        // MMA per piece with the rows of the other pieces of C zeroed
        mbar_wait(&bar_ld0, 0);
        int piece_start = pst_s[k0];
        uint32_t acc = 0;
        while (true) {
            const float* s0;
            const float* s1;
            if (piece_start == 0) {
                s0 = incoming + st_off(d, b, c, h0);
                s1 = incoming + st_off(d, b, c, h0 + 1);
            } else {
                const int sq = seq_s[piece_start];
                s0 = init_states + seqst_off(d, b, sq, h0);
                s1 = init_states + seqst_off(d, b, sq, h0 + 1);
            }
            build_hs(s0, s1);
            // masked copy of this row block's C into the L o G buffer
            const bool mine = (my_pst == piece_start);
#pragma unroll
            for (int kb = 0; kb < N / 64; ++kb)
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint32_t off = kb * S::kBox + sw128_off(tid, ch);
                    *reinterpret_cast<uint4*>(LG + off) =
                        mine ? *reinterpret_cast<const uint4*>(Cs + off) : make_uint4(0, 0, 0, 0);
                }
            fence_async_shared();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                issue_yo(LG, acc);
                mma_commit(&bar_yo);
            }
            mbar_wait(&bar_yo, yo_phase);
            yo_phase ^= 1;
            acc = 1;
            // next piece start among this block's rows
            int next = -1;
            for (int k = k0; k < k0 + 128; ++k)
                if (pst_s[k] > piece_start) {
                    next = pst_s[k];
                    break;
                }
            __syncthreads();
            if (next < 0) break;
            piece_start = next;
        }
        if (tid == 0) mma_commit(&bar_yo);  // re-arm: the final wait below sees one more phase
    }

    // ---- diagonal blocks: G = C B^T per column block, L o G, Yd += (L o G) X ----
    uint32_t g_phase = 0, yd_phase = 0, ldb_phase = 0;
    for (int cb = 0; cb <= rb; ++cb) {
        const bool diag = (cb == rb);
        uint8_t* Xc = (rb > 0 && diag) ? HX : Xa;  // diagonal X of a later row block lives in HX
        if (tid == 0) {
            if (cb == 0) {
                mbar_wait(&bar_ld0, 0);
            } else {
                mbar_wait(&bar_ldb, ldb_phase);
                ldb_phase ^= 1;
            }
            tc_fence_after();
            const uint32_t c_addr = smem_u32(Cs), b_addr = smem_u32(Bs);
#pragma unroll
            for (int j = 0; j < N / 16; ++j) {
                const uint32_t off = (j >> 2) * S::kBox + (j & 3) * 32;
                mma_bf16_ss(tm_g, smem_desc_sw128(c_addr + off, 16, 1024), smem_desc_sw128(b_addr + off, 16, 1024),
                            idesc_128x128, j > 0 ? 1u : 0u);
            }
            mma_commit(&bar_g);
            if (cb < rb) {
                // next column block: B after this G has read Bs; X (the diagonal
                // one) into HX once the left-factor MMA has read Hs
                mbar_wait(&bar_g, g_phase);
                mbar_arrive_expect_tx(&bar_ldb, S::kB);
#pragma unroll
                for (int j = 0; j < N / 64; ++j)
                    tma_load_4d(Bs + j * S::kBox, &tm_b, &bar_ldb, 64 * j, g, t0 + 128 * (cb + 1), b);
                if (cb + 1 == rb) {
                    mbar_wait(&bar_yo, yo_phase);
                    mbar_arrive_expect_tx(&bar_ldx, S::kX);
                    tma_load_4d(HX, &tm_x, &bar_ldx, 0, h0, t0 + 128 * (cb + 1), b);
                    tma_load_4d(HX + S::kBox, &tm_x, &bar_ldx, 0, h0 + 1, t0 + 128 * (cb + 1), b);
                }
            }
        }
        // per-column decay factors of an off-diagonal block (reference row ref)
        const int l0 = 128 * cb;
        const int ref = k0 - 1;
        if (!diag) {
            for (int i = tid; i < 256; i += kTcThreads) {
                const int hh = i >> 7, l = l0 + (i & 127);
                colf[hh][i & 127] = __expf(cs_s[hh][ref] - cs_s[hh][l]);
            }
        }
        __syncthreads();
        mbar_wait(&bar_g, g_phase);
        g_phase ^= 1;
        if (cb > 0) {  // the previous Yd MMAs must have finished reading L o G
            mbar_wait(&bar_yd, yd_phase);
            yd_phase ^= 1;
        }
        tc_fence_after();
        // thread tid: row kk of L o G for both heads, 128 columns
        const float cs_k0 = cs_s[0][kk], cs_k1 = cs_s[1][kk];
        const float rf0 = diag ? 0.f : __expf(cs_k0 - cs_s[0][ref]);
        const float rf1 = diag ? 0.f : __expf(cs_k1 - cs_s[1][ref]);
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
            float gv[32];
            tmem_ld32(tm_g + lane_off + 32 * q, gv);
#pragma unroll
            for (int ch4 = 0; ch4 < 4; ++ch4) {
                uint32_t u0[4], u1[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float a0[2], a1[2];
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        const int lc = 32 * q + 8 * ch4 + 2 * i + t;  // column inside the block
                        const int l = l0 + lc;
                        const float gg = gv[8 * ch4 + 2 * i + t];
                        const bool same = pst_s[l] == my_pst;
                        if (diag) {
                            const bool ok = same && l <= kk;
                            a0[t] = ok ? gg * __expf(cs_k0 - cs_s[0][l]) : 0.f;
                            a1[t] = ok ? gg * __expf(cs_k1 - cs_s[1][l]) : 0.f;
                        } else {
                            a0[t] = same ? gg * rf0 * colf[0][lc] : 0.f;
                            a1[t] = same ? gg * rf1 * colf[1][lc] : 0.f;
                        }
                    }
                    u0[i] = pack_bf16(a0[0], a0[1]);
                    u1[i] = pack_bf16(a1[0], a1[1]);
                }
                const int lc8 = 4 * q + ch4;  // 16-byte chunk index over the 128 columns
                const uint32_t off = (lc8 >> 3) * S::kBox + sw128_off(tid, lc8 & 7);
                *reinterpret_cast<uint4*>(LG + off) = make_uint4(u0[0], u0[1], u0[2], u0[3]);
                *reinterpret_cast<uint4*>(LG + 2 * S::kBox + off) = make_uint4(u1[0], u1[1], u1[2], u1[3]);
            }
        }
        fence_async_shared();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            if (rb > 0 && diag) {
                mbar_wait(&bar_ldx, 0);
            }
            tc_fence_after();
            const uint32_t lg_addr = smem_u32(LG), x_addr = smem_u32(Xc);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t aoff = hh * 2 * S::kBox + (j >> 2) * S::kBox + (j & 3) * 32;
                    const uint32_t boff = hh * S::kBox + j * 2048;
                    mma_bf16_ss(tm_yd + 64 * hh, smem_desc_sw128(lg_addr + aoff, 16, 1024),
                                smem_desc_sw128(x_addr + boff, S::kBox, 1024), idesc_128x64_mn,
                                (cb > 0 || j > 0) ? 1u : 0u);
                }
            }
            mma_commit(&bar_yd);
        }
    }

    // ---- epilogue: Y = Yd + rscale Yo + D x, staged in the L o G buffer ----
    mbar_wait(&bar_yd, yd_phase);
    mbar_wait(&bar_yo, yo_phase);
    tc_fence_after();
    uint8_t* Xr = (rb > 0) ? HX : Xa;  // X of this row block
    uint8_t* Ys = LG;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const float csk = cs_s[hh][kk];
        float rs;
        if (my_pst == 0) rs = __expf(csk);
        else rs = init_states ? __expf(csk - cs_s[hh][my_pst - 1]) : 0.f;
        const float dh = Dv ? Dv[h0 + hh] : 0.f;
#pragma unroll
        for (int p0 = 0; p0 < 64; p0 += 32) {
            float yd[32], yo[32];
            tmem_ld32(tm_yd + lane_off + 64 * hh + p0, yd);
            tmem_ld32(tm_yo + lane_off + 64 * hh + p0, yo);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                const int c16 = (p0 >> 3) + ch;  // 16-byte chunk of the 128-byte row
                const uint4 xv = *reinterpret_cast<const uint4*>(Xr + hh * S::kBox + sw128_off(tid, c16));
                const uint32_t* xu = reinterpret_cast<const uint32_t*>(&xv);
                uint32_t out[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xu[i]));
                    const int e0 = 8 * ch + 2 * i;
                    const float y0 = fmaf(dh, xf.x, fmaf(rs, yo[e0], yd[e0]));
                    const float y1 = fmaf(dh, xf.y, fmaf(rs, yo[e0 + 1], yd[e0 + 1]));
                    out[i] = pack_bf16(y0, y1);
                }
                *reinterpret_cast<uint4*>(Ys + hh * S::kBox + sw128_off(tid, c16)) =
                    make_uint4(out[0], out[1], out[2], out[3]);
            }
        }
    }
    fence_async_shared();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        tma_store_4d(&tm_y, Ys, 0, h0, t0 + k0, b);
        tma_store_4d(&tm_y, Ys + S::kBox, 0, h0 + 1, t0 + k0, b);
        tma_store_commit();
        tma_store_wait_read0();
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem_base, 512);
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes, int slot) {
    return ensure_smem_attr(reinterpret_cast<const void*>(kernel), bytes, slot);
}

}  // namespace

// ---------------------------------------------------------------------------
// host: tensor maps
// ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// 4-D bf16 map over a [batch][token][mid][inner] row-major tensor, addressed as
// (inner, mid, token, batch) = (d0, d1, d2, d3) so the strides increase; a box
// is 64 inner elements (128 bytes, 128-byte swizzle) x 1 x box_tok tokens x 1.
cudaError_t make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t mid, uint64_t tokens,
                     uint64_t batch, uint32_t box_tok) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[4] = {inner, mid, tokens, batch};
    const cuuint64_t strides[3] = {inner * 2, mid * inner * 2, tokens * mid * inner * 2};
    const cuuint32_t box[4] = {64, 1, box_tok, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t x_map(CUtensorMap* m, const Dims& d, const void* X, uint32_t box_tok) {
    return make_map(m, X, d.headdim, d.nheads, d.seqlen, d.batch, box_tok);
}

cudaError_t bc_map(CUtensorMap* m, const Dims& d, const void* Bp, uint32_t box_tok) {
    return make_map(m, Bp, d.dstate, d.ngroups, d.seqlen, d.batch, box_tok);
}



bool tc_supported(const ssd_problem* p) {
    if (p->dtype != SSD_DTYPE_BF16) return false;
    if (p->headdim != kP) return false;
    if (p->dstate != 64 && p->dstate != 128) return false;
    if (p->chunk != 128 && p->chunk != 256) return false;
    if ((p->nheads / p->ngroups) % 2 != 0) return false;  // head pairs must share a group
    return true;
}

cudaError_t launch_chunk_state_tc(const Dims& d, const void* X, const void* B, const float* cs, const int32_t* seq_idx,
                                  float* states, float* final_states, cudaStream_t st) {
    CUtensorMap mx, mb;
    cudaError_t e;
    if ((e = x_map(&mx, d, X, d.chunk)) != cudaSuccess) return e;
    if ((e = bc_map(&mb, d, B, d.chunk)) != cudaSuccess) return e;
    const dim3 grid(d.batch * (d.nheads / 2) * d.nchunks);
    // X tile + B tile + 1 KB alignment slack + one X-head tile of padding, so
    // that every operand read of the MMA stays inside the allocation
    const int smem = 2 * d.chunk * 128 + (d.dstate / 64) * d.chunk * 128 + 1024 + d.chunk * 128;
#define SSD_STATE_CASE(QQ, NN, SLOT)                                                                  \
    if (d.chunk == QQ && d.dstate == NN) {                                                            \
        auto k = chunk_state_tc_kernel<QQ, NN>;                                                       \
        if ((e = set_smem(k, smem, SLOT)) != cudaSuccess) return e;                                   \
        k<<<grid, kTcThreads, smem, st>>>(mx, mb, d, cs, seq_idx, states, final_states);              \
        return cudaGetLastError();                                                                    \
    }
    SSD_STATE_CASE(128, 64, 10)
    SSD_STATE_CASE(128, 128, 11)
    SSD_STATE_CASE(256, 64, 12)
    SSD_STATE_CASE(256, 128, 13)
#undef SSD_STATE_CASE
    return cudaErrorNotSupported;
}

cudaError_t launch_chunk_scan_tc(const Dims& d, const void* X, const void* B, const void* C, const float* cs,
                                 const float* D, const float* incoming, const float* init_states,
                                 const int32_t* seq_idx, void* Y, cudaStream_t st) {
    CUtensorMap mx, mb, mc, my;
    cudaError_t e;
    if ((e = x_map(&mx, d, X, 128)) != cudaSuccess) return e;
    if ((e = bc_map(&mb, d, B, 128)) != cudaSuccess) return e;
    if ((e = bc_map(&mc, d, C, 128)) != cudaSuccess) return e;
    if ((e = x_map(&my, d, Y, 128)) != cudaSuccess) return e;
    const dim3 grid(d.batch * (d.nheads / 2) * d.nchunks * (d.chunk / 128));
#define SSD_SCAN_CASE(QQ, NN, SLOT)                                                                   \
    if (d.chunk == QQ && d.dstate == NN) {                                                            \
        auto k = chunk_scan_tc_kernel<QQ, NN>;                                                        \
        const int smem = ScanSmem<QQ, NN>::kBytes + 1024;                                             \
        if ((e = set_smem(k, smem, SLOT)) != cudaSuccess) return e;                                   \
        k<<<grid, kTcThreads, smem, st>>>(mx, mb, mc, my, d, cs, D, incoming, init_states, seq_idx);  \
        return cudaGetLastError();                                                                    \
    }
    SSD_SCAN_CASE(128, 64, 20)
    SSD_SCAN_CASE(128, 128, 21)
    SSD_SCAN_CASE(256, 64, 22)
    SSD_SCAN_CASE(256, 128, 23)
#undef SSD_SCAN_CASE
    return cudaErrorNotSupported;
}

}  // namespace ssd
