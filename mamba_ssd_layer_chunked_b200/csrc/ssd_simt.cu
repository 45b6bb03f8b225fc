// ssd_simt.cu -- the four steps of the SSD block decomposition as SIMT fp32
// kernels: chunk_cumsum, chunk_state, state_passing, chunk_scan.
//
// These are the fp32-input path (their fp32 FMA arithmetic meets a 1e-5
// relative tolerance) and the general fallback for shapes outside the tensor-core
// kernels' domain. chunk_cumsum and state_passing are also the production
// kernels of those two steps for every path.
//
// Source of the decomposition: "Mamba-2: writing the recurrent state as a
// structured matrix" (wq-win.github.io/llm/088-mamba2.html), section 3 (block
// algorithm), and "Mamba-2 - Transformer and SSM share one algebra"
// (awesome.papernotes.org, 2024_mamba2), design 2 (cumsum within chunks,
// L = exp(segment sum), diagonal blocks, right factors, chunk scan, left factors).

#include <atomic>

#include "ssd_common.cuh"

namespace ssd {

namespace {

constexpr int kThreads = 256;

// --------------------------------------------------------------------------
// Step 1: chunk_cumsum. cs[b, h, c, k] = sum_{j<=k} log_a[b, c*Q + j, h].
// grid.x = batch * nchunks, grid.y = head tiles of 32. The [Q x 32] slab of
// log_a is read coalesced (heads contiguous), then each warp scans one head,
// summing in double. CsT is the stored type: fp32 for the step entry points,
// fp64 inside ssd_fwd's SIMT family, whose factors exp(cs_k - cs_l) need the
// difference to fp32 accuracy: a stored fp32 prefix sum carries an absolute
// error of ~6e-8 |cs|, i.e. ~1e-5 relative in the factor once |cs| nears 150
// (strongly decaying heads), which is the fp32 parity bound itself.
// --------------------------------------------------------------------------
template <int Q, typename CsT>
__global__ void __launch_bounds__(kThreads) chunk_cumsum_kernel(Dims d, const float* __restrict__ log_a,
                                                                CsT* __restrict__ cs) {
    __shared__ float slab[Q][33];
    const int c = blockIdx.x % d.nchunks;
    const int b = blockIdx.x / d.nchunks;
    const int h0 = blockIdx.y * 32;
    const int nh = min(32, d.nheads - h0);
    for (int i = threadIdx.x; i < Q * 32; i += kThreads) {
        const int k = i >> 5, j = i & 31;
        float v = 0.f;
        if (j < nh && c * Q + k < d.seqlen) v = log_a[((int64_t)b * d.seqlen + (int64_t)c * Q + k) * d.nheads + h0 + j];
        slab[k][j] = v;
    }
    __syncthreads();
    constexpr int PER = Q / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int j = warp; j < nh; j += kThreads / 32) {
        double v[PER];
        double run = 0.0;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            run += (double)slab[lane * PER + i][j];
            v[i] = run;
        }
        double x = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        const double excl = x - run;
        CsT* out = cs + cs_off(d, b, h0 + j, c) + lane * PER;
#pragma unroll
        for (int i = 0; i < PER; ++i) out[i] = (CsT)(v[i] + excl);
    }
}

// Shared-memory prologue used by the chunk kernels: the chunk's cs row, its
// clamped sequence ids and, per position, the start of its sequence piece
// inside the chunk (pst[k] = first position k' <= k with the same id).
struct ChunkMeta {
    double* cs;  // [Q] (fp64, so that differences of the stored values are exact)
    int* seq;    // [Q]
    int* pst;    // [Q]
};
// shared-memory words (4 bytes) of a ChunkMeta for chunk length Q
__host__ __device__ constexpr int meta_words(int Q) { return 4 * Q; }

__device__ __forceinline__ ChunkMeta chunk_meta_at(float* smem, int Q) {
    return ChunkMeta{reinterpret_cast<double*>(smem), reinterpret_cast<int*>(smem + 2 * Q),
                     reinterpret_cast<int*>(smem + 3 * Q)};
}

template <typename CsT>
__device__ void load_chunk_meta(const Dims& d, const CsT* cs, const int32_t* seq_idx, int b, int h,
                                int c, ChunkMeta m) {
    const int Q = d.chunk;
    const int64_t row = (int64_t)b * d.seqlen;
    for (int k = threadIdx.x; k < Q; k += blockDim.x) {
        m.cs[k] = (double)cs[cs_off(d, b, h, c) + k];
        m.seq[k] = seq_at_padded(seq_idx, row, c * Q + k, d.seqlen, d.nseq);
    }
    __syncthreads();
    // ids are non-decreasing inside a chunk (in contract): the piece start is the
    // lower bound of the id in seq[0..k]; for any input it stays inside [0, k]
    for (int k = threadIdx.x; k < Q; k += blockDim.x) {
        const int v = m.seq[k];
        int lo = 0, hi = k;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (m.seq[mid] < v) lo = mid + 1;
            else hi = mid;
        }
        m.pst[k] = lo;
    }
    __syncthreads();
}

// Pieces of a chunk (maximal runs of one sequence id): starts, ids and count.
// Needs blockDim.x >= Q (256 threads, Q <= 256). seqbuf holds the chunk's ids.
__device__ void chunk_pieces(const int* seqbuf, int Q, int* pstart, int* pseq, int* npieces, int* warp_tot) {
    const int k = threadIdx.x, lane = k & 31, warp = k >> 5;
    const bool flag = k < Q && (k == 0 || seqbuf[k] != seqbuf[k - 1]);
    const unsigned mask = __ballot_sync(0xffffffffu, flag);
    if (lane == 0) warp_tot[warp] = __popc(mask);
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += warp_tot[w];
    if (flag) {
        const int i = base + __popc(mask & ((1u << lane) - 1u));
        pstart[i] = k;
        pseq[i] = seqbuf[k];
    }
    if (k == blockDim.x - 1) {
        int tot = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += warp_tot[w];
        pstart[tot] = Q;
        *npieces = tot;
    }
    __syncthreads();
}

// --------------------------------------------------------------------------
// Step 2: chunk_state (SIMT). For the chunk's last piece [st, Q):
//   states[b,c,h][n,p] = sum_l exp(cs[Q-1] - cs[l]) B_l[n] x_l[p]
// and, if final_states != NULL and seq_idx != NULL, the zero-start partial of
// every other piece (each ends inside the chunk) into final_states[b, s].
// grid.x = (b, h, c) flattened, grid.y = tiles of 8192 outputs; 32 outputs per thread.
// --------------------------------------------------------------------------
template <typename T, typename CsT>
__global__ void __launch_bounds__(kThreads) chunk_state_simt_kernel(Dims d, const T* __restrict__ X,
                                                                    const T* __restrict__ B,
                                                                    const CsT* __restrict__ cs,
                                                                    const int32_t* __restrict__ seq_idx,
                                                                    float* __restrict__ states,
                                                                    float* __restrict__ final_states) {
    extern __shared__ float smem[];
    const int Q = d.chunk, N = d.dstate, P = d.headdim;
    const int c = blockIdx.x % d.nchunks;
    const int bh = blockIdx.x / d.nchunks;
    const int h = bh % d.nheads, b = bh / d.nheads, g = h / d.heads_per_group;
    const ChunkMeta m = chunk_meta_at(smem, Q);
    float* Bs = smem + meta_words(Q);  // [32][N]
    float* Xs = Bs + 32 * N;   // [32][P]
    load_chunk_meta(d, cs, seq_idx, b, h, c, m);

    const int NP = N * P;
    const int tile0 = blockIdx.y * 8192;
    const int t0 = c * Q;
    // pieces from the last one backwards; only the last one unless partials are wanted
    int e = Q - 1;
    while (e >= 0) {
        const int st = m.pst[e];
        const bool last = (e == Q - 1);
        if (!last && (final_states == nullptr || seq_idx == nullptr)) break;
        float acc[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = 0.f;
        const double cs_end = m.cs[e];
        for (int l0 = st; l0 <= e; l0 += 32) {
            const int nl = min(32, e - l0 + 1);
            for (int i = threadIdx.x; i < 32 * N; i += kThreads) {
                const int li = i / N, n = i % N;
                Bs[i] = li < nl && t0 + l0 + li < d.seqlen ? to_f32(B[bc_off(d, b, t0 + l0 + li, g) + n]) : 0.f;
            }
            for (int i = threadIdx.x; i < 32 * P; i += kThreads) {
                const int li = i / P, p = i % P;
                float v = 0.f;
                if (li < nl && t0 + l0 + li < d.seqlen)
                    v = expf((float)(cs_end - m.cs[l0 + li])) * to_f32(X[x_off(d, b, t0 + l0 + li, h) + p]);
                Xs[i] = v;
            }
            __syncthreads();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int o = tile0 + j * kThreads + threadIdx.x;
                if (o < NP) {
                    const int n = o / P, p = o % P;
                    float a = acc[j];
                    for (int li = 0; li < nl; ++li) a = fmaf(Bs[li * N + n], Xs[li * P + p], a);
                    acc[j] = a;
                }
            }
            __syncthreads();
        }
        float* dst = last ? states + st_off(d, b, c, h) : final_states + seqst_off(d, b, m.seq[e], h);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int o = tile0 + j * kThreads + threadIdx.x;
            if (o < NP) dst[o] = acc[j];
        }
        e = st - 1;
    }
}

// --------------------------------------------------------------------------
// Step 3: state_passing. One thread owns 4 consecutive state entries of one
// (b, h); the loop over chunks is sequential:
//   incoming_c = carried H if token cQ continues the sequence of token cQ-1,
//                else the initial state of seq[cQ] (or 0)
//   H_c = exp(cs[Q-1] - cs[st-1]) * H_start + S_c  (st = start of the last piece)
// Partials of sequences that end inside chunk c (written by chunk_state) are
// completed with their decayed starting state; a sequence ending at the chunk
// end gets H_c. grid.x = b * H, grid.y = slices of 1024 entries.
// --------------------------------------------------------------------------
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ float4 axpy4(float a, float4 x, float4 y) {
    return make_float4(fmaf(a, x.x, y.x), fmaf(a, x.y, y.y), fmaf(a, x.z, y.z), fmaf(a, x.w, y.w));
}

template <typename CsT>
__global__ void __launch_bounds__(kThreads) state_passing_kernel(Dims d, const CsT* __restrict__ cs,
                                                                 const float* chunk_states, float* incoming,
                                                                 const float* __restrict__ init_states,
                                                                 const int32_t* __restrict__ seq_idx,
                                                                 float* final_states) {
    __shared__ int pstart[257];
    __shared__ int pseq[257];
    __shared__ int seqbuf[256];
    __shared__ int warp_tot[kThreads / 32];
    __shared__ int npieces;
    const int bh = blockIdx.x;
    const int h = bh % d.nheads, b = bh / d.nheads;
    const int NP = d.dstate * d.headdim;
    const int idx = (blockIdx.y * kThreads + threadIdx.x) * 4;
    const bool active = idx < NP;
    const int Q = d.chunk;
    const int64_t row = (int64_t)b * d.seqlen;
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    auto init_of = [&](int s) -> float4 {
        if (!init_states || !active) return zero;
        return ld4(init_states + seqst_off(d, b, s, h) + idx);
    };
    float4 H = zero;
    int s_prev_last = 0;
    for (int c = 0; c < d.nchunks; ++c) {
        const CsT* csr = cs + cs_off(d, b, h, c);
        // decay over positions (st - 1, e] of the chunk, the difference taken in fp64
        auto piece_decay = [&](int st, int e) {
            return expf((float)((double)csr[e] - (st > 0 ? (double)csr[st - 1] : 0.0)));
        };
        if (seq_idx) {
            __syncthreads();
            if (threadIdx.x < Q) seqbuf[threadIdx.x] = seq_at_padded(seq_idx, row, c * Q + threadIdx.x, d.seqlen, d.nseq);
            __syncthreads();
            chunk_pieces(seqbuf, Q, pstart, pseq, &npieces, warp_tot);
        }
        const int np = seq_idx ? npieces : 1;
        const int s_first = seq_idx ? pseq[0] : 0;
        const int s_last = seq_idx ? pseq[np - 1] : 0;
        const bool continues = (c > 0) && (s_first == s_prev_last);
        const float4 hin = continues ? H : init_of(s_first);
        const float* src = chunk_states + st_off(d, b, c, h);
        float* dst = incoming + st_off(d, b, c, h);
        float4 S = active ? ld4(src + idx) : zero;
        if (active) st4(dst + idx, hin);
        // ids that never occur (between the previous sequence and this chunk's
        // first, or between two pieces of this chunk) keep their initial state
        if (seq_idx && final_states && active) {
            if (!continues)
                for (int s = (c > 0 ? s_prev_last : -1) + 1; s < s_first; ++s)
                    st4(final_states + seqst_off(d, b, s, h) + idx, init_of(s));
            for (int j = 1; j < np; ++j)
                for (int s = pseq[j - 1] + 1; s < pseq[j]; ++s)
                    st4(final_states + seqst_off(d, b, s, h) + idx, init_of(s));
        }
        if (seq_idx && final_states && active) {
            for (int j = 0; j + 1 < np; ++j) {
                const int st = pstart[j], e = pstart[j + 1] - 1, s = pseq[j];
                const float4 hs = (j == 0) ? hin : init_of(s);
                const float decay = piece_decay(st, e);
                float* f = final_states + seqst_off(d, b, s, h) + idx;
                st4(f, axpy4(decay, hs, ld4(f)));
            }
        }
        const int st_last = seq_idx ? pstart[np - 1] : 0;
        const float4 hstart = (np == 1) ? hin : init_of(s_last);
        const float decay = piece_decay(st_last, Q - 1);
        H = axpy4(decay, hstart, S);
        if (final_states && active) {
            bool ends = (c == d.nchunks - 1);
            if (!ends && seq_idx) ends = seq_at(seq_idx, row, (c + 1) * Q, d.nseq) != s_last;
            if (ends) st4(final_states + seqst_off(d, b, s_last, h) + idx, H);
        }
        s_prev_last = s_last;
    }
    // ids after the row's last sequence never occur: they keep their initial state
    if (final_states && seq_idx && active)
        for (int s = s_prev_last + 1; s < d.nseq; ++s) st4(final_states + seqst_off(d, b, s, h) + idx, init_of(s));
}

// --------------------------------------------------------------------------
// Step 4: chunk_scan (SIMT). A block computes 64 rows x P outputs of one chunk:
//   y_k = exp(cs[k] - cs[st_k - 1]) C_k . H_start(k)                (left factor)
//       + sum_{l <= k, same piece} exp(cs[k] - cs[l]) (C_k . B_l) x_l  (diagonal block)
//       + D_h x_k
// grid.x = (b, h, c, row tile) flattened.
// --------------------------------------------------------------------------
constexpr int kRows = 64;
constexpr int kMaxOut = kRows * 256 / kThreads;  // 64 outputs per thread at P = 256

template <typename T, typename CsT>
__global__ void __launch_bounds__(kThreads) chunk_scan_simt_kernel(
    Dims d, const T* __restrict__ X, const T* __restrict__ B, const T* __restrict__ C,
    const CsT* __restrict__ cs, const float* __restrict__ D, const float* __restrict__ incoming,
    const float* __restrict__ init_states, const int32_t* __restrict__ seq_idx, T* __restrict__ Y) {
    extern __shared__ float smem[];
    const int Q = d.chunk, N = d.dstate, P = d.headdim;
    const int ntile = Q / kRows;
    int r = blockIdx.x;
    const int rt = r % ntile;
    r /= ntile;
    const int c = r % d.nchunks;
    r /= d.nchunks;
    const int h = r % d.nheads, b = r / d.nheads, g = h / d.heads_per_group;
    const ChunkMeta m = chunk_meta_at(smem, Q);
    const int NS = N + 1;               // padded row stride of Cs and Bs
    float* Cs = smem + meta_words(Q);   // [64][N+1]
    float* Bs = Cs + kRows * NS;    // [32][N+1]
    float* Xs = Bs + 32 * NS;       // [32][P]
    float* Ws = Xs + 32 * P;        // [64][33]
    float* Hs = Ws + kRows * 33;    // [32][P]
    load_chunk_meta(d, cs, seq_idx, b, h, c, m);
    const int k0 = rt * kRows, t0 = c * Q;
    for (int i = threadIdx.x; i < kRows * N; i += kThreads) {
        const int t = t0 + k0 + i / N;  // positions past the row end: C = 0
        Cs[(i / N) * NS + i % N] = t < d.seqlen ? to_f32(C[bc_off(d, b, t, g) + i % N]) : 0.f;
    }
    __syncthreads();

    const int nout = kRows * P / kThreads;
    float acc[kMaxOut];
#pragma unroll
    for (int j = 0; j < kMaxOut; ++j) acc[j] = 0.f;

    // ---- left factor: the state entering each row's sequence piece ----
    for (int r0 = k0; r0 < k0 + kRows;) {
        const int pst = m.pst[r0];
        int r1 = r0 + 1;
        while (r1 < k0 + kRows && m.pst[r1] == pst) ++r1;
        const float* src = nullptr;
        if (pst == 0) src = incoming + st_off(d, b, c, h);
        else if (init_states) src = init_states + seqst_off(d, b, m.seq[pst], h);
        if (src) {
            for (int n0 = 0; n0 < N; n0 += 32) {
                const int nn = min(32, N - n0);  // N is a multiple of 16, not of 32
                __syncthreads();
                for (int i = threadIdx.x; i < nn * P; i += kThreads) Hs[i] = src[(int64_t)(n0 + i / P) * P + i % P];
                __syncthreads();
#pragma unroll
                for (int j = 0; j < kMaxOut; ++j) {
                    if (j < nout) {
                        const int o = j * kThreads + threadIdx.x;
                        const int rr = o / P, p = o % P;
                        const int k = k0 + rr;
                        if (k >= r0 && k < r1) {
                            float a = acc[j];
#pragma unroll 8
                            for (int n = 0; n < nn; ++n) a = fmaf(Cs[rr * NS + n0 + n], Hs[n * P + p], a);
                            acc[j] = a;
                        }
                    }
                }
            }
        }
        r0 = r1;
    }
#pragma unroll
    for (int j = 0; j < kMaxOut; ++j) {
        if (j < nout) {
            const int o = j * kThreads + threadIdx.x;
            const int k = k0 + o / P;
            const int pst = m.pst[k];
            acc[j] *= expf((float)(m.cs[k] - (pst > 0 ? m.cs[pst - 1] : 0.0)));
        }
    }

    // ---- diagonal block: masked (L o C B^T) X over column tiles of 32 ----
    for (int l0 = 0; l0 < k0 + kRows; l0 += 32) {
        __syncthreads();
        for (int i = threadIdx.x; i < 32 * N; i += kThreads) {
            const int t = t0 + l0 + i / N;
            Bs[(i / N) * NS + i % N] = t < d.seqlen ? to_f32(B[bc_off(d, b, t, g) + i % N]) : 0.f;
        }
        for (int i = threadIdx.x; i < 32 * P; i += kThreads) {
            const int t = t0 + l0 + i / P;
            Xs[i] = t < d.seqlen ? to_f32(X[x_off(d, b, t, h) + i % P]) : 0.f;
        }
        __syncthreads();
        for (int i = threadIdx.x; i < kRows * 32; i += kThreads) {
            const int rr = i / 32, li = i % 32;
            const int k = k0 + rr, l = l0 + li;
            float w = 0.f;
            if (l <= k && m.pst[l] == m.pst[k]) {
                float dot = 0.f;
                for (int n = 0; n < N; ++n) dot = fmaf(Cs[rr * NS + n], Bs[li * NS + n], dot);
                w = expf((float)(m.cs[k] - m.cs[l])) * dot;
            }
            Ws[rr * 33 + li] = w;
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kMaxOut; ++j) {
            if (j < nout) {
                const int o = j * kThreads + threadIdx.x;
                const int rr = o / P, p = o % P;
                float a = acc[j];
#pragma unroll 8
                for (int li = 0; li < 32; ++li) a = fmaf(Ws[rr * 33 + li], Xs[li * P + p], a);
                acc[j] = a;
            }
        }
    }

    // ---- skip term and store ----
    const float dh = D ? D[h] : 0.f;
#pragma unroll
    for (int j = 0; j < kMaxOut; ++j) {
        if (j < nout) {
            const int o = j * kThreads + threadIdx.x;
            const int rr = o / P, p = o % P;
            if (t0 + k0 + rr >= d.seqlen) continue;  // past the row end of a partial last chunk
            const int64_t off = x_off(d, b, t0 + k0 + rr, h) + p;
            float y = acc[j];
            if (D) y = fmaf(dh, to_f32(X[off]), y);
            Y[off] = from_f32<T>(y);
        }
    }
}

}  // namespace

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------

cudaError_t ensure_smem_attr(const void* func, int bytes, int slot) {
    // one flag per (slot, device); setting the attribute twice is harmless
    static std::atomic<unsigned> done[64][16];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (slot < 0 || slot >= 64 || dev < 0 || dev >= 16)
        return cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    unsigned prev = done[slot][dev].load(std::memory_order_acquire);
    if (prev >= (unsigned)bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done[slot][dev].store((unsigned)bytes, std::memory_order_release);
    return e;
}

namespace {

// shared-memory attribute slots: 0-3 with fp32 cs, 4-7 with fp64 cs
template <typename CsT>
constexpr int cs_slot() {
    return sizeof(CsT) == 8 ? 4 : 0;
}

template <typename CsT>
cudaError_t chunk_cumsum_impl(const Dims& d, const float* log_a, CsT* cs, cudaStream_t st) {
    dim3 grid(d.batch * d.nchunks, (d.nheads + 31) / 32);
    switch (d.chunk) {
        case 64: chunk_cumsum_kernel<64, CsT><<<grid, kThreads, 0, st>>>(d, log_a, cs); break;
        case 128: chunk_cumsum_kernel<128, CsT><<<grid, kThreads, 0, st>>>(d, log_a, cs); break;
        case 256: chunk_cumsum_kernel<256, CsT><<<grid, kThreads, 0, st>>>(d, log_a, cs); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

template <typename CsT>
cudaError_t chunk_state_simt_impl(const Dims& d, ssd_dtype dt, const void* X, const void* B, const CsT* cs,
                                  const int32_t* seq_idx, float* states, float* final_states, cudaStream_t st) {
    const int smem = (meta_words(d.chunk) + 32 * d.dstate + 32 * d.headdim) * 4;
    dim3 grid(d.batch * d.nheads * d.nchunks, (d.dstate * d.headdim + 8191) / 8192);
    cudaError_t e;
    if (dt == SSD_DTYPE_F32) {
        auto k = chunk_state_simt_kernel<float, CsT>;
        if ((e = ensure_smem_attr((const void*)k, smem, cs_slot<CsT>() + 0)) != cudaSuccess) return e;
        k<<<grid, kThreads, smem, st>>>(d, (const float*)X, (const float*)B, cs, seq_idx, states, final_states);
    } else {
        auto k = chunk_state_simt_kernel<__nv_bfloat16, CsT>;
        if ((e = ensure_smem_attr((const void*)k, smem, cs_slot<CsT>() + 1)) != cudaSuccess) return e;
        k<<<grid, kThreads, smem, st>>>(d, (const __nv_bfloat16*)X, (const __nv_bfloat16*)B, cs, seq_idx, states,
                                        final_states);
    }
    return cudaGetLastError();
}

template <typename CsT>
cudaError_t state_passing_impl(const Dims& d, const CsT* cs, const float* chunk_states, float* incoming,
                               const float* init_states, const int32_t* seq_idx, float* final_states,
                               cudaStream_t st) {
    dim3 grid(d.batch * d.nheads, (d.dstate * d.headdim + 4 * kThreads - 1) / (4 * kThreads));
    state_passing_kernel<CsT><<<grid, kThreads, 0, st>>>(d, cs, chunk_states, incoming, init_states, seq_idx,
                                                         final_states);
    return cudaGetLastError();
}

template <typename CsT>
cudaError_t chunk_scan_simt_impl(const Dims& d, ssd_dtype dt, const void* X, const void* B, const void* C,
                                 const CsT* cs, const float* D, const float* incoming, const float* init_states,
                                 const int32_t* seq_idx, void* Y, cudaStream_t st) {
    const int smem = (meta_words(d.chunk) + kRows * (d.dstate + 1) + 32 * (d.dstate + 1) + 32 * d.headdim +
                      kRows * 33 + 32 * d.headdim) * 4;
    dim3 grid(d.batch * d.nheads * d.nchunks * (d.chunk / kRows));
    cudaError_t e;
    if (dt == SSD_DTYPE_F32) {
        auto k = chunk_scan_simt_kernel<float, CsT>;
        if ((e = ensure_smem_attr((const void*)k, smem, cs_slot<CsT>() + 2)) != cudaSuccess) return e;
        k<<<grid, kThreads, smem, st>>>(d, (const float*)X, (const float*)B, (const float*)C, cs, D, incoming,
                                        init_states, seq_idx, (float*)Y);
    } else {
        auto k = chunk_scan_simt_kernel<__nv_bfloat16, CsT>;
        if ((e = ensure_smem_attr((const void*)k, smem, cs_slot<CsT>() + 3)) != cudaSuccess) return e;
        k<<<grid, kThreads, smem, st>>>(d, (const __nv_bfloat16*)X, (const __nv_bfloat16*)B,
                                        (const __nv_bfloat16*)C, cs, D, incoming, init_states, seq_idx,
                                        (__nv_bfloat16*)Y);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_cumsum(const Dims& d, const float* log_a, float* cs, cudaStream_t st) {
    return chunk_cumsum_impl(d, log_a, cs, st);
}
cudaError_t launch_chunk_cumsum(const Dims& d, const float* log_a, double* cs, cudaStream_t st) {
    return chunk_cumsum_impl(d, log_a, cs, st);
}

cudaError_t launch_chunk_state_simt(const Dims& d, ssd_dtype dt, const void* X, const void* B,
                                    const float* cs, const int32_t* seq_idx, float* states,
                                    float* final_states, cudaStream_t st) {
    return chunk_state_simt_impl(d, dt, X, B, cs, seq_idx, states, final_states, st);
}
cudaError_t launch_chunk_state_simt(const Dims& d, ssd_dtype dt, const void* X, const void* B,
                                    const double* cs, const int32_t* seq_idx, float* states,
                                    float* final_states, cudaStream_t st) {
    return chunk_state_simt_impl(d, dt, X, B, cs, seq_idx, states, final_states, st);
}

cudaError_t launch_state_passing(const Dims& d, const float* cs, const float* chunk_states, float* incoming,
                                 const float* init_states, const int32_t* seq_idx, float* final_states,
                                 cudaStream_t st) {
    return state_passing_impl(d, cs, chunk_states, incoming, init_states, seq_idx, final_states, st);
}
cudaError_t launch_state_passing(const Dims& d, const double* cs, const float* chunk_states, float* incoming,
                                 const float* init_states, const int32_t* seq_idx, float* final_states,
                                 cudaStream_t st) {
    return state_passing_impl(d, cs, chunk_states, incoming, init_states, seq_idx, final_states, st);
}

cudaError_t launch_chunk_scan_simt(const Dims& d, ssd_dtype dt, const void* X, const void* B, const void* C,
                                   const float* cs, const float* D, const float* incoming,
                                   const float* init_states, const int32_t* seq_idx, void* Y, cudaStream_t st) {
    return chunk_scan_simt_impl(d, dt, X, B, C, cs, D, incoming, init_states, seq_idx, Y, st);
}
cudaError_t launch_chunk_scan_simt(const Dims& d, ssd_dtype dt, const void* X, const void* B, const void* C,
                                   const double* cs, const float* D, const float* incoming,
                                   const float* init_states, const int32_t* seq_idx, void* Y, cudaStream_t st) {
    return chunk_scan_simt_impl(d, dt, X, B, C, cs, D, incoming, init_states, seq_idx, Y, st);
}

}  // namespace ssd
