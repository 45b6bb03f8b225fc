// ssd_sp.cu -- sequence parallelism: every batch row's tokens split into
// consecutive segments, one per rank.
//
// The recurrence H_t = a_t H_{t-1} + B_t x_t^T is affine in the state, so over
// a segment the state at its end is E = dec * H_start + loc, where loc is the
// end state reached from a zero state at the start of the segment's last
// sequence piece and dec the product of a over that piece ("Mamba-2: writing
// the recurrent state as a structured matrix", wq-win section 3: the chunk's
// local end state and block decay, here for a whole segment; the pages'
// sequence-parallel variant exchanges exactly these per-segment states). Each
// rank computes (loc, dec) and its first and last sequence ids (segment_state
// in whole-row mode where the fused family's kernels cover the problem, else
// the chunked steps from zero initial states and sp_finish), the ranks
// all-gather them, and each rank chains the
// segments before its own (sp_combine) to get the state entering its first
// token, which then runs the ordinary forward pass as that sequence's initial
// state. Final states: the rank holding a sequence's last token owns it
// (sp_own_finals zeroes the others), and a sum over ranks assembles them.
//
// Layouts: g_loc [R, batch, nheads, dstate, headdim] fp32; g_dec [R, batch,
// nheads] fp32; g_ids [R, batch, 2] int32 (first id, last id of the segment);
// init_states / init_local / final_states [batch, nseq, nheads, dstate, headdim].

#include "ssd_common.cuh"

namespace ssd {

namespace {

constexpr int kSpThreads = 256;

// init_local[b, s, h] = the state entering rank `rank`'s first token for the
// sequence s it continues, else init_states[b, s, h] (or zero). Chain over the
// earlier ranks j: start_j = E_{j-1} when segment j is one sequence piece that
// continues rank j-1's last sequence, else the initial state of its last
// sequence; E_j = dec_j start_j + loc_j.
// Index split of thread i over [b, s, h, NP4] in the index type I (32-bit
// where the element count fits: a 64-bit division by a runtime divisor costs
// more than the rest of these threads' work).
template <typename I>
struct BshIndex {
    int b, s, h, e4;
    __device__ BshIndex(I i, const Dims& d, I NP4) {
        const I bsh = i / NP4;
        e4 = (int)(i - bsh * NP4);
        const I bs = bsh / (I)d.nheads;
        h = (int)(bsh - bs * (I)d.nheads);
        const I bb = bs / (I)d.nseq;
        s = (int)(bs - bb * (I)d.nseq);
        b = (int)bb;
    }
};

template <typename I>
__global__ void __launch_bounds__(kSpThreads) sp_combine_kernel(Dims d, int nranks, int rank,
                                                                const float4* __restrict__ g_loc,
                                                                const float* __restrict__ g_dec,
                                                                const int32_t* __restrict__ g_ids,
                                                                const float4* __restrict__ init_states,
                                                                float4* __restrict__ init_local, I n_all) {
    const int NP4 = d.dstate * d.headdim / 4;
    const I i = (I)blockIdx.x * kSpThreads + threadIdx.x;
    if (i >= n_all) return;
    const BshIndex<I> x(i, d, (I)NP4);
    const int b = x.b, s = x.s, h = x.h, e4 = x.e4;
    auto init_of = [&](int sq) -> float4 {
        return init_states ? init_states[seqst_off(d, b, sq, h) / 4 + e4] : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    const int32_t* ids = g_ids + 2 * b;  // rank j: ids[2 * batch * j], ids[2 * batch * j + 1]
    const int64_t rs_ids = 2 * (int64_t)d.batch;
    float4 v = init_of(s);
    const int first = ids[rs_ids * rank];
    if (rank > 0 && s == first && ids[rs_ids * (rank - 1) + 1] == first) {
        const int64_t rs_loc = (int64_t)d.batch * d.nheads * NP4;
        const int64_t bh = (int64_t)b * d.nheads + h;
        float4 E = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < rank; ++j) {
            const int fj = ids[rs_ids * j], lj = ids[rs_ids * j + 1];
            const bool carried = j > 0 && fj == lj && ids[rs_ids * (j - 1) + 1] == fj;
            const float4 st = carried ? E : init_of(lj);
            const float a = g_dec[(int64_t)j * d.batch * d.nheads + bh];
            const float4 l = g_loc[rs_loc * j + bh * NP4 + e4];
            E = make_float4(fmaf(a, st.x, l.x), fmaf(a, st.y, l.y), fmaf(a, st.z, l.z), fmaf(a, st.w, l.w));
        }
        v = E;
    }
    init_local[i] = v;
}

// zero final_states[b, s] unless rank is its owner: the last rank whose first
// id is <= s (rank 0 when there is none)
template <typename I>
__global__ void __launch_bounds__(kSpThreads) sp_own_finals_kernel(Dims d, int nranks, int rank,
                                                                   const int32_t* __restrict__ g_ids,
                                                                   float4* __restrict__ final_states, I n_all) {
    const int NP4 = d.dstate * d.headdim / 4;
    const I i = (I)blockIdx.x * kSpThreads + threadIdx.x;
    if (i >= n_all) return;
    const BshIndex<I> x(i, d, (I)NP4);
    const int b = x.b, s = x.s;
    int owner = 0;
    for (int j = 0; j < nranks; ++j)
        if (g_ids[2 * ((int64_t)j * d.batch + b)] <= s) owner = j;
    if (owner != rank) final_states[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// The summary from the chunked steps' final states (zero initial states), one
// block per (b, h): loc = the final state of the segment's last sequence (its
// piece here started from zero), dec = exp of the sum of log a over that
// piece, ids = the first and last sequence ids of the row (ids ascend along a
// row, so the piece starts at the first token carrying the last id).
__global__ void __launch_bounds__(kSpThreads) sp_finish_kernel(Dims d, const float* __restrict__ log_a,
                                                               const int32_t* __restrict__ seq_idx,
                                                               const float* __restrict__ finals,
                                                               float* __restrict__ loc, float* __restrict__ dec,
                                                               int32_t* __restrict__ ids) {
    __shared__ float part[kSpThreads / 32];
    const int64_t bh = blockIdx.x;
    const int b = (int)(bh / d.nheads), h = (int)(bh % d.nheads);
    const int64_t row = (int64_t)b * d.seqlen;
    const int first = seq_at(seq_idx, row, 0, d.nseq), last = seq_at(seq_idx, row, d.seqlen - 1, d.nseq);
    int lo = 0, hi = d.seqlen - 1;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (seq_at(seq_idx, row, mid, d.nseq) < last) lo = mid + 1;
        else hi = mid;
    }
    float acc = 0.f;
    for (int t = lo + (int)threadIdx.x; t < d.seqlen; t += kSpThreads) acc += log_a[(row + t) * d.nheads + h];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        float s = 0.f;
        for (int w = 0; w < kSpThreads / 32; ++w) s += part[w];
        dec[bh] = expf(s);
        if (h == 0) {
            ids[2 * b] = first;
            ids[2 * b + 1] = last;
        }
    }
    const int NP = d.dstate * d.headdim;
    const float* src = finals + seqst_off(d, b, last, h);
    float* dst = loc + bh * NP;
    for (int i = (int)threadIdx.x; i < NP; i += kSpThreads) dst[i] = src[i];
}

unsigned blocks_for(int64_t n) { return (unsigned)((n + kSpThreads - 1) / kSpThreads); }

// grids of one thread per float4 of the state arrays stay within 2^31 - 1 blocks
bool grid_fits(int64_t n) { return (n + kSpThreads - 1) / kSpThreads <= INT32_MAX; }

}  // namespace

cudaError_t launch_sp_combine(const Dims& d, int nranks, int rank, const float* g_loc, const float* g_dec,
                              const int32_t* g_ids, const float* init_states, float* init_local, cudaStream_t st) {
    const int64_t n = (int64_t)d.batch * d.nseq * d.nheads * (d.dstate * d.headdim / 4);
    if (n == 0) return cudaSuccess;
    if (!grid_fits(n)) return cudaErrorInvalidConfiguration;
    if (n + kSpThreads < (int64_t)UINT32_MAX)
        sp_combine_kernel<uint32_t><<<blocks_for(n), kSpThreads, 0, st>>>(
            d, nranks, rank, (const float4*)g_loc, g_dec, g_ids, (const float4*)init_states, (float4*)init_local,
            (uint32_t)n);
    else
        sp_combine_kernel<int64_t><<<blocks_for(n), kSpThreads, 0, st>>>(
            d, nranks, rank, (const float4*)g_loc, g_dec, g_ids, (const float4*)init_states, (float4*)init_local, n);
    return cudaGetLastError();
}

cudaError_t launch_sp_finish(const Dims& d, const float* log_a, const int32_t* seq_idx, const float* finals,
                             float* loc, float* dec, int32_t* ids, cudaStream_t st) {
    const int64_t n = (int64_t)d.batch * d.nheads;
    if (n == 0) return cudaSuccess;
    sp_finish_kernel<<<(unsigned)n, kSpThreads, 0, st>>>(d, log_a, seq_idx, finals, loc, dec, ids);
    return cudaGetLastError();
}

cudaError_t launch_sp_own_finals(const Dims& d, int nranks, int rank, const int32_t* g_ids, float* final_states,
                                 cudaStream_t st) {
    const int64_t n = (int64_t)d.batch * d.nseq * d.nheads * (d.dstate * d.headdim / 4);
    if (n == 0) return cudaSuccess;
    if (!grid_fits(n)) return cudaErrorInvalidConfiguration;
    if (n + kSpThreads < (int64_t)UINT32_MAX)
        sp_own_finals_kernel<uint32_t><<<blocks_for(n), kSpThreads, 0, st>>>(d, nranks, rank, g_ids,
                                                                             (float4*)final_states, (uint32_t)n);
    else
        sp_own_finals_kernel<int64_t><<<blocks_for(n), kSpThreads, 0, st>>>(d, nranks, rank, g_ids,
                                                                            (float4*)final_states, n);
    return cudaGetLastError();
}

}  // namespace ssd
