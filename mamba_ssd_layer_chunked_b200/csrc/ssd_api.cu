// ssd_api.cu -- host side of the C ABI declared in include/ssd.h: argument
// validation, workspace sizing, kernel-family selection and the launch
// sequence chunk_cumsum -> chunk_state -> state_passing -> chunk_scan on the
// caller's stream. Nothing here allocates, synchronises or reads device memory.

#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <cstdio>
#include <cstring>

#include "ssd_common.cuh"
#include "ssd_tc.cuh"

// The library's device error word: a kernel whose bounded wait gives up ORs a
// code into it (the output of that call is then invalid). One per device; read
// and cleared by ssd_device_error.
__device__ unsigned int g_ssd_device_error = 0u;

namespace ssd {

cudaError_t device_error_word(unsigned int** out) {
    constexpr int kMaxDevices = 64;
    static std::atomic<unsigned int*> addr[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    unsigned int* a = addr[dev].load(std::memory_order_acquire);
    if (!a) {
        void* p = nullptr;
        if ((e = cudaGetSymbolAddress(&p, g_ssd_device_error)) != cudaSuccess) return e;
        a = static_cast<unsigned int*>(p);
        addr[dev].store(a, std::memory_order_release);  // a race only repeats the lookup
    }
    *out = a;
    return cudaSuccess;
}

}  // namespace ssd

namespace {

thread_local char g_cuda_err[256] = "";

// An NVTX range around the host-side enqueue of one entry point or one kernel
// launch, named after it ("ssd_fwd", "fused_scan", ...): a profiler attaches
// the kernels launched inside a range to its name (Nsight Systems' timeline,
// `ncu --nvtx --nvtx-include`). With no tool attached a push or pop costs one
// check of a function pointer.
struct TraceRange {
    explicit TraceRange(const char* name) { nvtxRangePushA(name); }
    ~TraceRange() { nvtxRangePop(); }
    TraceRange(const TraceRange&) = delete;
    TraceRange& operator=(const TraceRange&) = delete;
};

ssd_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return SSD_OK;
    std::snprintf(g_cuda_err, sizeof(g_cuda_err), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    return SSD_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Host-only checks of the problem description (no device access).
ssd_status check_dims(const ssd_problem* p) {
    if (!p) return SSD_ERR_INVALID_ARG;
    if (p->batch < 1 || p->seqlen < 1 || p->nheads < 1 || p->headdim < 1 || p->dstate < 1 ||
        p->ngroups < 1 || p->chunk < 1 || p->nseq < 1)
        return SSD_ERR_INVALID_ARG;
    if (p->nheads % p->ngroups != 0) return SSD_ERR_INVALID_ARG;
    if (p->dtype != SSD_DTYPE_F32 && p->dtype != SSD_DTYPE_BF16) return SSD_ERR_INVALID_ARG;
    if (p->path != SSD_PATH_AUTO && p->path != SSD_PATH_SIMT && p->path != SSD_PATH_FUSED)
        return SSD_ERR_INVALID_ARG;
    if (p->chunk != 64 && p->chunk != 128 && p->chunk != 256) return SSD_ERR_UNSUPPORTED;
    if (p->headdim % 16 != 0 || p->headdim > 256 || p->dstate % 16 != 0 || p->dstate > 256)
        return SSD_ERR_UNSUPPORTED;
    // grid and index limits: every flattened grid dimension stays below 2^31
    const int64_t nchunks = (p->seqlen + p->chunk - 1) / p->chunk;
    if (p->batch > (1 << 20) || p->seqlen > (1 << 26) || p->nheads > (1 << 16) || p->nseq > (1 << 24))
        return SSD_ERR_UNSUPPORTED;
    if (p->batch * p->nheads * nchunks * 4 > INT32_MAX) return SSD_ERR_UNSUPPORTED;
    if (p->batch * p->seqlen > INT32_MAX) return SSD_ERR_UNSUPPORTED;
    return SSD_OK;
}

// The build targets sm_100a only: the device must be compute capability 10.0.
// Also binds the calling thread to its current device's primary context: this
// library carries its own CUDA runtime, so a host thread that has not used it
// before (a thread per rank, say) would otherwise reach the first launch
// without a current context.
ssd_status check_device() {
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) {
        cudaGetLastError();
        return SSD_ERR_UNSUPPORTED;
    }
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return SSD_ERR_UNSUPPORTED;
    }
    return (major == 10 && minor == 0) ? SSD_OK : SSD_ERR_UNSUPPORTED;
}

ssd::Dims make_dims(const ssd_problem* p) {
    ssd::Dims d;
    d.batch = (int)p->batch;
    d.seqlen = (int)p->seqlen;
    d.nheads = (int)p->nheads;
    d.headdim = (int)p->headdim;
    d.dstate = (int)p->dstate;
    d.ngroups = (int)p->ngroups;
    d.chunk = (int)p->chunk;
    d.nseq = (int)p->nseq;
    d.nchunks = (int)((p->seqlen + p->chunk - 1) / p->chunk);  // the last chunk may be partial
    d.heads_per_group = (int)(p->nheads / p->ngroups);
    return d;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// chunks per row: the last one is partial when chunk does not divide seqlen
int64_t chunk_count(const ssd_problem* p) { return (p->seqlen + p->chunk - 1) / p->chunk; }

// entries of the within-chunk cumsum [b, H, nchunks, Q]
size_t cs_elems(const ssd_problem* p) { return (size_t)p->batch * chunk_count(p) * p->chunk * p->nheads; }

size_t states_bytes(const ssd_problem* p) {
    return (size_t)p->batch * chunk_count(p) * p->nheads * p->dstate * p->headdim * sizeof(float);
}

// family ssd_fwd runs
ssd_path fwd_family(const ssd_problem* p) {
    switch (p->path) {
        case SSD_PATH_SIMT: return SSD_PATH_SIMT;
        case SSD_PATH_FUSED: return SSD_PATH_FUSED;
        default: break;
    }
    if (ssd::fused_fwd_supported(p)) return SSD_PATH_FUSED;
    return SSD_PATH_SIMT;
}

// Workspace of the chunked steps inside ssd_fwd: the cumsum (fp64: the SIMT
// kernels take exp(cs_k - cs_l) from it) and the chunk states.
size_t chunked_workspace_bytes(const ssd_problem* p) {
    return align256(cs_elems(p) * sizeof(double)) + align256(states_bytes(p));
}

// The sequence-parallel summary runs segment_state where the fused family's
// kernels cover p (and the path allows it), else the chunked steps, which need
// a workspace: their cumsum and chunk states, and final states from zero.
bool sp_fused(const ssd_problem* p) {
    return (p->path == SSD_PATH_AUTO || p->path == SSD_PATH_FUSED) && ssd::fused_supported(p);
}

size_t sp_workspace_bytes(const ssd_problem* p) {
    if (sp_fused(p)) return 0;
    return chunked_workspace_bytes(p) +
           align256((size_t)p->batch * p->nseq * p->nheads * p->dstate * p->headdim * sizeof(float));
}

// The fused family on the dstate it was given directly (64 or 128), or on
// slices of at most 128 state rows padded to Np (64 when dstate <= 64, else
// 128): the work-range states of the padded problem, the padded B and C,
// padded initial and final states, and one more Y for slices after the first.
struct FusedPlan {
    bool direct;
    int pieces, np;
};

FusedPlan fused_plan(const ssd_problem* p) {
    FusedPlan f;
    f.direct = p->dstate == 64 || p->dstate == 128;
    f.pieces = (int)((p->dstate + 127) / 128);
    f.np = f.direct ? (int)p->dstate : (p->dstate <= 64 ? 64 : 128);
    return f;
}

struct FusedLayout {
    size_t work, bc, st, y, total;
};

FusedLayout fused_layout(const ssd_problem* p) {
    const FusedPlan f = fused_plan(p);
    ssd::Dims d = make_dims(p);
    d.dstate = f.np;
    FusedLayout l;
    l.work = align256(ssd::fused_workspace_bytes(d, ssd::fused_default_work_tiles(d)));
    l.bc = l.st = l.y = 0;
    if (!f.direct) {
        l.bc = align256((size_t)p->batch * p->seqlen * p->ngroups * f.np * 2);
        l.st = align256((size_t)p->batch * p->nseq * p->nheads * f.np * p->headdim * sizeof(float));
    }
    l.total = l.work + 2 * l.bc + 2 * l.st + l.y;
    return l;
}

// The three fused launches on dims d (dstate 64 or 128), workspace ws.
// Yacc: Y of the state slices before this one, added in the scan's epilogue.
cudaError_t run_fused(const ssd::Dims& d, const void* X, const float* log_a, const void* B, const void* C,
                      const float* D, const float* init_states, const int32_t* seq_idx, void* Y, float* final_states,
                      void* ws, cudaStream_t st, const void* Yacc = nullptr) {
    const int64_t wt = ssd::fused_default_work_tiles(d);
    const size_t nwork = (size_t)ssd::fused_work_count(d, wt);
    const size_t stb = nwork * 2 * d.dstate * d.headdim * sizeof(float);
    float* work_local = static_cast<float*>(ws);
    float* work_in = reinterpret_cast<float*>(static_cast<char*>(ws) + align256(stb));
    float* work_decay = reinterpret_cast<float*>(static_cast<char*>(ws) + 2 * align256(stb));
    const bool cuts = ssd::fused_needs_cut_states(d, wt);
    cudaError_t e = cudaSuccess;
    (void)work_in;  // the fused scan chains the pieces before each cut itself
    if (cuts) {
        TraceRange r("segment_state");
        if ((e = ssd::launch_segment_state(d, wt, X, log_a, B, seq_idx, work_local, work_decay, st)) != cudaSuccess)
            return e;
    }
    TraceRange r("fused_scan");
    return ssd::launch_fused_scan(d, wt, X, log_a, B, C, D, nullptr, init_states, seq_idx, Y, final_states, st,
                                  cuts ? work_local : nullptr, cuts ? work_decay : nullptr, cuts, Yacc);
}

ssd_status check_common(const ssd_problem* p, const int32_t* seq_idx) {
    ssd_status s = check_dims(p);
    if (s != SSD_OK) return s;
    if (!seq_idx && p->nseq != 1) return SSD_ERR_INVALID_ARG;
    return SSD_OK;
}

// Device-dependent checks, run after every host-side argument check.
ssd_status check_runnable(const ssd_problem* p) {
    ssd_status s = check_device();
    if (s != SSD_OK) return s;
    if (p->path == SSD_PATH_FUSED && !ssd::fused_fwd_supported(p)) return SSD_ERR_UNSUPPORTED;
    return SSD_OK;
}

template <typename... Ptrs>
bool all_aligned(Ptrs... ps) {
    const void* arr[] = {static_cast<const void*>(ps)...};
    for (const void* q : arr)
        if (q && !aligned16(q)) return false;
    return true;
}

// log a, D and seq_idx are read one element at a time: their natural 4-byte
// alignment suffices (a segment of a batch-1 tensor, for one, starts wherever
// its first token does)
template <typename... Ptrs>
bool all_aligned4(Ptrs... ps) {
    const void* arr[] = {static_cast<const void*>(ps)...};
    for (const void* q : arr)
        if (q && (reinterpret_cast<uintptr_t>(q) & 3u)) return false;
    return true;
}

}  // namespace

extern "C" {

const char* ssd_status_string(ssd_status s) {
    switch (s) {
        case SSD_OK: return "ok";
        case SSD_ERR_INVALID_ARG: return "invalid argument";
        case SSD_ERR_UNSUPPORTED: return "unsupported problem or device";
        case SSD_ERR_WORKSPACE: return "workspace missing or too small";
        case SSD_ERR_CUDA: return "CUDA error";
        case SSD_ERR_DEVICE_TIMEOUT: return "a device-side wait gave up (outputs invalid)";
    }
    return "unknown status";
}

const char* ssd_last_cuda_error_string(void) { return g_cuda_err; }

ssd_status ssd_device_error(uint32_t* code, void* stream) {
    ssd_status s = check_device();
    if (s != SSD_OK) return s;
    unsigned int* word = nullptr;
    cudaError_t e = ssd::device_error_word(&word);
    if (e != cudaSuccess) return cuda_status(e);
    cudaStream_t st = (cudaStream_t)stream;
    unsigned int v = 0u;
    // the read, then the clear, in stream order; the stream is then drained
    if ((e = cudaMemcpyAsync(&v, word, sizeof(v), cudaMemcpyDeviceToHost, st)) != cudaSuccess ||
        (e = cudaMemsetAsync(word, 0, sizeof(v), st)) != cudaSuccess ||
        (e = cudaStreamSynchronize(st)) != cudaSuccess)
        return cuda_status(e);
    if (code) *code = v;
    return v ? SSD_ERR_DEVICE_TIMEOUT : SSD_OK;
}

ssd_status ssd_check_problem(const ssd_problem* p) {
    ssd_status s = check_dims(p);
    if (s != SSD_OK) return s;
    return check_runnable(p);
}

int ssd_path_supported(const ssd_problem* p, ssd_path path) {
    if (check_dims(p) != SSD_OK || check_device() != SSD_OK) return 0;
    if (path == SSD_PATH_SIMT) return 1;
    if (path == SSD_PATH_FUSED) return ssd::fused_fwd_supported(p) ? 1 : 0;
    return 0;
}

size_t ssd_states_bytes(const ssd_problem* p) {
    if (check_dims(p) != SSD_OK) return (size_t)-1;
    return states_bytes(p);
}

size_t ssd_fwd_workspace_bytes(const ssd_problem* p) {
    if (check_dims(p) != SSD_OK) return (size_t)-1;
    // the family ssd_fwd runs for p (the same host-side decision)
    const ssd_path fam = fwd_family(p);
    return fam == SSD_PATH_FUSED ? fused_layout(p).total : chunked_workspace_bytes(p);
}

int64_t ssd_fused_work_tiles(const ssd_problem* p) {
    if (check_dims(p) != SSD_OK || !ssd::fused_supported(p)) return -1;
    return ssd::fused_default_work_tiles(make_dims(p));
}

int64_t ssd_fused_work_count(const ssd_problem* p, int64_t work_tiles) {
    if (check_dims(p) != SSD_OK) return -1;
    const ssd::Dims d = make_dims(p);
    if (!ssd::fused_work_ok(d, work_tiles)) return -1;
    return ssd::fused_work_count(d, work_tiles);
}

ssd_status ssd_segment_state(const ssd_problem* p, int64_t work_tiles, const void* X, const float* log_a,
                             const void* B, const int32_t* seq_idx, float* work_local, float* work_decay,
                             void* stream) {
    TraceRange trace("ssd_segment_state");
    ssd_status s = check_common(p, seq_idx);
    if (s != SSD_OK) return s;
    if (!X || !log_a || !B || !work_local || !work_decay) return SSD_ERR_INVALID_ARG;
    if (!all_aligned(X, B, work_local, work_decay) || !all_aligned4(log_a, seq_idx)) return SSD_ERR_INVALID_ARG;
    const ssd::Dims d = make_dims(p);
    if (!ssd::fused_work_ok(d, work_tiles)) return SSD_ERR_INVALID_ARG;
    if ((s = check_device()) != SSD_OK) return s;
    if (!ssd::fused_supported(p)) return SSD_ERR_UNSUPPORTED;
    return cuda_status(ssd::launch_segment_state(d, work_tiles, X, log_a, B, seq_idx, work_local, work_decay,
                                                 (cudaStream_t)stream));
}

ssd_status ssd_segment_passing(const ssd_problem* p, int64_t work_tiles, const float* work_local,
                               const float* work_decay, const float* init_states, const int32_t* seq_idx,
                               float* work_incoming, void* stream) {
    TraceRange trace("ssd_segment_passing");
    ssd_status s = check_common(p, seq_idx);
    if (s != SSD_OK) return s;
    if (!work_local || !work_decay || !work_incoming) return SSD_ERR_INVALID_ARG;
    if (!all_aligned(work_local, work_decay, init_states, work_incoming) || !all_aligned4(seq_idx))
        return SSD_ERR_INVALID_ARG;
    const ssd::Dims d = make_dims(p);
    if (!ssd::fused_work_ok(d, work_tiles)) return SSD_ERR_INVALID_ARG;
    if ((s = check_device()) != SSD_OK) return s;
    if (!ssd::fused_supported(p)) return SSD_ERR_UNSUPPORTED;
    return cuda_status(ssd::launch_segment_passing(d, work_tiles, work_local, work_decay, init_states, seq_idx,
                                                   work_incoming, (cudaStream_t)stream));
}

ssd_status ssd_fused_scan(const ssd_problem* p, int64_t work_tiles, const void* X, const float* log_a, const void* B,
                          const void* C, const float* D, const float* work_incoming, const float* init_states,
                          const int32_t* seq_idx, void* Y, float* final_states, void* stream) {
    TraceRange trace("ssd_fused_scan");
    ssd_status s = check_common(p, seq_idx);
    if (s != SSD_OK) return s;
    if (!X || !log_a || !B || !C || !Y) return SSD_ERR_INVALID_ARG;
    if (!all_aligned(X, B, C, work_incoming, init_states, Y, final_states) || !all_aligned4(log_a, D, seq_idx))
        return SSD_ERR_INVALID_ARG;
    const ssd::Dims d = make_dims(p);
    if (!ssd::fused_work_ok(d, work_tiles)) return SSD_ERR_INVALID_ARG;
    if (ssd::fused_needs_cut_states(d, work_tiles) && !work_incoming) return SSD_ERR_INVALID_ARG;
    if ((s = check_device()) != SSD_OK) return s;
    if (!ssd::fused_supported(p)) return SSD_ERR_UNSUPPORTED;
    return cuda_status(ssd::launch_fused_scan(d, work_tiles, X, log_a, B, C, D, work_incoming, init_states, seq_idx,
                                              Y, final_states, (cudaStream_t)stream));
}

ssd_status ssd_fused_scan_chained(const ssd_problem* p, int64_t work_tiles, const void* X, const float* log_a,
                                  const void* B, const void* C, const float* D, const float* work_local,
                                  const float* work_decay, const float* init_states, const int32_t* seq_idx,
                                  void* Y, float* final_states, void* stream) {
    TraceRange trace("ssd_fused_scan_chained");
    ssd_status s = check_common(p, seq_idx);
    if (s != SSD_OK) return s;
    if (!X || !log_a || !B || !C || !Y) return SSD_ERR_INVALID_ARG;
    if (!all_aligned(X, B, C, work_local, work_decay, init_states, Y, final_states) || !all_aligned4(log_a, D, seq_idx))
        return SSD_ERR_INVALID_ARG;
    const ssd::Dims d = make_dims(p);
    if (!ssd::fused_work_ok(d, work_tiles)) return SSD_ERR_INVALID_ARG;
    if (ssd::fused_needs_cut_states(d, work_tiles) && (!work_local || !work_decay)) return SSD_ERR_INVALID_ARG;
    if ((s = check_device()) != SSD_OK) return s;
    if (!ssd::fused_supported(p)) return SSD_ERR_UNSUPPORTED;
    return cuda_status(ssd::launch_fused_scan(d, work_tiles, X, log_a, B, C, D, nullptr, init_states, seq_idx, Y,
                                              final_states, (cudaStream_t)stream, work_local, work_decay));
}

size_t ssd_sp_summary_workspace_bytes(const ssd_problem* p) {
    if (check_dims(p) != SSD_OK) return (size_t)-1;
    return sp_workspace_bytes(p);
}

ssd_status ssd_sp_summary(const ssd_problem* p, const void* X, const float* log_a, const void* B,
                          const int32_t* seq_idx, float* loc, float* dec, int32_t* ids, void* workspace,
                          size_t workspace_bytes, void* stream) {
    TraceRange trace("ssd_sp_summary");
    ssd_status s = check_common(p, seq_idx);
    if (s != SSD_OK) return s;
    if (!X || !log_a || !B || !loc || !dec || !ids) return SSD_ERR_INVALID_ARG;
    if (!all_aligned(X, B, loc, dec, ids, workspace) || !all_aligned4(log_a, seq_idx)) return SSD_ERR_INVALID_ARG;
    const size_t need = sp_workspace_bytes(p);
    if (need > 0 && (!workspace || workspace_bytes < need)) return SSD_ERR_WORKSPACE;
    if ((s = check_runnable(p)) != SSD_OK) return s;
    const ssd::Dims d = make_dims(p);
    cudaStream_t st = (cudaStream_t)stream;
    if (sp_fused(p)) {
        const int64_t nt = ((int64_t)p->seqlen + 127) / 128;  // one work range per (batch row, head pair)
        return cuda_status(ssd::launch_segment_state(d, nt, X, log_a, B, seq_idx, loc, dec, st, ids));
    }
    char* w = static_cast<char*>(workspace);
    float* states = reinterpret_cast<float*>(w + align256(cs_elems(p) * sizeof(double)));
    float* finals = reinterpret_cast<float*>(w + chunked_workspace_bytes(p));
    double* cs = reinterpret_cast<double*>(w);
    cudaError_t e;
    if ((e = ssd::launch_chunk_cumsum(d, log_a, cs, st)) != cudaSuccess ||
        (e = ssd::launch_chunk_state_simt(d, p->dtype, X, B, cs, seq_idx, states, finals, st)) != cudaSuccess ||
        (e = ssd::launch_state_passing(d, cs, states, states, nullptr, seq_idx, finals, st)) != cudaSuccess)
        return cuda_status(e);
    return cuda_status(ssd::launch_sp_finish(d, log_a, seq_idx, finals, loc, dec, ids, st));
}

ssd_status ssd_sp_combine(const ssd_problem* p, int nranks, int rank, const float* g_loc, const float* g_dec,
                          const int32_t* g_ids, const float* init_states, float* init_local, void* stream) {
    TraceRange trace("ssd_sp_combine");
    ssd_status s = check_dims(p);
    if (s != SSD_OK) return s;
    if (nranks < 1 || rank < 0 || rank >= nranks) return SSD_ERR_INVALID_ARG;
    if (!g_loc || !g_dec || !g_ids || !init_local) return SSD_ERR_INVALID_ARG;
    if (!all_aligned(g_loc, g_dec, g_ids, init_states, init_local)) return SSD_ERR_INVALID_ARG;
    if ((p->dstate * p->headdim) % 4 != 0) return SSD_ERR_INVALID_ARG;
    if ((s = check_device()) != SSD_OK) return s;
    return cuda_status(ssd::launch_sp_combine(make_dims(p), nranks, rank, g_loc, g_dec, g_ids, init_states,
                                              init_local, (cudaStream_t)stream));
}

ssd_status ssd_sp_own_finals(const ssd_problem* p, int nranks, int rank, const int32_t* g_ids, float* final_states,
                             void* stream) {
    TraceRange trace("ssd_sp_own_finals");
    ssd_status s = check_dims(p);
    if (s != SSD_OK) return s;
    if (nranks < 1 || rank < 0 || rank >= nranks) return SSD_ERR_INVALID_ARG;
    if (!g_ids || !final_states) return SSD_ERR_INVALID_ARG;
    if (!all_aligned(g_ids, final_states)) return SSD_ERR_INVALID_ARG;
    if ((p->dstate * p->headdim) % 4 != 0) return SSD_ERR_INVALID_ARG;
    if ((s = check_device()) != SSD_OK) return s;
    return cuda_status(
        ssd::launch_sp_own_finals(make_dims(p), nranks, rank, g_ids, final_states, (cudaStream_t)stream));
}

ssd_status ssd_discretize(const ssd_problem* p, const float* dt, const float* dt_bias, const float* A,
                          const void* x, int zoh, float* log_a, void* X, void* stream) {
    TraceRange trace("ssd_discretize");
    if (!p) return SSD_ERR_INVALID_ARG;
    if (p->batch < 1 || p->seqlen < 1 || p->nheads < 1 || p->headdim < 1) return SSD_ERR_INVALID_ARG;
    if (p->dtype != SSD_DTYPE_F32 && p->dtype != SSD_DTYPE_BF16) return SSD_ERR_INVALID_ARG;
    // 16-byte rows: 8 bf16 or 4 fp32 elements per thread
    if (p->headdim % (p->dtype == SSD_DTYPE_F32 ? 4 : 8) != 0) return SSD_ERR_UNSUPPORTED;
    if (p->batch * p->seqlen * p->nheads * p->headdim / 4 > ((int64_t)1 << 40)) return SSD_ERR_UNSUPPORTED;
    if (!dt || !A || !x || !log_a || !X) return SSD_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(dt) & 3u) || (reinterpret_cast<uintptr_t>(dt_bias) & 3u) ||
        (reinterpret_cast<uintptr_t>(A) & 3u) || (reinterpret_cast<uintptr_t>(log_a) & 3u) || !aligned16(x) ||
        !aligned16(X))
        return SSD_ERR_INVALID_ARG;
    ssd_status s = check_device();
    if (s != SSD_OK) return s;
    return cuda_status(ssd::launch_discretize(p->batch * p->seqlen * p->nheads, (int)p->nheads, (int)p->headdim,
                                              p->dtype, dt, dt_bias, A, x, zoh, log_a, X, (cudaStream_t)stream));
}

ssd_status ssd_decode_step(const ssd_problem* p, const void* x, const float* log_a, const void* B, const void* C,
                           const float* D, float* state, void* y, void* stream) {
    TraceRange trace("ssd_decode_step");
    if (!p) return SSD_ERR_INVALID_ARG;
    if (p->batch < 1 || p->nheads < 1 || p->headdim < 1 || p->dstate < 1 || p->ngroups < 1 ||
        p->nheads % p->ngroups != 0)
        return SSD_ERR_INVALID_ARG;
    if (p->dtype != SSD_DTYPE_F32 && p->dtype != SSD_DTYPE_BF16) return SSD_ERR_INVALID_ARG;
    if (p->headdim % 4 != 0 || p->headdim > 1024) return SSD_ERR_UNSUPPORTED;
    if (p->batch * p->nheads > INT32_MAX || p->dstate > (1 << 20)) return SSD_ERR_UNSUPPORTED;
    if (!x || !log_a || !B || !C || !state || !y) return SSD_ERR_INVALID_ARG;
    const uintptr_t vec = p->dtype == SSD_DTYPE_F32 ? 15u : 7u;  // float4 / 4 x bf16 accesses
    if ((reinterpret_cast<uintptr_t>(x) & vec) || (reinterpret_cast<uintptr_t>(y) & vec) || !aligned16(state) ||
        (reinterpret_cast<uintptr_t>(log_a) & 3u) || (reinterpret_cast<uintptr_t>(B) & 1u) ||
        (reinterpret_cast<uintptr_t>(C) & 1u) || (reinterpret_cast<uintptr_t>(D) & 3u))
        return SSD_ERR_INVALID_ARG;
    ssd_status s = check_device();
    if (s != SSD_OK) return s;
    return cuda_status(ssd::launch_decode_step((int)p->batch, (int)p->nheads, (int)p->headdim, (int)p->dstate,
                                               (int)p->ngroups, p->dtype, x, log_a, B, C, D, state, y,
                                               (cudaStream_t)stream));
}

ssd_status ssd_chunk_cumsum(const ssd_problem* p, const float* log_a, float* cs, void* stream) {
    TraceRange trace("ssd_chunk_cumsum");
    ssd_status s = check_dims(p);  // log a only: nseq and seq_idx play no part here
    if (s != SSD_OK) return s;
    if (!log_a || !cs) return SSD_ERR_INVALID_ARG;
    if (!all_aligned(cs) || !all_aligned4(log_a)) return SSD_ERR_INVALID_ARG;
    if ((s = check_device()) != SSD_OK) return s;
    return cuda_status(ssd::launch_chunk_cumsum(make_dims(p), log_a, cs, (cudaStream_t)stream));
}

ssd_status ssd_chunk_state(const ssd_problem* p, const void* X, const void* B, const float* cs,
                           const int32_t* seq_idx, float* states, float* final_states, void* stream) {
    TraceRange trace("ssd_chunk_state");
    ssd_status s = check_common(p, seq_idx);
    if (s != SSD_OK) return s;
    if (!X || !B || !cs || !states) return SSD_ERR_INVALID_ARG;
    if (!all_aligned(X, B, cs, states, final_states) || !all_aligned4(seq_idx)) return SSD_ERR_INVALID_ARG;
    if ((s = check_runnable(p)) != SSD_OK) return s;
    const ssd::Dims d = make_dims(p);
    cudaStream_t st = (cudaStream_t)stream;
    return cuda_status(ssd::launch_chunk_state_simt(d, p->dtype, X, B, cs, seq_idx, states, final_states, st));
}

ssd_status ssd_state_passing(const ssd_problem* p, const float* cs, const float* chunk_states, float* incoming,
                             const float* init_states, const int32_t* seq_idx, float* final_states,
                             void* stream) {
    TraceRange trace("ssd_state_passing");
    ssd_status s = check_common(p, seq_idx);
    if (s != SSD_OK) return s;
    if (!cs || !chunk_states || !incoming) return SSD_ERR_INVALID_ARG;
    if (!all_aligned(cs, chunk_states, incoming, init_states, final_states) || !all_aligned4(seq_idx))
        return SSD_ERR_INVALID_ARG;
    if ((s = check_runnable(p)) != SSD_OK) return s;
    return cuda_status(ssd::launch_state_passing(make_dims(p), cs, chunk_states, incoming, init_states, seq_idx,
                                                 final_states, (cudaStream_t)stream));
}

ssd_status ssd_chunk_scan(const ssd_problem* p, const void* X, const void* B, const void* C, const float* cs,
                          const float* D, const float* incoming, const float* init_states,
                          const int32_t* seq_idx, void* Y, void* stream) {
    TraceRange trace("ssd_chunk_scan");
    ssd_status s = check_common(p, seq_idx);
    if (s != SSD_OK) return s;
    if (!X || !B || !C || !cs || !incoming || !Y) return SSD_ERR_INVALID_ARG;
    if (!all_aligned(X, B, C, cs, incoming, init_states, Y) || !all_aligned4(D, seq_idx)) return SSD_ERR_INVALID_ARG;
    if ((s = check_runnable(p)) != SSD_OK) return s;
    const ssd::Dims d = make_dims(p);
    cudaStream_t st = (cudaStream_t)stream;
    return cuda_status(
        ssd::launch_chunk_scan_simt(d, p->dtype, X, B, C, cs, D, incoming, init_states, seq_idx, Y, st));
}

ssd_status ssd_fwd(const ssd_problem* p, const void* X, const float* log_a, const void* B, const void* C,
                   const float* D, const float* init_states, const int32_t* seq_idx, void* Y,
                   float* final_states, void* workspace, size_t workspace_bytes, void* stream) {
    TraceRange trace("ssd_fwd");
    ssd_status s = check_common(p, seq_idx);
    if (s != SSD_OK) return s;
    if (!X || !log_a || !B || !C || !Y) return SSD_ERR_INVALID_ARG;
    if (!all_aligned(X, B, C, init_states, Y, final_states, workspace) || !all_aligned4(log_a, D, seq_idx))
        return SSD_ERR_INVALID_ARG;
    const size_t need = ssd_fwd_workspace_bytes(p);
    if (!workspace || workspace_bytes < need) return SSD_ERR_WORKSPACE;
    if ((s = check_runnable(p)) != SSD_OK) return s;
    const ssd::Dims d = make_dims(p);
    cudaStream_t st = (cudaStream_t)stream;
    const ssd_path fam = fwd_family(p);
    if (fam == SSD_PATH_FUSED) {
        const FusedPlan f = fused_plan(p);
        if (f.direct)
            return cuda_status(run_fused(d, X, log_a, B, C, D, init_states, seq_idx, Y, final_states, workspace, st));
        // slices of the state rows, each padded to np columns of B and C
        const FusedLayout l = fused_layout(p);
        char* w = static_cast<char*>(workspace);
        void* Bp = w + l.work;
        void* Cp = w + l.work + l.bc;
        float* init_p = reinterpret_cast<float*>(w + l.work + 2 * l.bc);
        float* fin_p = reinterpret_cast<float*>(w + l.work + 2 * l.bc + l.st);
        ssd::Dims dp = d;
        dp.dstate = f.np;
        const int64_t rows = (int64_t)d.batch * d.seqlen * d.ngroups;
        const int64_t S = (int64_t)d.batch * d.nseq * d.nheads;
        cudaError_t e = cudaSuccess;
        for (int k = 0; k < f.pieces && e == cudaSuccess; ++k) {
            const int n0 = 128 * k, wd = d.dstate - n0 < 128 ? d.dstate - n0 : 128;
            if ((e = ssd::launch_pad_bc(B, Bp, rows, d.dstate, n0, wd, f.np, st)) != cudaSuccess) break;
            if ((e = ssd::launch_pad_bc(C, Cp, rows, d.dstate, n0, wd, f.np, st)) != cudaSuccess) break;
            if (init_states &&
                (e = ssd::launch_pad_states(init_states, init_p, S, d.dstate, n0, wd, f.np, d.headdim, st)) !=
                    cudaSuccess)
                break;
            // slices after the first add their Y to the one in place (read in the epilogue)
            if ((e = run_fused(dp, X, log_a, Bp, Cp, k == 0 ? D : nullptr, init_states ? init_p : nullptr, seq_idx, Y,
                               final_states ? fin_p : nullptr, w, st, k > 0 ? Y : nullptr)) != cudaSuccess)
                break;
            if (final_states &&
                (e = ssd::launch_unpad_states(fin_p, final_states, S, d.dstate, n0, wd, f.np, d.headdim, st)) !=
                    cudaSuccess)
                break;
        }
        return cuda_status(e);
    }
    char* w = static_cast<char*>(workspace);
    float* states = reinterpret_cast<float*>(w + align256(cs_elems(p) * sizeof(double)));
    cudaError_t e;
    // the SIMT kernels take the cumsum in fp64 (fp32 parity for strongly decaying heads);
    // state_passing works in place: the chunk states become the incoming states
    double* cs = reinterpret_cast<double*>(w);
    {
        TraceRange r("chunk_cumsum");
        if ((e = ssd::launch_chunk_cumsum(d, log_a, cs, st)) != cudaSuccess) return cuda_status(e);
    }
    {
        TraceRange r("chunk_state");
        if ((e = ssd::launch_chunk_state_simt(d, p->dtype, X, B, cs, seq_idx, states, final_states, st)) !=
            cudaSuccess)
            return cuda_status(e);
    }
    {
        TraceRange r("state_passing");
        if ((e = ssd::launch_state_passing(d, cs, states, states, init_states, seq_idx, final_states, st)) !=
            cudaSuccess)
            return cuda_status(e);
    }
    TraceRange r("chunk_scan");
    return cuda_status(
        ssd::launch_chunk_scan_simt(d, p->dtype, X, B, C, cs, D, states, init_states, seq_idx, Y, st));
}

}  // extern "C"
