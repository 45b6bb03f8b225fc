/*
 * ssd.h -- C ABI of the B200 (sm_100a) SSD chunked-scan forward library
 * (libssd_b200.so).
 *
 * The operation is the Mamba-2 SSD layer (A, X, B, C) -> Y for a scalar decay
 * per head. For every batch row b and head h, with group g = h / (nheads/ngroups):
 *
 *   H_t = a_t H_{t-1} + B_t x_t^T,   y_t = C_t^T H_t + D_h x_t,   a_t = exp(log_a_t)
 *
 * with H_t in R^{dstate x headdim}. Source: "Mamba-2: writing the recurrent state
 * as a structured matrix" (wq-win.github.io/llm/088-mamba2.html), section 2.1
 * (recurrence and unrolled sum) and section 2.2 (dual form Y = [L o (C B^T)] X,
 * L_ts = prod_{j=s+1..t} a_j); the D x skip term is the discrete state space form
 * of "Mamba and state space models" (wang-x-xia.github.io), section 2.
 *
 * The library computes it with the block decomposition of the same page,
 * section 3 ("Mamba-2 - Transformer and SSM share one algebra",
 * awesome.papernotes.org, design 2, gives the same four steps): within-chunk
 * cumulative sum of log a (chunk_cumsum), per-chunk end states with a zero
 * incoming state (chunk_state), a short scan of the states over chunks
 * (state_passing), and the per-chunk output = masked quadratic term plus the
 * incoming state decayed to each position and read out by C (chunk_scan).
 *
 * Conventions (all entry points):
 *  - All tensor pointers are DEVICE pointers owned by the caller. The library
 *    never allocates, frees or synchronises, never exits or aborts, and keeps no
 *    mutable global state besides a per-device cache of kernel attributes that
 *    is set once. Every call is asynchronous on `stream` (a cudaStream_t passed
 *    as void*; NULL means the legacy default stream) and is thread-safe.
 *  - Layouts are dense row-major (C order) with the last dimension contiguous.
 *    Every pointer must be 16-byte aligned, except log_a, D and seq_idx,
 *    which are read one element at a time and need only their natural 4-byte
 *    alignment (a segment of a batch-1 tensor starts wherever its first token
 *    does); the exceptions each entry point states.
 *  - Arguments are validated on the host before anything is launched; on an
 *    error status nothing has been enqueued. SSD_ERR_CUDA reports a launch
 *    error (the message of cudaGetLastError is available from
 *    ssd_last_cuda_error_string on the calling thread).
 *  - seq_idx is device memory and is never read on the host. In-contract values
 *    are: seq_idx[b, 0] = 0, non-decreasing along t, steps of 0 or 1, and every
 *    value < nseq. A change between t-1 and t starts an independent sequence:
 *    its state starts from init_states[b, seq_idx[b, t]] (or zero) and the
 *    finished sequence's state becomes its final state (the pages require that
 *    only independent-sample boundaries stop state propagation: section 2.3 and
 *    the section 5 testing advice of the wq-win page). Out-of-contract values
 *    give unspecified results but never out-of-bounds accesses (kernels clamp
 *    ids to [0, nseq)).
 *  - init_states is the state before the first token of each sequence (H_{-1}):
 *    the first a_t decays it (the chunk-split example of the wq-win page,
 *    section 2.3, decays the carried state 5 by 0.5).
 *  - final_states[b, s] is the state after the last token of sequence s; ids
 *    in (seq_idx[b, seqlen-1], nseq) that never occur keep their initial state
 *    (or zero).
 */
#ifndef SSD_B200_H
#define SSD_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1,  /* null required pointer, bad dims, misaligned pointer */
    SSD_ERR_UNSUPPORTED = 2,  /* valid problem this build or device cannot run */
    SSD_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required */
    SSD_ERR_CUDA = 4,         /* a CUDA call or kernel launch failed */
    SSD_ERR_DEVICE_TIMEOUT = 5  /* ssd_device_error: a kernel's bounded wait gave up */
} ssd_status;

typedef enum {
    SSD_DTYPE_F32 = 0,   /* X, B, C, Y in fp32 */
    SSD_DTYPE_BF16 = 1   /* X, B, C, Y in bfloat16 */
} ssd_dtype;

/* Kernel family.
 *   SIMT     the four steps as fp32 SIMT kernels (any supported shape, fp32 or bf16);
 *   FUSED    the two-level tensor-core path of ssd_segment_state /
 *            ssd_segment_passing / ssd_fused_scan (bf16, headdim 64 or 128, dstate
 *            a multiple of 16 up to 256, any number of heads per group; any chunk):
 *            the state stays on chip within a work range and crosses HBM only
 *            where a range boundary cuts a row. (The fused step entry points
 *            below take headdim 64, dstate 64 or 128 and an even number of heads
 *            per group; ssd_fwd covers the rest of the family's domain.)
 * AUTO picks FUSED where the problem allows it, else SIMT. An explicit family
 * outside its domain returns SSD_ERR_UNSUPPORTED. (Value 2 is not used.) */
typedef enum {
    SSD_PATH_AUTO = 0,
    SSD_PATH_SIMT = 1,
    SSD_PATH_FUSED = 3
} ssd_path;

typedef struct {
    int64_t batch;     /* b  >= 1 */
    int64_t seqlen;    /* T  >= 1, any length: on the chunked families the last chunk
                          may be partial */
    int64_t nheads;    /* H  >= 1, a multiple of ngroups */
    int64_t headdim;   /* P: multiple of 16, <= 256 */
    int64_t dstate;    /* N: multiple of 16, <= 256 */
    int64_t ngroups;   /* G: heads h*G/H .. share B, C group g */
    int64_t chunk;     /* Q: 64, 128 or 256 */
    int64_t nseq;      /* sequences per batch row: 1 when seq_idx is NULL */
    ssd_dtype dtype;   /* dtype of X, B, C and Y; log_a, D and states are fp32 */
    ssd_path path;
} ssd_problem;

/* Status text, static storage. */
const char* ssd_status_string(ssd_status s);

/* Text of the last CUDA error seen by an entry point on the calling thread
 * ("" if none). */
const char* ssd_last_cuda_error_string(void);

/*
 * ssd_device_error: the failure report of the kernels' bounded waits. The
 * tensor-core kernels wait on shared-memory barriers for their copies and
 * matrix products; every such wait is bounded (about 2 s), and a wait that
 * gives up lets its CTA run to its end without hanging or faulting, where the
 * CTA sets a bit in a device-wide 32-bit error word: the outputs of that call
 * are then INVALID, although the call itself returned SSD_OK (the library does not
 * synchronise, so the launch cannot see it). The word is per device and shared
 * by every call and stream since it was last cleared.
 * This entry point enqueues a read of the word on `stream`, then its clearing,
 * and SYNCHRONISES `stream` (the one entry point that does). *code (if
 * code is non-NULL) receives the word: 0, or bit 0 for a barrier wait that
 * gave up. Returns SSD_OK when the word was 0, SSD_ERR_DEVICE_TIMEOUT when it
 * was not, SSD_ERR_CUDA if the read failed. The pages have no counterpart.
 */
ssd_status ssd_device_error(uint32_t* code, void* stream);

/* ssd_selftest_wait_timeout: checks the report above end to end. Launches one
 * small kernel whose single wait, limited to limit_ns (1000 .. 10^9, else
 * SSD_ERR_INVALID_ARG), is on a barrier that nothing completes: the wait gives
 * up and sets the error word exactly as a production kernel's would, and the
 * kernel ends normally (no copy or product is in flight). The next
 * ssd_device_error then returns SSD_ERR_DEVICE_TIMEOUT and clears the word.
 * Asynchronous on `stream`. The pages have no counterpart. */
ssd_status ssd_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/* Host-side validation of a problem (no device access besides querying the
 * current device's compute capability). */
ssd_status ssd_check_problem(const ssd_problem* p);

/* 1 if `path` (SIMT or FUSED) can run problem p on the current device. */
int ssd_path_supported(const ssd_problem* p, ssd_path path);

/* Bytes of workspace ssd_fwd needs for p, or (size_t)-1 if p is invalid: for
 * the family ssd_fwd runs (p->path, or for AUTO the fused family where it
 * applies, else the chunked SIMT one), the chunked need (the chunk cumulative
 * sums, batch*nchunks*chunk*nheads fp64 values, and one state per chunk,
 * batch*nchunks*nheads*dstate*headdim fp32) or the fused path's (two states and
 * two decays per work range, see ssd_fused_work_tiles, plus the padded slices
 * when dstate is not 64 or 128), each part 256-byte aligned. */
size_t ssd_fwd_workspace_bytes(const ssd_problem* p);

/*
 * ssd_fwd: the whole forward pass, Y and final states from X, log a, B, C.
 *   X            [batch, seqlen, nheads, headdim]            dtype, required
 *   log_a        [batch, seqlen, nheads]                     fp32, required; finite,
 *                                                            <= 0 is the tested domain
 *   B, C         [batch, seqlen, ngroups, dstate]            dtype, required
 *   D            [nheads]                                    fp32 or NULL (= 0)
 *   init_states  [batch, nseq, nheads, dstate, headdim]      fp32 or NULL (= 0)
 *   seq_idx      [batch, seqlen]                             int32 or NULL (one sequence)
 *   Y            [batch, seqlen, nheads, headdim]            dtype, out, required
 *   final_states [batch, nseq, nheads, dstate, headdim]      fp32, out, or NULL
 *   workspace    >= ssd_fwd_workspace_bytes(p) bytes of device memory (its
 *                contents on entry are ignored; on exit they are unspecified)
 * Y is rounded to nearest even from the fp32 result when dtype is bf16.
 */
ssd_status ssd_fwd(const ssd_problem* p, const void* X, const float* log_a, const void* B,
                   const void* C, const float* D, const float* init_states,
                   const int32_t* seq_idx, void* Y, float* final_states, void* workspace,
                   size_t workspace_bytes, void* stream);

/* Size of the fixed scratch array used by ssd_fwd_noalloc (64 MiB). */
#define SSD_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/*
 * ssd_fwd_noalloc: ssd_fwd without a workspace argument, for callers that may
 * not allocate device memory (hosts that plan all device memory ahead of time,
 * or loops that cannot afford an allocation's implicit synchronisation). The
 * pages have no counterpart of this entry point; it only changes where the
 * scratch lives.
 *   Arguments, layouts and results are those of ssd_fwd. The scratch is a fixed
 *   SSD_NOALLOC_SCRATCH_BYTES array in the library's device memory, reserved on
 *   every GPU that loads the library until the process exits; nothing is
 *   allocated per call.
 *   Problems with ssd_fwd_workspace_bytes(p) > SSD_NOALLOC_SCRATCH_BYTES return
 *   SSD_ERR_WORKSPACE before anything is launched.
 *   The first call on a device looks the array's address up (once per device,
 *   with that device current); make that first call before any stream capture.
 *   If the lookup fails the call returns SSD_ERR_CUDA.
 *   All calls share the one array: calls that may overlap on the GPU (other
 *   streams or threads) race on it, so the caller must order them. Leftover
 *   contents from earlier calls are harmless: every scratch byte is written
 *   before it is read.
 */
ssd_status ssd_fwd_noalloc(const ssd_problem* p, const void* X, const float* log_a, const void* B,
                           const void* C, const float* D, const float* init_states,
                           const int32_t* seq_idx, void* Y, float* final_states, void* stream);

/* ---- the four steps, callable one by one (ssd_fwd runs them in this order) ----
 * nchunks = ceil(seqlen / chunk). cs is [batch, nheads, nchunks, chunk] fp32; a
 * "state buffer" is [batch, nchunks, nheads, dstate, headdim] fp32. Positions of
 * a partial last chunk past the row end count as tokens with log a = 0 and
 * x = B = C = 0 in the last token's sequence: they change no state, cs stays
 * constant over them, and no Y is written for them. */

/* Bytes of one state buffer. */
size_t ssd_states_bytes(const ssd_problem* p);

/* Step 1, chunk_cumsum: cs[b, h, c, k] = sum_{j <= k} log_a[b, c*chunk + j, h],
 * the within-chunk inclusive cumulative sum; exp(cs[k] - cs[l]) is the decay
 * prod_{j=l+1..k} a_j of the segment mask L (papernotes design 2, "A_cumsum"
 * and "L = exp(segment_sum(A))"). Summed in fp64, stored as fp32: a stored
 * value carries ~6e-8 |cs| of absolute error, so exp(cs[k] - cs[l]) from these
 * steps is good to ~1e-7 |cs| relative (ssd_fwd's SIMT family keeps the sums in
 * fp64 internally, which the 1e-5 fp32 parity needs once |cs| nears 100). */
ssd_status ssd_chunk_cumsum(const ssd_problem* p, const float* log_a, float* cs, void* stream);

/* Step 2, chunk_state: per chunk c, the end state of the chunk's LAST sequence
 * piece with a zero incoming state,
 *   states[b, c, h] = sum_{l in last piece} exp(cs[Q-1] - cs[l]) B_l x_l^T
 * (wq-win section 3 "local_end_state"; papernotes design 2 right factors).
 * When seq_idx and final_states are both non-NULL, it also writes, for every
 * sequence s that ends strictly inside chunk c at token e, the zero-start partial
 * sum_{l in s's piece of c, l <= e} exp(cs[e] - cs[l]) B_l x_l^T into
 * final_states[b, s]; ssd_state_passing completes those entries. */
ssd_status ssd_chunk_state(const ssd_problem* p, const void* X, const void* B, const float* cs,
                           const int32_t* seq_idx, float* states, float* final_states,
                           void* stream);

/* Step 3, state_passing: the short recurrence over chunks
 *   H_c = exp(cs_c[Q-1] - cs_c[st-1]) H_start + S_c
 * (wq-win section 3 "real_end_state = block_decay * previous_state +
 * local_end_state"; st is the start of the chunk's last piece, cs[-1] = 0,
 * H_start is the carried state or, after a boundary, the new sequence's initial
 * state). Reads the chunk states from `chunk_states` and writes the INCOMING
 * state of every chunk (the state before its first token, for that token's
 * sequence) to `incoming`; the two may be the same buffer (in place). Writes
 * final_states when non-NULL (completing the partials of ssd_chunk_state). */
ssd_status ssd_state_passing(const ssd_problem* p, const float* cs, const float* chunk_states,
                             float* incoming, const float* init_states, const int32_t* seq_idx,
                             float* final_states, void* stream);

/* Step 4, chunk_scan: per chunk,
 *   y_k = sum_{l <= k, same sequence} exp(cs[k] - cs[l]) (C_k . B_l) x_l
 *       + exp(cs[k] - cs[st_k - 1]) C_k^T H_start(k) + D_h x_k
 * (wq-win section 3: local_output = (L o C B^T) X plus the incoming state decayed
 * to each position and read out by C; H_start(k) is `incoming[b, c, h]` for the
 * chunk's first sequence and init_states (or zero) for a sequence starting at
 * st_k inside the chunk). */
ssd_status ssd_chunk_scan(const ssd_problem* p, const void* X, const void* B, const void* C,
                          const float* cs, const float* D, const float* incoming,
                          const float* init_states, const int32_t* seq_idx, void* Y,
                          void* stream);

/* ---- the fused path: the same block decomposition at two levels ----
 * Each batch row is split into head pairs (heads 2j, 2j+1) and each (batch
 * row, head pair) "row" into ceil(seqlen / 128) tiles of 128 tokens (the last
 * may be shorter). The rows' tiles, laid end to end in the order (batch row,
 * head pair, tile), are cut into `nwork` work ranges of `work_tiles` tiles (the
 * last may be shorter): nwork = ceil(batch * nheads/2 * ceil(seqlen/128) /
 * work_tiles). One CTA walks one range and carries the state on chip from
 * tile to tile; a range may start or end inside a row, and only the states at
 * those cuts go through HBM. Buffers indexed by range i:
 *   work_local / work_incoming  [nwork, 2, dstate, headdim] fp32 (the two heads
 *                               of the row the range ends / starts in)
 *   work_decay                  [nwork, 2] fp32
 * These entry points take bf16, headdim 64, dstate 64 or 128 and an even
 * number of heads per group (SSD_ERR_UNSUPPORTED elsewhere); 1 <= work_tiles
 * <= the number of tiles, else SSD_ERR_INVALID_ARG. */

/* Tiles per range ssd_fwd uses for p on the current device (about one range
 * per SM), or -1 if p is invalid or outside the fused domain. */
int64_t ssd_fused_work_tiles(const ssd_problem* p);

/* nwork for p and work_tiles, or -1 if either is invalid. */
int64_t ssd_fused_work_count(const ssd_problem* p, int64_t work_tiles);

/* Right factors at the cuts: for every range i whose last piece [s0, s1) ends
 * inside its row (s1 < seqlen), over the last sequence piece [st, s1) of it:
 *   work_local[i, j]  = sum_{l in [st, s1)} (prod_{k=l+1..s1-1} a_k) B_l x_l^T
 *   work_decay[i, j]  = prod_{k in [st, s1)} a_k        (head 2 hp + j)
 * (wq-win section 3, "local_end_state" and "block_decay", for a block that is
 * a range's piece). Terms that reach s1 through a product of a below e^-40 for
 * both heads of the pair are left out (below the fp32 rounding of the rest),
 * and work_decay is then 0. Entries of ranges that end at a row end are not
 * written. */
ssd_status ssd_segment_state(const ssd_problem* p, int64_t work_tiles, const void* X, const float* log_a,
                             const void* B, const int32_t* seq_idx, float* work_local, float* work_decay,
                             void* stream);

/* Centre factors: over the pieces of each row in order, H_end = decay *
 * H_start + local for every piece that ends inside the row, with H_start =
 * H_end of the previous piece when the piece's last sequence continues from
 * it, else that sequence's initial state (or zero). For every range i whose
 * first piece starts inside its row, writes work_incoming[i, j]: the state
 * entering that piece for the sequence of its first token (H_end of the
 * previous piece when that token continues the previous token's sequence,
 * else its initial state or zero). Other entries are not written. */
ssd_status ssd_segment_passing(const ssd_problem* p, int64_t work_tiles, const float* work_local,
                               const float* work_decay, const float* init_states,
                               const int32_t* seq_idx, float* work_incoming, void* stream);

/* Per range: walks 128-token tiles aligned to sequence starts; per tile
 *   y_k = sum_{l <= k in tile} exp(cs_k - cs_l) (C_k . B_l) x_l + exp(cs_k) C_k^T H + D_h x_k
 *   H  <- exp(cs_end) H + sum_{l in tile} exp(cs_end - cs_l) B_l x_l^T
 * starting from work_incoming[i] (the output of ssd_segment_passing) when the
 * range starts inside a row, and from the initial state (or zero) for every
 * sequence that starts in the range; writes Y and, when non-NULL,
 * final_states for every sequence that ends in the range (and the initial
 * state for ids after a row's last sequence). work_incoming may be NULL when
 * no range starts inside a row (nwork == 1, or work_tiles a multiple of
 * ceil(seqlen / 128)). */
ssd_status ssd_fused_scan(const ssd_problem* p, int64_t work_tiles, const void* X, const float* log_a,
                          const void* B, const void* C, const float* D, const float* work_incoming,
                          const float* init_states, const int32_t* seq_idx, void* Y,
                          float* final_states, void* stream);

/* ---- sequence parallelism: each batch row's tokens in consecutive segments,
 * one per rank (rank r holds tokens [t_r, t_{r+1}) of every row; segments may
 * differ in length; seq_idx ids ascend along a row as everywhere) ----
 * Over a segment the recurrence is affine in its state: the state after the
 * segment is E = dec * H_start + loc, with loc the state reached from zero at
 * the start of the segment's last sequence piece and dec the product of a over
 * that piece (wq-win section 3: a block's local end state and block decay, for
 * a block that is a whole segment; the pages' sequence-parallel scheme
 * exchanges these per-segment states once). Per rank: ssd_sp_summary on its
 * segment, an all-gather of (loc, dec, ids) over the R ranks (in rank order),
 * ssd_sp_combine for the initial states of its segment, ssd_fwd with them; for
 * final states, ssd_sp_own_finals on ssd_fwd's final states and a sum over
 * the ranks. p is the rank's local problem (seqlen = its segment length).
 *   loc   [batch, nheads, dstate, headdim] fp32     dec [batch, nheads] fp32
 *   ids   [batch, 2] int32: the segment's first and last sequence id (0, 0
 *         without seq_idx)
 *   g_loc, g_dec, g_ids: the R ranks' loc, dec, ids stacked in rank order
 *   init_states, init_local, final_states [batch, nseq, nheads, dstate, headdim]
 * ssd_sp_summary runs segment_state (whole-row ranges) where those kernels
 * cover p (bf16, headdim 64, dstate 64 or 128, an even number of heads per
 * group; path AUTO or FUSED): no workspace, and dec is 0 where the product is
 * below e^-40 (the start state's share of E is then below the rounding of
 * loc). Elsewhere it runs the chunked steps (chunk length p->chunk) from zero
 * initial states: loc is the last sequence's final state, dec the exp of the
 * fp32 sum of log a over its piece; that needs a device workspace of
 * ssd_sp_summary_workspace_bytes(p) bytes (16-byte aligned, contents
 * overwritten; SSD_ERR_WORKSPACE when missing or smaller). The caller owns
 * every buffer; nothing is allocated. */
size_t ssd_sp_summary_workspace_bytes(const ssd_problem* p);  /* (size_t)-1 on invalid p */
ssd_status ssd_sp_summary(const ssd_problem* p, const void* X, const float* log_a, const void* B,
                          const int32_t* seq_idx, float* loc, float* dec, int32_t* ids, void* workspace,
                          size_t workspace_bytes, void* stream);

/* init_local[b, s] = the state entering this rank's first token when that
 * token continues sequence s from the previous rank, else init_states[b, s]
 * (or zero when init_states is NULL). The state entering rank r is E_{r-1},
 * chained over ranks j < r: E_j = dec_j * start_j + loc_j, start_j = E_{j-1}
 * when segment j is one sequence piece continuing rank j-1's last sequence,
 * else the initial state of segment j's last sequence. Reads only batch,
 * nheads, dstate, headdim, nseq of p. */
ssd_status ssd_sp_combine(const ssd_problem* p, int nranks, int rank, const float* g_loc, const float* g_dec,
                          const int32_t* g_ids, const float* init_states, float* init_local, void* stream);

/* Zeroes final_states[b, s] (in place) unless this rank owns sequence s of
 * row b: the last rank whose first id is <= s (rank 0 when none is), which
 * holds s's last token or, for an id that never occurs, reports its initial
 * state. Summing the ranks' results gives the final states of the whole
 * sequence. Reads only batch, nheads, dstate, headdim, nseq of p. */
ssd_status ssd_sp_own_finals(const ssd_problem* p, int nranks, int rank, const int32_t* g_ids, float* final_states,
                             void* stream);

/* ssd_fused_scan with the centre factors folded in: each range that starts
 * inside a row chains the pieces of that row before its cut itself, from
 * work_local / work_decay (the output of ssd_segment_state), by the rule of
 * ssd_segment_passing; ssd_fwd runs the fused family as ssd_segment_state
 * then this. work_local and work_decay may be NULL when no range starts
 * inside a row. */
ssd_status ssd_fused_scan_chained(const ssd_problem* p, int64_t work_tiles, const void* X, const float* log_a,
                                  const void* B, const void* C, const float* D, const float* work_local,
                                  const float* work_decay, const float* init_states, const int32_t* seq_idx,
                                  void* Y, float* final_states, void* stream);

/* ---- discretisation: the step before the scan in the Mamba block ----
 * For every (b, t, h), with z = dt[b, t, h] + dt_bias[h]:
 *   delta = softplus(z) = log(1 + exp(z)),   log_a[b, t, h] = delta * A[h]
 *   X[b, t, h, :] = s * x[b, t, h, :],  s = delta                    (zoh == 0)
 *                                       s = (exp(delta A) - 1) / A   (zoh != 0; delta when A == 0)
 * (ai.tomabc.com "Mamba": delta = softplus(linear + bias), A_bar = exp(delta A);
 * wang-x-xia "Mamba and state space models" section 2: zero-order hold). X and
 * log_a are the X and log_a inputs of ssd_fwd: zoh == 0 puts B_bar = delta B on
 * x, zoh != 0 the zero-order-hold B_bar = (exp(delta A) - 1) / A B.
 *   dt, log_a   [batch, seqlen, nheads]           fp32
 *   dt_bias, A  [nheads] fp32 (dt_bias may be NULL => 0; A <= 0 expected)
 *   x, X        [batch, seqlen, nheads, headdim]  p->dtype (X may alias x)
 * Only batch, seqlen, nheads, headdim (a multiple of 8 for bf16, of 4 for
 * fp32: 16-byte rows) and dtype of p are read; x and X 16-byte aligned.
 * SSD_ERR_INVALID_ARG / SSD_ERR_UNSUPPORTED before any launch. */
ssd_status ssd_discretize(const ssd_problem* p, const float* dt, const float* dt_bias, const float* A,
                          const void* x, int zoh, float* log_a, void* X, void* stream);

/* ---- decoding: one step of the recurrence with an fp32 state cache ----
 * For every (b, h), with g = h / (nheads / ngroups) and a = exp(log_a[b, h]):
 *   state[b, h] <- a * state[b, h] + B[b, g] x[b, h]^T      (in place)
 *   y[b, h]      = C[b, g]^T state[b, h] + D[h] x[b, h]
 * (wang-x-xia "Mamba and state space models" section 2; wq-win section 2.1):
 * the same recurrence as ssd_fwd, one token at a time, so that a sequence fed
 * token by token from init_states gives ssd_fwd's Y and final states.
 *   x, y      [batch, nheads, headdim]            p->dtype
 *   log_a     [batch, nheads]                     fp32
 *   B, C      [batch, ngroups, dstate]            p->dtype
 *   D         [nheads] fp32 or NULL (=> 0)
 *   state     [batch, nheads, dstate, headdim]    fp32, read and written
 * Only batch, nheads, headdim (a multiple of 4, at most 1024), dstate, ngroups
 * and dtype of p are read. Pointers 16-byte aligned (x, y: 8-byte for bf16).
 * SSD_ERR_INVALID_ARG / SSD_ERR_UNSUPPORTED on bad arguments before any
 * launch; asynchronous on `stream`. */
ssd_status ssd_decode_step(const ssd_problem* p, const void* x, const float* log_a, const void* B, const void* C,
                           const float* D, float* state, void* y, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SSD_B200_H */
