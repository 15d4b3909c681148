/*
 * moba.h - C ABI of the B200 MoBA (Mixture of Block Attention) causal prefill forward.
 *
 * The operation is the one defined on the page "《MoBA: Mixture of Block Attention for
 * Long-Context LLMs》深度解读报告" (an analysis of the MoBA paper), sections 2.1-2.3 and 3.2:
 *
 *   1. every packed sequence is cut into blocks of `chunk_size` tokens (§2.1);
 *   2. each block is summarised per KV head by the mean of its keys (§2.2);
 *   3. each query row (token t, query head h) scores every block j of its sequence by
 *      s_j = <q, mean_j> (§2.2);
 *   4. blocks after the row's own block c are masked to -inf, block c is always taken
 *      and the best `topk - 1` blocks j < c are routed (§2.3, hard top-k of §2.2);
 *   5. the row attends, softmax-normalised, over the union of its selected blocks, with a
 *      causal mask inside block c (§2.2-§2.3); the history blocks and the current block are
 *      computed separately and merged by their log-sum-exp (§3.2).
 *
 * Conventions shared by every entry point
 *   - Tensors are packed varlen ("THD"): q is bf16 [T, Hq, d], k and v are bf16 [T, Hkv, d],
 *     row-major, rows of all sequences back to back.  cu_seqlens is int32 [batch + 1],
 *     cu_seqlens[0] = 0, non-decreasing, cu_seqlens[batch] = T.  The caller guarantees
 *     cu_seqlens matches `total_tokens`; it is read on the device only.
 *   - GQA: query head h reads KV head h / (Hq / Hkv).
 *   - Blocks are numbered globally, sequence by sequence: the blocks of sequence i are
 *     cu_blocks[i] .. cu_blocks[i+1]-1 with cu_blocks[i+1]-cu_blocks[i] = ceil(L_i / chunk).
 *     A final partial block is allowed; its mean is over its valid tokens.
 *   - Selections are int32 [Hq, T, topk]: block indices local to the row's sequence,
 *     ascending, padded with -1.  `topk` counts the forced current block.
 *   - All device pointers are owned by the caller, must be 16-byte aligned and stay valid
 *     until the work on `stream` finishes.  The library allocates no device memory and keeps
 *     no state between calls, apart from the static scratch array behind
 *     moba_attn_fwd_noalloc (see below).  `stream` is a cudaStream_t (NULL = legacy default
 *     stream).
 *   - Every call checks its arguments on the host and returns a status before launching
 *     anything; on success all work is queued asynchronously on `stream`.  A launch failure
 *     returns MOBA_ERR_CUDA.  moba_last_error() describes the most recent failure of the
 *     calling host thread.
 *   - GPU path limits: head_dim in {64, 128}; chunk_size a positive multiple of 128;
 *     1 <= topk <= 32; Hq % Hkv == 0.  Other values return MOBA_ERR_UNSUPPORTED
 *     (or MOBA_ERR_INVALID_ARG when they are meaningless, e.g. topk < 1).
 */
#ifndef MOBA_H_
#define MOBA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOBA_OK = 0,
    MOBA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, Hq % Hkv != 0, topk < 1 ... */
    MOBA_ERR_UNSUPPORTED = 2,   /* valid but outside the GPU path limits above */
    MOBA_ERR_WORKSPACE = 3,     /* workspace pointer NULL or smaller than moba_workspace_size */
    MOBA_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
    MOBA_ERR_DEVICE_TIMEOUT = 5 /* a bounded device-side wait gave up (see moba_device_status) */
} moba_status;

typedef struct {
    int batch;            /* number of packed sequences, >= 1 */
    int total_tokens;     /* T = cu_seqlens[batch], >= 0 */
    int max_seqlen;       /* length of the longest sequence, or 0 when not known on the host.
                             When given it must satisfy max_seqlen <= T <= batch * max_seqlen
                             (else MOBA_ERR_INVALID_ARG) and the caller guarantees that no
                             sequence is longer; it sizes the gate by the most blocks one
                             sequence has (ceil(max_seqlen / chunk_size)) instead of by the
                             block count of the whole batch.  A sequence longer than a given
                             max_seqlen never causes an out-of-bounds access: rows of its
                             blocks past the bound may select their own block only, and
                             moba_attn_fwd then records MOBA_ERR_INVALID_ARG in its status
                             word (moba_device_status). */
    int num_q_heads;      /* Hq >= 1 */
    int num_kv_heads;     /* Hkv >= 1, Hq % Hkv == 0 */
    int head_dim;         /* d */
    int chunk_size;       /* B, tokens per block */
    int topk;             /* blocks per query row, counting its own block */
    float softmax_scale;  /* logit scale of the attention softmax; <= 0 means 1/sqrt(d) */
    int wave_tokens;      /* moba_attn_fwd only: query tokens per wave, 0 = all tokens in one
                             wave; otherwise a positive multiple of 128.  Bounds the workspace
                             (per-wave partial outputs), see moba_workspace_size. */
    int gate;             /* moba_attn_fwd / moba_attn_fwd_noalloc only: the block summary the
                             gate scores against, MOBA_GATE_MEAN (0, the paper's mean pooling)
                             or MOBA_GATE_MINMAX (1, the min/max summary, see
                             moba_gate_minmax_topk).  Other values: MOBA_ERR_INVALID_ARG. */
} moba_params;

enum { MOBA_GATE_MEAN = 0, MOBA_GATE_MINMAX = 1 };

/* Optional instrumentation for moba_attn_fwd.  All fields may be left zero. */
typedef struct {
    void** events;   /* in: cudaEvent_t array or NULL.  When non-NULL the call records
                        events[MOBA_EV_*] (and, per wave w, events[MOBA_EV_WAVE0 + 4*w + i])
                        on `stream` at the stage boundaries listed below, as long as the
                        index is < n_events. */
    int n_events;
    int launches;    /* out: number of kernel launches the call queued */
    int waves;       /* out: number of query waves */
    int gate_path;   /* out: which gate kernel ran, MOBA_GATE_PATH_* */
} moba_run_info;

enum {
    MOBA_GATE_PATH_NONE = 0,         /* no gate (the selection came in through sel_in) */
    MOBA_GATE_PATH_TENSOR_CORES = 1, /* tcgen05 gate: every sequence has <= 257 blocks (the
                                        longest by max_seqlen, else the whole call's bound) */
    MOBA_GATE_PATH_CUDA_CORES = 2    /* fp32 CUDA-core gate: a sequence may have more */
};

enum {
    MOBA_EV_BEGIN = 0,      /* before the first launch */
    MOBA_EV_MEANS_DONE = 1, /* after the mean-pool kernel */
    MOBA_EV_GATE_DONE = 2,  /* after the gate kernel (same point as 1 when sel_in is given) */
    MOBA_EV_WAVE0 = 3       /* per wave w: +4w route start, +4w+1 attention start,
                               +4w+2 attention end, +4w+3 merge end */
};

/* Upper bound of the total number of blocks, ceil(T / B) + batch - 1 (0 when T = 0).
 * Size k_mean buffers with it when the exact count is not known on the host.
 * Returns -1 when params are invalid. */
int moba_num_blocks_bound(const moba_params* p);

/* Bytes of device workspace moba_attn_fwd needs for these params (wave size included).
 * Returns 0 when params are invalid. */
size_t moba_workspace_size(const moba_params* p);

/* Step 2 (analysis §2.2): k_mean[b, g, :] = mean over the valid tokens of block b of
 * k[t, g, :], fp32 accumulation, fp32 out.
 *   k        bf16 [T, Hkv, d] device
 *   cu_seqlens int32 [batch + 1] device
 *   k_mean   fp32 [NB, Hkv, d] device, NB >= the true block count (moba_num_blocks_bound
 *            is always enough); rows past the true count are left untouched.
 * Uses no workspace. */
moba_status moba_meanpool(const moba_params* p, const void* k, const int* cu_seqlens,
                          float* k_mean, void* stream);

/* Min/max block summary, the Quest-style alternative to the mean (the analysis names Quest as
 * the MoBA variant with min/max pooling, §1.3, and as the stronger summary, §5.1 item 6 and
 * §6.3; the summary is Quest's): k_min[b, g, i] and k_max[b, g, i] = minimum and maximum of
 * k[t, g, i] over the valid tokens t of block b.  Exact (the extrema of bf16 values are bf16).
 *   k              bf16 [T, Hkv, d] device
 *   cu_seqlens     int32 [batch + 1] device
 *   k_min, k_max   bf16 [NB, Hkv, d] device each, NB as for moba_meanpool; rows past the true
 *                  block count are left untouched
 * Uses no workspace; asynchronous on `stream`; argument errors return before any launch. */
moba_status moba_minmaxpool(const moba_params* p, const void* k, const int* cu_seqlens,
                            void* k_min, void* k_max, void* stream);

/* Steps 3-4 (analysis §2.2-§2.3): per query row, gate scores against the means of the past
 * blocks of its sequence (fp32), future blocks excluded, the own block forced, the best
 * topk-1 past blocks kept (ties to the lower block index).
 *   q       bf16 [T, Hq, d] device
 *   k_mean  fp32 [NB, Hkv, d] device, as written by moba_meanpool
 *   sel     int32 [Hq, T, topk] device, written in full (ascending, -1 padded).
 * Uses no workspace. */
moba_status moba_gate_topk(const moba_params* p, const void* q, const float* k_mean,
                           const int* cu_seqlens, int* sel, void* stream);

/* Steps 3-4 with the min/max (Quest-style) block summary in place of the mean (the analysis
 * names Quest as the MoBA variant that pools blocks by min and max, §1.3, the stronger summary,
 * §5.1 item 6 and §6.3): an earlier block j is scored by
 *   s_j = sum_i max(q_i k_min[j, g, i], q_i k_max[j, g, i])
 * (the largest q . x over the block's bounding box), computed exactly as
 * q+ . k_max_j + q- . k_min_j with q+ = max(q, 0), q- = min(q, 0) on the tensor cores (bf16
 * products exact, fp32 sum).  Mask, forced own block, top-k and tie rule as moba_gate_topk.
 *   q              bf16 [T, Hq, d] device
 *   k_min, k_max   bf16 [NB, Hkv, d] device, as written by moba_minmaxpool
 *   sel            int32 [Hq, T, topk] device, written in full (ascending, -1 padded)
 * Every sequence must have at most 257 blocks (bounded by max_seqlen, else by the whole
 * call's block count), else MOBA_ERR_UNSUPPORTED.  Uses no workspace. */
moba_status moba_gate_minmax_topk(const moba_params* p, const void* q, const void* k_min,
                                  const void* k_max, const int* cu_seqlens, int* sel, void* stream);

/* The whole forward (steps 1-5): mean-pool, gate (unless sel_in is given), routing of rows
 * to (KV head, block) lists, block attention on the tensor cores, log-sum-exp merge.
 *   q, k, v     bf16 device, see conventions
 *   sel_in      int32 [Hq, T, topk] device or NULL.  NULL: the gate runs.  Otherwise the
 *               selection is taken from it (e.g. the oracle's): per row, entries in [0, c)
 *               are routed past blocks (the first topk-1 such entries, in row order), the
 *               own block c is always attended whether listed or not, anything else is
 *               ignored.
 *   sel_out     int32 [Hq, T, topk] device or NULL: receives the gate's selection (ignored
 *               when sel_in is given).
 *   workspace   device, >= moba_workspace_size(p) bytes, 256-byte aligned
 *   out         bf16 [T, Hq, d] device (fp32 merge rounded to nearest even)
 *   lse         fp32 [Hq, T] device: natural-log log-sum-exp of the scaled logits
 *   info        optional instrumentation, may be NULL
 * With p->gate = MOBA_GATE_MINMAX the gate scores with the min/max summary (computed in the
 * workspace, in place of the means) as moba_gate_minmax_topk does, under its 257-block limit.
 * Workspace contents are undefined after the call. */
moba_status moba_attn_fwd(const moba_params* p, const void* q, const void* k, const void* v,
                          const int* cu_seqlens, const int* sel_in, int* sel_out,
                          void* workspace, size_t workspace_bytes, void* out, float* lse,
                          moba_run_info* info, void* stream);

/* ---- Backward pass --------------------------------------------------------------------
 *
 * Gradients of the forward's out and lse with respect to q, k and v.  The analysis page of the
 * MoBA paper trains with MoBA (§3.3: continual pre-training up to 1M tokens) and makes it a
 * parameter-equivalent replacement of full attention (§2.5): the gate has no parameters and
 * routes by hard top-k (§2.2), so the selection is piecewise constant and the gradient flows
 * only through the softmax attention over the selected blocks (§2.2-§2.3).  The backward
 * therefore holds the forward's selection fixed and differentiates the attention:
 *   p_u = exp(scale q.k_u - lse),  dv_u += p_u dO,  dz_u = p_u (dO.v_u - <dO, out> + d_lse),
 *   dq = scale sum_u dz_u k_u,  dk_u += scale dz_u q  (summed over the query heads of a KV head).
 *   q, k, v      bf16, as for moba_attn_fwd
 *   out, lse     the forward's outputs (bf16 [T, Hq, d], fp32 [Hq, T])
 *   d_out        bf16 [T, Hq, d]; d_lse fp32 [Hq, T] or NULL (zero)
 *   sel          int32 [Hq, T, topk]: the selection the forward used (moba_attn_fwd's sel_out, or
 *                the sel_in it was given), read with the same rule as sel_in
 *   workspace    >= moba_bwd_workspace_size(p) bytes, 256-byte aligned (routing lists of all
 *                rows and an fp32 dq accumulator [T, Hq, d]); p->wave_tokens is ignored
 *   dq           bf16 [T, Hq, d]; dk, dv bf16 [T, Hkv, d]: written in full
 * Runs on the tensor cores (tcgen05); asynchronous on `stream`; argument errors return before
 * any launch; T * Hq * topk must stay below 2^31 (MOBA_ERR_UNSUPPORTED).  A bounded device wait
 * that gives up is reported through moba_device_status on this workspace. */
size_t moba_bwd_workspace_size(const moba_params* p);
moba_status moba_attn_bwd(const moba_params* p, const void* q, const void* k, const void* v,
                          const void* out, const float* lse, const void* d_out, const float* d_lse,
                          const int* cu_seqlens, const int* sel, void* workspace,
                          size_t workspace_bytes, void* dq, void* dk, void* dv, void* stream);

/* Reads (synchronously, on `stream`) the device status word a previous moba_attn_fwd (or
 * moba_attn_bwd) left in `workspace`: MOBA_OK, or MOBA_ERR_DEVICE_TIMEOUT when a bounded device-side wait gave up.
 * Waits for the stream. */
moba_status moba_device_status(const moba_params* p, const void* workspace, void* stream);

/* ---- Decode step -------------------------------------------------------------------------
 *
 * One new query per sequence against its KV cache (the analysis page of the MoBA paper,
 * §2.2-§2.3, applied to the query at the last cache row t = L-1 of each sequence; the
 * partial results per block are merged as in §3.2).  Exactly the prefill forward's row t:
 * the own block c = (L-1) / chunk_size is forced (attended whole), the topk-1 best earlier
 * blocks by q . mean_j are routed (ties to the lower index), softmax over the union.
 *   p->batch         number of sequences (= query rows); p->total_tokens = T, the cache rows
 *   q                bf16 [batch, Hq, d]: the new token's query of each sequence
 *   k, v             bf16 [T, Hkv, d] packed caches (cu_seqlens); each sequence's last row is
 *                    the new token's key / value
 *   cu_seqlens       int32 [batch + 1], device; an empty sequence yields out = 0, lse = -inf
 *   k_mean           fp32 [NB, Hkv, d]: the block means moba_meanpool computes for these
 *                    caches, NB >= the true block count (moba_num_blocks_bound(p) is always
 *                    enough; only complete earlier blocks are read).  The Python binding,
 *                    which cannot see the true count without a device sync, asks for the bound
 *   workspace        moba_decode_workspace_size(p) bytes, caller-owned device memory
 *   out              bf16 [batch, Hq, d]; lse fp32 [Hq, batch] (natural log, scale included)
 * Runs on the CUDA cores (HBM-bound: it streams the selected K/V blocks).  Asynchronous on
 * `stream`; argument errors return before any launch.  batch <= 65535. */
size_t moba_decode_workspace_size(const moba_params* p);
moba_status moba_decode_fwd(const moba_params* p, const void* q, const void* k, const void* v,
                            const int* cu_seqlens, const float* k_mean, void* workspace,
                            size_t ws_bytes, void* out, float* lse, void* stream);

/* The decode step with the min/max gate: as moba_decode_fwd, except that an earlier block j
 * is scored by s_j = sum_i max(q_i k_min[j, g, i], q_i k_max[j, g, i]) (fp32; Quest's bound of
 * q . k over the block), from the summary moba_minmaxpool computes for these caches:
 *   k_min, k_max   bf16 [NB, Hkv, d] device each, NB as for k_mean
 * Same workspace (moba_decode_workspace_size), outputs, errors and limits. */
moba_status moba_decode_minmax_fwd(const moba_params* p, const void* q, const void* k, const void* v,
                                   const int* cu_seqlens, const void* k_min, const void* k_max,
                                   void* workspace, size_t workspace_bytes, void* out, float* lse,
                                   void* stream);

/* ---- Self-test of the bounded device waits (no counterpart in the paper) ---------------
 *
 * Launches, on `stream`, one warp that waits on an mbarrier nothing completes, through the
 * same bounded wait the attention and gate kernels use, giving up after `polls` polls
 * (1 <= polls <= 2^20; each poll is one mbarrier.try_wait, which may itself suspend the warp
 * for a short hardware-defined time).  The wait must expire: the kernel then writes
 * MOBA_ERR_DEVICE_TIMEOUT (5) to *status_dev (a caller-owned device int, which should hold 0
 * before the call) and returns; a wait that wrongly succeeds writes -1.  Nothing faults,
 * traps or hangs, and the context stays usable.  Returns MOBA_ERR_INVALID_ARG for a NULL
 * status word or polls out of range, MOBA_ERR_CUDA on a launch error, else MOBA_OK; the
 * result is in *status_dev once the stream has reached the kernel's end. */
moba_status moba_selftest_timeout(int* status_dev, unsigned polls, void* stream);

/* ---- Allocation-free forward (no counterpart in the paper) -----------------------------
 *
 * Some callers cannot allocate device memory or hand over a workspace: plugin hosts that own
 * every device allocation, or services that forbid allocation once they are running.  For
 * them moba_attn_fwd_noalloc computes exactly what moba_attn_fwd computes with
 * sel_in = sel_out = NULL and info = NULL, and allocates nothing (no cudaMalloc, cudaFree or
 * allocating library call).  Its scratch is one array of MOBA_NOALLOC_SCRATCH_BYTES in
 * static device memory inside the library, held on every GPU that loads the library until
 * the process exits.
 *   - p->wave_tokens is ignored: the call picks the largest query wave (a multiple of 128
 *     tokens) whose workspace fits the array.  A problem that does not fit even with
 *     128-token waves returns MOBA_ERR_UNSUPPORTED before any launch; moba_last_error() gives
 *     the bytes it would need.  Other arguments are checked as in moba_attn_fwd.
 *   - The caller still owns and passes q, k, v, cu_seqlens, out and lse (same layouts).
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current and keeps it for the life of the
 *     process; make that first call before any stream capture.  cudaDeviceReset (or anything
 *     else that destroys the device's primary context) invalidates the kept address: do not
 *     call this entry point on that device afterwards.
 *   - All calls on a device share the array and it keeps the previous call's contents; the
 *     forward re-initialises everything it reads.  Calls whose GPU work overlaps (other
 *     streams or host threads on the same device) race on the array and must be serialised
 *     by the caller.
 *   - A bounded device-side wait that gives up records MOBA_ERR_DEVICE_TIMEOUT in the array;
 *     read it with moba_device_status_noalloc. */
#define MOBA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
moba_status moba_attn_fwd_noalloc(const moba_params* p, const void* q, const void* k,
                                  const void* v, const int* cu_seqlens, void* out, float* lse,
                                  void* stream);

/* The device status word of the most recent moba_attn_fwd_noalloc on the current device:
 * MOBA_OK, or MOBA_ERR_DEVICE_TIMEOUT when one of its bounded device-side waits gave up.
 * Waits for `stream` (enqueue it on the stream the forward ran on).  Returns MOBA_OK without
 * touching the device when no allocation-free forward has run on the current device in this
 * process, and MOBA_ERR_CUDA when the device cannot be queried or read.  Allocates nothing. */
moba_status moba_device_status_noalloc(void* stream);

/* Static description of a status code. */
const char* moba_status_string(moba_status s);

/* Description of the last failure on the calling host thread ("" if none). */
const char* moba_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MOBA_H_ */
