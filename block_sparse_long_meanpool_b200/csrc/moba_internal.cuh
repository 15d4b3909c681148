// Internal declarations shared by the MoBA CUDA sources (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace moba {

// Rows of a query tile (one tensor-core M tile); an attention work item holds up to two.
constexpr int kTileM = 128;
constexpr int kItemRows = 2 * kTileM;

// Device-side header at the start of the workspace.
struct WsHeader {
    int nb_total;           // number of blocks (sum over sequences of ceil(L / B))
    int status;             // 0 or a moba_status code written by a kernel
    unsigned work_counter;  // persistent-kernel work cursor (zeroed per wave)
    int n_items;            // work items of the current wave
    int n_past_items;       // of which routed history tiles (the rest are current-block tiles)
    int pad[11];
};

// One unit of attention work: up to two 128-row query tiles against one KV range of one KV
// head, so that every K/V chunk loaded serves both tiles.
//   kind 0 (history): a = list id (g * nb_cap + block), b = first entry, c = rows (<= 256;
//          rows 0-127 form tile 0, rows 128-255 tile 1)
//   kind 1 (current block, one head):  a = block, b = query head h, c = query tile index
//   kind 2 (current block, two heads): as kind 1 for heads h and h + 1 (same KV head)
//   kind 3 (current block, two query tiles of one head): a = block, b = head h, c = tile p;
//          the other tile is lv - 1 - p (lv = query tiles of the block), which comes first
struct WorkItem {
    int a, b, c, kind;
};

// Problem description passed by value to kernels.
struct Problem {
    int batch, T, hq, hkv, d, chunk, topk;
    int group;       // hq / hkv
    int nb_cap;      // capacity of per-block arrays (upper bound of the block count)
    int max_blocks;  // most blocks one sequence may have (from max_seqlen), <= nb_cap
    float scale;     // softmax scale (natural units)
    float scale_log2;  // scale * log2(e)
};

// Views into the workspace of one moba_attn_fwd call.
struct Workspace {
    WsHeader* hdr;
    int* cu_blocks;   // [batch + 1]
    int* blk_start;   // [nb_cap]
    int* blk_len;     // [nb_cap]
    int* blk_seq;     // [nb_cap]
    int* blk_local;   // [nb_cap]
    float* means;     // [nb_cap, hkv, d]
    int* sel;         // [hq, T, topk]
    int* counts;      // [hkv * nb_cap]
    int* offsets;     // [hkv * nb_cap + 1]
    int* cursor;      // [hkv * nb_cap]
    int* item_off;    // [hkv * nb_cap + 1]: index of each list's first history work item
    int* entries;     // [wave * hq * (topk - 1)]
    WorkItem* items;  // [max_items]
    __nv_bfloat16* part_o;  // [wave * hq * topk, d]: normalised partial outputs
    float* part_lse;  // [wave * hq * topk]
    unsigned char* nslots;  // [wave * hq]: 1 + routed history blocks of each row
};

// ---------------------------------------------------------------------------------------
// Device helpers

// Index of the sequence holding token t: the last i with cu[i] <= t (empty sequences skipped).
__device__ __forceinline__ int seq_of_token(const int* __restrict__ cu, int batch, int t) {
    int lo = 0, hi = batch;  // answer in [0, batch)
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (__ldg(cu + mid) <= t) lo = mid; else hi = mid;
    }
    return lo;
}

// Selection rule of the routing pass: entry i of a row is a routed history block iff
// 0 <= j < c, it is not a repeat of an earlier routed entry, and fewer than topk-1 entries
// have been routed before it.  The row (topk <= K entries) is read into registers once.
// Returns the number of routed entries and, for each routed entry, calls f(slot, j) with
// slot = 1 + its rank among the routed entries.
template <int K, typename F>
__device__ __forceinline__ int for_each_routed(const int* __restrict__ row, int topk, int c, F f) {
    int v[K];
#pragma unroll
    for (int i = 0; i < K; ++i) v[i] = (i < topk) ? __ldg(row + i) : -1;
    int n = 0;
#pragma unroll
    for (int i = 0; i < K; ++i) {
        const int j = v[i];
        bool take = j >= 0 && j < c && n < topk - 1;
#pragma unroll
        for (int i2 = 0; i2 < i; ++i2) take = take && v[i2] != j;
        if (take) {
            f(n + 1, j);
            ++n;
        }
    }
    return n;
}

// Top-k lists kept in registers (gate and decode gate).
// Inserts (x, id) into a descending list of K (score, index) pairs when it beats the last
// entry; an equal score never displaces an entry already in the list.  Every position is
// updated independently of the others (x is compared with all entries first, then entry i
// keeps its value, takes x, or takes its left neighbour's old value), so an insertion is one
// level of selects rather than a chain of K dependent compare-and-swaps.
template <int K>
__device__ __forceinline__ void insert_desc(float (&val)[K], int (&idx)[K], float x, int id,
                                            bool ok) {
    if (ok && x > val[K - 1]) {
        bool gt[K];
#pragma unroll
        for (int i = 0; i < K; ++i) gt[i] = x > val[i];
#pragma unroll
        for (int i = K - 1; i > 0; --i) {
            val[i] = gt[i] ? (gt[i - 1] ? val[i - 1] : x) : val[i];
            idx[i] = gt[i] ? (gt[i - 1] ? idx[i - 1] : id) : idx[i];
        }
        val[0] = gt[0] ? x : val[0];
        idx[0] = gt[0] ? id : idx[0];
    }
}

// Inserts (x, id) into a list sorted by (score descending, index ascending) under that same
// order (used to merge two lists); positions are updated independently as above.
template <int K>
__device__ __forceinline__ void insert_ordered(float (&val)[K], int (&idx)[K], float x, int id) {
    bool gt[K];
#pragma unroll
    for (int i = 0; i < K; ++i) gt[i] = x > val[i] || (x == val[i] && id < idx[i]);
    if (gt[K - 1]) {
#pragma unroll
        for (int i = K - 1; i > 0; --i) {
            val[i] = gt[i] ? (gt[i - 1] ? val[i - 1] : x) : val[i];
            idx[i] = gt[i] ? (gt[i - 1] ? idx[i - 1] : id) : idx[i];
        }
        val[0] = gt[0] ? x : val[0];
        idx[0] = gt[0] ? id : idx[0];
    }
}

// ---------------------------------------------------------------------------------------
// Launchers (defined in the .cu files).  Each returns cudaGetLastError() of its launch.

cudaError_t launch_plan_blocks(const Problem& P, const int* cu_seqlens, const Workspace& ws,
                               cudaStream_t st);
cudaError_t launch_meanpool(const Problem& P, const __nv_bfloat16* k, const int* cu_seqlens,
                            float* means, cudaStream_t st);
cudaError_t launch_minmaxpool(const Problem& P, const __nv_bfloat16* k, const int* cu_seqlens,
                              __nv_bfloat16* kmin, __nv_bfloat16* kmax, cudaStream_t st);
cudaError_t launch_gate(const Problem& P, const __nv_bfloat16* q, const float* means,
                        const int* cu_seqlens, int* sel, cudaStream_t st);
struct GateSummary;
// Runs the tensor-core gate (mean or min/max summary) when every sequence fits it, else the
// CUDA-core gate (mean summary only; the min/max summary returns cudaErrorNotSupported); *path
// (when non-null) receives MOBA_GATE_PATH_TENSOR_CORES (1) or MOBA_GATE_PATH_CUDA_CORES (2).
cudaError_t launch_gate_best(const Problem& P, const __nv_bfloat16* q, const GateSummary& s,
                             const int* cu_seqlens, int* sel, int* status, cudaStream_t st,
                             int* path = nullptr);
cudaError_t launch_route_count(const Problem& P, const int* cu_seqlens, const int* sel,
                               const Workspace& ws, int t0, int t1, cudaStream_t st);
cudaError_t launch_route_plan(const Problem& P, const Workspace& ws, int t0, int t1,
                              cudaStream_t st);
cudaError_t launch_route_scatter(const Problem& P, const int* cu_seqlens, const int* sel,
                                 const Workspace& ws, int t0, int t1, cudaStream_t st);
cudaError_t launch_attention(const Problem& P, const __nv_bfloat16* q, const __nv_bfloat16* k,
                             const __nv_bfloat16* v, const Workspace& ws, int t0, int t1,
                             int num_sms, cudaStream_t st);
cudaError_t launch_merge(const Problem& P, const int* cu_seqlens, const int* sel,
                         const Workspace& ws, int t0, int t1, __nv_bfloat16* out, float* lse,
                         cudaStream_t st);

// Buffers of one backward call (moba_attn_bwd).
struct BwdArgs {
    const __nv_bfloat16 *q, *k, *v, *out, *dout;
    const float* lse;   // [hq, T]
    const float* dlse;  // [hq, T] or nullptr
    float2* rs;         // [hq, T]: (lse * log2 e, <dO, out> - dlse)
    float* dq_acc;      // [T, hq, d] fp32 accumulator, zeroed before the dQ kernel
    __nv_bfloat16 *dq, *dk, *dv;
};
// Row statistics, dK/dV, dQ and the dq conversion, after the routing pass over all rows
// (one wave from token 0).  *launches is incremented per kernel queued.
cudaError_t launch_backward(const Problem& P, const BwdArgs& a, const Workspace& ws, int num_sms,
                            cudaStream_t st, int* launches);

// Views into the workspace of one decode step (P.batch sequences, one query row each).
struct DecodeWorkspace {
    int* sel;         // [batch * hq, topk]: own block, routed blocks best-first, then -1
    int* nsl;         // [batch * hq]: 1 + routed blocks (0 for an empty sequence)
    float* part_o;    // [batch * hq * topk * splits, d]: normalised partial outputs
    float* part_lse;  // [batch * hq * topk * splits]
    int splits;       // key ranges per selected block (a power of two, topk * splits <= 64)
};
// Key ranges per selected block for a decode step: enough (row, block, range) tasks to fill
// the GPU, while every row's partials still fit one warp's merge (topk * splits <= 64, two per
// lane) and a range keeps at least 128 keys.  A function of the parameters only.
inline int decode_splits(int batch, int hq, int topk, int chunk) {
    int s = 1;
    while ((long long)batch * hq * topk * s < 1184 && topk * s * 2 <= 64 && chunk / (s * 2) >= 128) s *= 2;
    return s;
}
// Block summary a gate scores against: the fp32 means (kmin == kmax == nullptr) or the bf16
// min/max pair (means == nullptr), each [NB, Hkv, d].
struct GateSummary {
    const float* means;
    const __nv_bfloat16* kmin;
    const __nv_bfloat16* kmax;
};
using DecodeGate = GateSummary;
cudaError_t launch_decode(const Problem& P, const __nv_bfloat16* q, const __nv_bfloat16* k,
                          const __nv_bfloat16* v, const int* cu_seqlens, const DecodeGate& gate,
                          const DecodeWorkspace& ws, __nv_bfloat16* out, float* lse,
                          cudaStream_t st);

}  // namespace moba

namespace moba {

// Locates global block b without a precomputed block table: a warp scans the per-sequence
// block counts ceil(L_i / chunk) over cu_seqlens.  Must be called by all 32 lanes of a warp;
// every lane gets the same answer.  Returns false when b is past the last block.
struct BlockRef {
    int seq, local, start, len, first;  // first = global index of the sequence's block 0
};

__device__ __forceinline__ bool find_block(const int* __restrict__ cu, int batch, int chunk,
                                           int b, BlockRef& r) {
    const unsigned full = 0xffffffffu;
    const int lane = threadIdx.x & 31;
    int base = 0;
    for (int i0 = 0; i0 < batch; i0 += 32) {
        const int i = i0 + lane;
        int s = 0, e = 0, n = 0;
        if (i < batch) {
            s = __ldg(cu + i);
            e = __ldg(cu + i + 1);
            n = (e - s + chunk - 1) / chunk;
        }
        int incl = n;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            int y = __shfl_up_sync(full, incl, off);
            if (lane >= off) incl += y;
        }
        const int excl = incl - n;
        const bool hit = (i < batch) && (b >= base + excl) && (b < base + incl);
        const unsigned m = __ballot_sync(full, hit);
        if (m) {
            const int src = __ffs(m) - 1;
            r.seq = __shfl_sync(full, i, src);
            r.first = base + __shfl_sync(full, excl, src);
            r.local = b - r.first;
            r.start = __shfl_sync(full, s, src) + r.local * chunk;
            const int e_src = __shfl_sync(full, e, src);
            r.len = min(chunk, e_src - r.start);
            return true;
        }
        base += __shfl_sync(full, incl, 31);
    }
    return false;
}

}  // namespace moba
