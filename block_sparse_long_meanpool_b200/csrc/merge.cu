// Last step of the forward: merge of the per-block partial results of every query row.
//
// The analysis page of the MoBA paper (§3.2): the history blocks and the current block are
// attended separately, and their partial softmax results are combined losslessly with the
// online-softmax rule.  For partials (o_i, lse_i), i = 0 .. n-1 (slot 0 = own block):
//   m = max_i lse_i,  w_i = exp(lse_i - m),  o = sum_i w_i o_i / sum_i w_i,
//   lse = m + log(sum_i w_i).
// The partial outputs o_i are bf16 (the precision an attention call returns its output in),
// the lse_i fp32; the combination is computed in fp32.
// A half-warp per query row (two rows per warp), the row's slot count loaded while the previous
// row is merged: the first partial rows are loaded before the weights are known, lane s reads
// slot s's lse (and s + 16), the maximum and the weights come from half-warp reductions, and
// each lane accumulates d/16 consecutive channels with four partial rows in flight (streaming
// loads).  The output is rounded once to bf16 (nearest even).  HBM-bound.
#include "moba_internal.cuh"

namespace moba {

namespace {

constexpr int kWarps = 8;

// V consecutive bf16 channels of one partial row (streaming load), widened to fp32; zeros
// when the slot is unused.
template <int V>
__device__ __forceinline__ void load_row(const __nv_bfloat16* p, bool valid, float (&x)[V]) {
    uint32_t w[V / 2];
    if constexpr (V == 8) {
        uint4 y = make_uint4(0u, 0u, 0u, 0u);
        if (valid) y = __ldcs(reinterpret_cast<const uint4*>(p));
        w[0] = y.x; w[1] = y.y; w[2] = y.z; w[3] = y.w;
    } else {
        uint2 y = make_uint2(0u, 0u);
        if (valid) y = __ldcs(reinterpret_cast<const uint2*>(p));
        w[0] = y.x; w[1] = y.y;
    }
#pragma unroll
    for (int e = 0; e < V / 2; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
        x[2 * e] = f.x;
        x[2 * e + 1] = f.y;
    }
}

template <int D>
__global__ void __launch_bounds__(kWarps * 32)
merge_kernel(const int* __restrict__ cu, const int* __restrict__ sel, Problem P, Workspace ws,
             int t0, int t1, __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
    constexpr int V = D / 16;   // channels per lane: a half-warp (16 lanes) owns one row
    constexpr int kUnroll = 4;  // partial rows in flight per half-warp
    const unsigned full = 0xffffffffu;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hl = lane & 15, half = lane >> 4;
    const long long n = (long long)(t1 - t0) * P.hq;
    const long long stride = (long long)gridDim.x * kWarps * 2;
    long long base = ((long long)blockIdx.x * kWarps + warp) * 2;
    // slot count (own block + routed history blocks) of this half-warp's next row, loaded one
    // row ahead so that the partial rows' loads do not wait for it
    int ns_next = (base + half < n) ? (int)ws.nslots[base + half] : 0;
    for (; base < n; base += stride) {
        const long long r = base + half;
        const bool valid = r < n;
        const int ns = ns_next;
        ns_next = (r + stride < n) ? (int)ws.nslots[r + stride] : 0;
        const size_t pbase = (size_t)(valid ? r : 0) * P.topk;
        const __nv_bfloat16* obase = ws.part_o + pbase * D + hl * V;
        // first partial rows in flight before the weights are known
        float x[kUnroll][V];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) load_row<V>(obase + (size_t)u * D, u < ns, x[u]);
        // slot lse: lane hl holds slots hl and hl + 16; max and weights by half-warp reductions
        const float la = (hl < ns) ? __ldcs(ws.part_lse + pbase + hl) : -INFINITY;
        const float lb = (hl + 16 < ns) ? __ldcs(ws.part_lse + pbase + hl + 16) : -INFINITY;
        float mx = fmaxf(la, lb);
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(full, mx, off));
        const float wa = (hl < ns) ? expf(la - mx) : 0.f;
        const float wb = (hl + 16 < ns) ? expf(lb - mx) : 0.f;
        float L = wa + wb;
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) L += __shfl_xor_sync(full, L, off);
        float acc[V];
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = 0.f;
        const int src0 = half * 16;
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const float w = __shfl_sync(full, wa, src0 + u);
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] = fmaf(w, x[u][e], acc[e]);
        }
        const int ns_max = max(__shfl_sync(full, ns, 0), __shfl_sync(full, ns, 16));
        for (int s0 = kUnroll; s0 < ns_max; s0 += kUnroll) {
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) load_row<V>(obase + (size_t)(s0 + u) * D, s0 + u < ns, x[u]);
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int sl = s0 + u;  // < 32
                const float w = (sl < 16) ? __shfl_sync(full, wa, src0 + (sl & 15))
                                          : __shfl_sync(full, wb, src0 + (sl & 15));
#pragma unroll
                for (int e = 0; e < V; ++e) acc[e] = fmaf(w, x[u][e], acc[e]);
            }
        }
        if (!valid) continue;
        const int t = t0 + (int)(r / P.hq);
        const int h = (int)(r % P.hq);
        const float inv = 1.f / L;
        __nv_bfloat16* dst = out + ((size_t)t * P.hq + h) * D + hl * V;
        uint32_t pk[V / 2];
#pragma unroll
        for (int e = 0; e < V; e += 2) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[e] * inv, acc[e + 1] * inv);
            pk[e / 2] = *reinterpret_cast<uint32_t*>(&b2);
        }
        if constexpr (V == 8)
            *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        else
            *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
        if (hl == 0) lse[(size_t)h * P.T + t] = mx + logf(L);
    }
}

}  // namespace

cudaError_t launch_merge(const Problem& P, const int* cu_seqlens, const int* sel,
                         const Workspace& ws, int t0, int t1, __nv_bfloat16* out, float* lse,
                         cudaStream_t st) {
    const long long n = (long long)(t1 - t0) * P.hq;
    long long grid = (n + 2 * kWarps - 1) / (2 * kWarps);
    if (grid > 148 * 64) grid = 148 * 64;
    if (grid < 1) grid = 1;
    if (P.d == 64)
        merge_kernel<64><<<(int)grid, kWarps * 32, 0, st>>>(cu_seqlens, sel, P, ws, t0, t1, out, lse);
    else
        merge_kernel<128><<<(int)grid, kWarps * 32, 0, st>>>(cu_seqlens, sel, P, ws, t0, t1, out, lse);
    return cudaGetLastError();
}

}  // namespace moba
