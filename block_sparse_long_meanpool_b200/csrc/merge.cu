// Last step of the forward: merge of the per-block partial results of every query row.
//
// The analysis page of the MoBA paper (§3.2): the history blocks and the current block are
// attended separately, and their partial softmax results are combined losslessly with the
// online-softmax rule.  For partials (o_i, lse_i), i = 0 .. n-1 (slot 0 = own block):
//   m = max_i lse_i,  w_i = exp(lse_i - m),  o = sum_i w_i o_i / sum_i w_i,
//   lse = m + log(sum_i w_i).
// One warp per query row: lane s reads slot s's lse, the maximum and the weights come from
// warp reductions, then each lane accumulates d/32 consecutive channels with several partial
// rows in flight (streaming loads).  The output is rounded once to bf16 (nearest even).
// HBM-bound.
#include "moba_internal.cuh"

namespace moba {

namespace {

constexpr int kWarps = 8;

template <int D>
__global__ void __launch_bounds__(kWarps * 32)
merge_kernel(const int* __restrict__ cu, const int* __restrict__ sel, Problem P, Workspace ws,
             int t0, int t1, __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
    constexpr int V = D / 32;
    constexpr int kUnroll = 4;  // partial rows in flight per warp
    const unsigned full = 0xffffffffu;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long n = (long long)(t1 - t0) * P.hq;
    for (long long r = (long long)blockIdx.x * kWarps + warp; r < n;
         r += (long long)gridDim.x * kWarps) {
        const int t = t0 + (int)(r / P.hq);
        const int h = (int)(r % P.hq);
        const int ns = ws.nslots[r];  // own block + routed history blocks (routing pass)
        const size_t pbase = (size_t)r * P.topk;
        // lane s holds slot s: max and weights by warp reductions
        const float lv = (lane < ns) ? __ldcs(ws.part_lse + pbase + lane) : -INFINITY;
        float mx = lv;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(full, mx, off));
        const float wv = (lane < ns) ? expf(lv - mx) : 0.f;
        float L = wv;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(full, L, off);
        float acc[V];
#pragma unroll
        for (int u = 0; u < V; ++u) acc[u] = 0.f;
        const float* base = ws.part_o + pbase * D + lane * V;
        for (int s0 = 0; s0 < ns; s0 += kUnroll) {
            float x[kUnroll][V];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                if (s0 + u < ns) {
                    if constexpr (V == 4) {
                        const float4 y = __ldcs(reinterpret_cast<const float4*>(base + (size_t)(s0 + u) * D));
                        x[u][0] = y.x; x[u][1] = y.y; x[u][2] = y.z; x[u][3] = y.w;
                    } else {
                        const float2 y = __ldcs(reinterpret_cast<const float2*>(base + (size_t)(s0 + u) * D));
                        x[u][0] = y.x; x[u][1] = y.y;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < V; ++e) x[u][e] = 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const float w = __shfl_sync(full, wv, (s0 + u) & 31);
#pragma unroll
                for (int e = 0; e < V; ++e) acc[e] = fmaf(w, x[u][e], acc[e]);
            }
        }
        const float inv = 1.f / L;
        __nv_bfloat16* dst = out + ((size_t)t * P.hq + h) * D + lane * V;
        if constexpr (V == 4) {
            __nv_bfloat162 a = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
            __nv_bfloat162 b = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
            uint2 pk;
            pk.x = *reinterpret_cast<uint32_t*>(&a);
            pk.y = *reinterpret_cast<uint32_t*>(&b);
            *reinterpret_cast<uint2*>(dst) = pk;
        } else {
            *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
        }
        if (lane == 0) lse[(size_t)h * P.T + t] = mx + logf(L);
    }
}

}  // namespace

cudaError_t launch_merge(const Problem& P, const int* cu_seqlens, const int* sel,
                         const Workspace& ws, int t0, int t1, __nv_bfloat16* out, float* lse,
                         cudaStream_t st) {
    const long long n = (long long)(t1 - t0) * P.hq;
    long long grid = (n + kWarps - 1) / kWarps;
    if (grid > 148 * 64) grid = 148 * 64;
    if (grid < 1) grid = 1;
    if (P.d == 64)
        merge_kernel<64><<<(int)grid, kWarps * 32, 0, st>>>(cu_seqlens, sel, P, ws, t0, t1, out, lse);
    else
        merge_kernel<128><<<(int)grid, kWarps * 32, 0, st>>>(cu_seqlens, sel, P, ws, t0, t1, out, lse);
    return cudaGetLastError();
}

}  // namespace moba
