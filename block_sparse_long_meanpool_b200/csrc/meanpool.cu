// Step 2 of the forward: mean-pooled key of every (block, KV head).
//
// The analysis page of the MoBA paper (§2.2) summarises block i by meanpool(K[I_i]).  K is
// [T, Hkv, d] bf16, so the rows of one block form one contiguous [len, Hkv*d] slab.  One CTA
// owns one block and a 256-column slice of that slab: each warp reads whole 512-byte row
// slices (16 bytes per lane, fully coalesced), the 8 warps take every 8th row, and the
// per-warp fp32 partial sums are added in a fixed order at the end.  The kernel is a pure
// stream over K (HBM-bound); there is no scratch memory and no atomics, so results are
// deterministic.
#include "moba_internal.cuh"

namespace moba {

namespace {

constexpr int kThreads = 256;
constexpr int kCols = 256;     // columns (bf16) per CTA: 32 lanes x 8
constexpr int kUnroll = 4;     // independent 16-byte loads in flight per thread

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4& x) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] += __uint_as_float(w[i] << 16);
        acc[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
    }
}

__global__ void __launch_bounds__(kThreads)
meanpool_kernel(const __nv_bfloat16* __restrict__ k, const int* __restrict__ cu, Problem P,
                float* __restrict__ means) {
    __shared__ float red[kThreads / 32][kCols];
    __shared__ int s_ok, s_start, s_len;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x;
    if (warp == 0) {
        BlockRef r;
        const bool ok = find_block(cu, P.batch, P.chunk, b, r);
        if (lane == 0) {
            s_ok = ok;
            s_start = ok ? r.start : 0;
            s_len = ok ? r.len : 0;
        }
    }
    __syncthreads();
    if (!s_ok) return;
    const int C = P.hkv * P.d;
    const int start = s_start, len = s_len;
    const int col = blockIdx.y * kCols + lane * 8;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    if (col < C) {
        const __nv_bfloat16* base = k + (size_t)start * C + col;
        int r = warp;
        constexpr int step = kThreads / 32;
        for (; r + step * (kUnroll - 1) < len; r += step * kUnroll) {
            uint4 x[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u)
                x[u] = __ldcs(reinterpret_cast<const uint4*>(base + (size_t)(r + step * u) * C));
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) add_bf16x8(acc, x[u]);
        }
        for (; r < len; r += step)
            add_bf16x8(acc, __ldcs(reinterpret_cast<const uint4*>(base + (size_t)r * C)));
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) red[warp][lane * 8 + i] = acc[i];
    __syncthreads();
    const int c2 = blockIdx.y * kCols + threadIdx.x;
    if (threadIdx.x < kCols && c2 < C) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) s += red[w][threadIdx.x];
        means[(size_t)b * C + c2] = s / (float)len;
    }
}

}  // namespace

cudaError_t launch_meanpool(const Problem& P, const __nv_bfloat16* k, const int* cu_seqlens,
                            float* means, cudaStream_t st) {
    const int C = P.hkv * P.d;
    dim3 grid(P.nb_cap, (C + kCols - 1) / kCols);
    if (P.nb_cap == 0) return cudaSuccess;
    meanpool_kernel<<<grid, kThreads, 0, st>>>(k, cu_seqlens, P, means);
    return cudaGetLastError();
}

}  // namespace moba
