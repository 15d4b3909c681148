// Min/max block summary of the keys, the Quest-style alternative to the mean-pooled gate.
//
// The analysis page of the MoBA paper names Quest as the MoBA variant that pools each block
// by its minimum and maximum instead of its mean (§1.3) and calls that summary the stronger
// one (§5.1 item 6, §6.3).  Quest's summary is the element-wise minimum and maximum of the
// block's keys; the decode gate then scores a block by the largest q . x over the box
// kmin <= x <= kmax.  The minimum or maximum of bf16 values is itself a bf16 value, so the
// summaries are stored as bf16 [NB, Hkv, d] with no rounding.
//
// Layout and schedule follow the mean-pool stream: K is [T, Hkv, d] bf16, the rows of one
// block are one contiguous [len, Hkv*d] slab; one CTA owns one block and a 256-column slice,
// each warp reads whole 512-byte row slices (16 bytes per lane), the 8 warps take every 8th
// row, and the per-warp extrema are combined through shared memory.  A pure HBM stream.
#include "moba_internal.cuh"

namespace moba {

namespace {

constexpr int kThreads = 256;
constexpr int kCols = 256;  // columns (bf16) per CTA: 32 lanes x 8
constexpr int kUnroll = 4;  // independent 16-byte loads in flight per thread

__device__ __forceinline__ void minmax_bf16x8(float (&lo)[8], float (&hi)[8], const uint4& x) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float a = __uint_as_float(w[i] << 16), b = __uint_as_float(w[i] & 0xffff0000u);
        lo[2 * i] = fminf(lo[2 * i], a);
        hi[2 * i] = fmaxf(hi[2 * i], a);
        lo[2 * i + 1] = fminf(lo[2 * i + 1], b);
        hi[2 * i + 1] = fmaxf(hi[2 * i + 1], b);
    }
}

__global__ void __launch_bounds__(kThreads)
minmaxpool_kernel(const __nv_bfloat16* __restrict__ k, const int* __restrict__ cu, Problem P,
                  __nv_bfloat16* __restrict__ kmin, __nv_bfloat16* __restrict__ kmax) {
    __shared__ float red_lo[kThreads / 32][kCols];
    __shared__ float red_hi[kThreads / 32][kCols];
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
    float lo[8], hi[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        lo[i] = INFINITY;
        hi[i] = -INFINITY;
    }
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
            for (int u = 0; u < kUnroll; ++u) minmax_bf16x8(lo, hi, x[u]);
        }
        for (; r < len; r += step)
            minmax_bf16x8(lo, hi, __ldcs(reinterpret_cast<const uint4*>(base + (size_t)r * C)));
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        red_lo[warp][lane * 8 + i] = lo[i];
        red_hi[warp][lane * 8 + i] = hi[i];
    }
    __syncthreads();
    const int c2 = blockIdx.y * kCols + threadIdx.x;
    if (threadIdx.x < kCols && c2 < C) {
        float l = INFINITY, h = -INFINITY;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) {
            l = fminf(l, red_lo[w][threadIdx.x]);
            h = fmaxf(h, red_hi[w][threadIdx.x]);
        }
        // every block holds at least one row, so l and h are key values (exact in bf16)
        kmin[(size_t)b * C + c2] = __float2bfloat16_rn(l);
        kmax[(size_t)b * C + c2] = __float2bfloat16_rn(h);
    }
}

}  // namespace

cudaError_t launch_minmaxpool(const Problem& P, const __nv_bfloat16* k, const int* cu_seqlens,
                              __nv_bfloat16* kmin, __nv_bfloat16* kmax, cudaStream_t st) {
    const int C = P.hkv * P.d;
    if (P.nb_cap == 0) return cudaSuccess;
    dim3 grid(P.nb_cap, (C + kCols - 1) / kCols);
    minmaxpool_kernel<<<grid, kThreads, 0, st>>>(k, cu_seqlens, P, kmin, kmax);
    return cudaGetLastError();
}

}  // namespace moba
