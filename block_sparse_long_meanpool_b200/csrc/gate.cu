// Steps 3-4 of the forward: gate scores, future-block mask, forced own block, hard top-k.
//
// The analysis page of the MoBA paper (§2.2-§2.3): s_j = <q, mean_j>; a block that ends after
// the query is masked to -inf; the query's own block c is always taken; the best topk-1 of
// the remaining (past) blocks are routed.  Only blocks j < c can compete, so only those scores
// are formed.
//
// One CTA owns a 128-row tile of one query block for one query head; all its rows share c and
// the sequence, so the loop over past blocks is uniform.  Each thread owns one query row in
// fp32 registers and keeps a sorted top-(topk-1) list in registers; the block means of the
// row's KV head are staged through shared memory 32 at a time and read as broadcasts.
// Arithmetic is fp32 (means are fp32, q is exact in fp32), which keeps score errors near 1e-6
// and far inside the 1e-3 relative near-tie band.  Ties keep the lower block index.
#include <climits>

#include "moba_internal.cuh"

namespace moba {

namespace {

constexpr int kRows = 128;
constexpr int kStage = 32;  // block means per shared-memory stage

template <int D, int KMAX>
__global__ void __launch_bounds__(kRows)
gate_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ means,
            const int* __restrict__ cu, Problem P, int tiles_per_block, int* __restrict__ sel) {
    __shared__ __align__(16) float sm[kStage][D];
    __shared__ int s_ok, s_start, s_len, s_local, s_first;
    const int tid = threadIdx.x;
    const int b = blockIdx.x / tiles_per_block;
    const int tile = blockIdx.x % tiles_per_block;
    const int h = blockIdx.y;
    if (tid < 32) {
        BlockRef r;
        const bool ok = find_block(cu, P.batch, P.chunk, b, r);
        if (tid == 0) {
            s_ok = ok && tile * kRows < r.len;
            s_start = r.start;
            s_len = r.len;
            s_local = r.local;
            s_first = r.first;
        }
    }
    __syncthreads();
    if (!s_ok) return;
    const int row = tile * kRows + tid;
    const bool valid = row < s_len;
    const int t = s_start + row;
    const int c = s_local;
    const int n_route = min(P.topk - 1, c);
    const int g = h / P.group;

    float val[KMAX];
    int idx[KMAX];
#pragma unroll
    for (int i = 0; i < KMAX; ++i) {
        val[i] = -INFINITY;
        idx[i] = INT_MAX;
    }

    if (n_route > 0) {
        float qr[D];
        if (valid) {
            const uint4* qp = reinterpret_cast<const uint4*>(q + ((size_t)t * P.hq + h) * D);
#pragma unroll
            for (int i = 0; i < D / 8; ++i) {
                const uint4 x = __ldg(qp + i);
                const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    qr[8 * i + 2 * u] = __uint_as_float(w[u] << 16);
                    qr[8 * i + 2 * u + 1] = __uint_as_float(w[u] & 0xffff0000u);
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < D; ++i) qr[i] = 0.f;
        }
        const float* mbase = means + ((size_t)s_first * P.hkv + g) * D;
        const size_t mstride = (size_t)P.hkv * D;
        for (int j0 = 0; j0 < c; j0 += kStage) {
            const int nj = min(kStage, c - j0);
            __syncthreads();
            for (int e = tid * 4; e < nj * D; e += kRows * 4) {
                const int jj = e / D, col = e % D;
                *reinterpret_cast<float4*>(&sm[jj][col]) =
                    __ldg(reinterpret_cast<const float4*>(mbase + (size_t)(j0 + jj) * mstride + col));
            }
            __syncthreads();
            if (valid) {
                for (int jj = 0; jj < nj; ++jj) {
                    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
                    for (int i = 0; i < D; i += 4) {
                        const float4 m = *reinterpret_cast<const float4*>(&sm[jj][i]);
                        a0 = fmaf(qr[i], m.x, a0);
                        a1 = fmaf(qr[i + 1], m.y, a1);
                        a2 = fmaf(qr[i + 2], m.z, a2);
                        a3 = fmaf(qr[i + 3], m.w, a3);
                    }
                    float v = (a0 + a1) + (a2 + a3);
                    int id = j0 + jj;
                    if (v > val[KMAX - 1]) {
                        // insertion into the descending list; an equal score never displaces
                        // an earlier (lower-index) block
#pragma unroll
                        for (int i = 0; i < KMAX; ++i) {
                            if (v > val[i]) {
                                const float tv = val[i];
                                const int ti = idx[i];
                                val[i] = v;
                                idx[i] = id;
                                v = tv;
                                id = ti;
                            }
                        }
                    }
                }
            }
        }
    }
    if (!valid) return;
    // routed blocks in ascending order, then the own block, then -1 padding
    int o[KMAX];
#pragma unroll
    for (int i = 0; i < KMAX; ++i) o[i] = (i < n_route) ? idx[i] : INT_MAX;
#pragma unroll
    for (int p = 0; p < KMAX; ++p) {
#pragma unroll
        for (int i = (p & 1); i + 1 < KMAX; i += 2) {
            const int lo = min(o[i], o[i + 1]), hi = max(o[i], o[i + 1]);
            o[i] = lo;
            o[i + 1] = hi;
        }
    }
    int* dst = sel + ((size_t)h * P.T + t) * P.topk;
#pragma unroll
    for (int i = 0; i <= KMAX; ++i) {
        if (i < P.topk) {
            const int vo = (i < n_route) ? o[i < KMAX ? i : KMAX - 1] : (i == n_route ? c : -1);
            dst[i] = vo;
        }
    }
    for (int i = KMAX + 1; i < P.topk; ++i) dst[i] = -1;
}

template <int D>
cudaError_t launch_gate_d(const Problem& P, const __nv_bfloat16* q, const float* means,
                          const int* cu, int* sel, cudaStream_t st) {
    const int tpb = (P.chunk + kRows - 1) / kRows;
    dim3 grid(P.nb_cap * tpb, P.hq);
    const int need = P.topk - 1;
    if (need <= 2)
        gate_kernel<D, 2><<<grid, kRows, 0, st>>>(q, means, cu, P, tpb, sel);
    else if (need <= 4)
        gate_kernel<D, 4><<<grid, kRows, 0, st>>>(q, means, cu, P, tpb, sel);
    else if (need <= 8)
        gate_kernel<D, 8><<<grid, kRows, 0, st>>>(q, means, cu, P, tpb, sel);
    else if (need <= 16)
        gate_kernel<D, 16><<<grid, kRows, 0, st>>>(q, means, cu, P, tpb, sel);
    else
        gate_kernel<D, 32><<<grid, kRows, 0, st>>>(q, means, cu, P, tpb, sel);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gate(const Problem& P, const __nv_bfloat16* q, const float* means,
                        const int* cu_seqlens, int* sel, cudaStream_t st) {
    if (P.nb_cap == 0) return cudaSuccess;
    if (P.d == 64) return launch_gate_d<64>(P, q, means, cu_seqlens, sel, st);
    return launch_gate_d<128>(P, q, means, cu_seqlens, sel, st);
}

}  // namespace moba
