// Steps 3-4 of the forward on the tensor cores: gate scores of 128-row query tiles against the
// block means by tcgen05 MMA, then the future-block mask, the forced own block and the hard
// top-k in registers.
//
// The analysis page of the MoBA paper (§2.2-§2.3): s_j = <q, mean_j>; blocks after the row's
// own block c are masked to -inf, block c is always taken, the best topk-1 past blocks
// (j < c) are routed.  Ties keep the lower block index.
//
// Precision: each fp32 mean is split exactly into three bf16 parts, m = hi + mid + lo
// (|m - hi - mid - lo| <= 2^-24 |m|), and the three products with the bf16 query row are
// accumulated in fp32 by three MMAs into the same TMEM accumulator.  The score is therefore
// the fp32-accurate dot product (about 1e-6 absolute here), far inside the 1e-3 relative
// near-tie band, unlike a single bf16 rounding of the means (about 2e-3 relative).
//
// One CTA per (query block b, KV head g): it stages the split means of the c past blocks of
// b's sequence in shared memory once (SWIZZLE_128B, K-major), then runs the 128-row tiles of
// block b for the query heads of g.  Warp 4 loads each Q tile by TMA and issues the MMAs
// (N = c rounded up to 16) into one of two TMEM accumulators; warps 0-3 (one thread per row)
// read the scores with tcgen05.ld and keep a sorted top-(topk-1) list in registers.  Rows
// with fewer than topk-1 past blocks take all of them.  Sequences longer than 256 blocks use
// the fp32 CUDA-core gate instead (gate.cu).
#include <climits>

#include "moba_internal.cuh"
#include "ptx.cuh"

namespace moba {

namespace {

using namespace ptx;

constexpr int kMaxPast = 256;   // past blocks scored in one MMA (N <= 256)
constexpr int kThreads = 160;   // warps 0-3 top-k, warp 4 TMA + MMA
constexpr int kWarpMMA = 4;

template <int D>
struct GateSmem {
    static constexpr int kQ = 0;                         // Q tile [128 x D] bf16, swizzled
    static constexpr int kMeans = kTileM * D * 2;        // 3 splits x [N x D] bf16
    static constexpr int kBars(int n) { return kMeans + 3 * n * D * 2; }
    static constexpr int kBytes(int n) { return kBars(n) + 8 * 8 + 16 + 1024; }
};

template <int D, int KMAX>
__global__ void __launch_bounds__(kThreads, 1)
gate_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const float* __restrict__ means,
               const int* __restrict__ cu, Problem P, int* __restrict__ sel, int* status,
               int n_cap) {
    using L = GateSmem<D>;
    constexpr int kHalfBytesQ = kTileM * 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    __shared__ int s_ok, s_start, s_len, s_local, s_first;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x, g = blockIdx.y;
    if (warp == 0) {
        BlockRef r;
        const bool ok = find_block(cu, P.batch, P.chunk, b, r);
        if (lane == 0) {
            s_ok = ok;
            s_start = r.start;
            s_len = r.len;
            s_local = r.local;
            s_first = r.first;
            s_abort = 0;
        }
    }
    __syncthreads();
    if (!s_ok) return;
    const int c = s_local, start = s_start, len = s_len;
    const int n_route = min(P.topk - 1, c);
    const int qtiles = (len + kTileM - 1) / kTileM;
    const int ntiles = qtiles * P.group;

    if (n_route == 0 || c > n_cap) {
        // nothing to score: every row takes its own block only.  c > n_cap means the sequence
        // is longer than the caller's max_seqlen promised: its rows keep the own block only
        // and the call's status word (when there is one) records the broken promise.
        if (c > n_cap && threadIdx.x == 0 && status) atomicExch(status, 1 /* INVALID_ARG */);
        for (int e = threadIdx.x; e < len * P.group; e += kThreads) {
            const int h = g * P.group + e / len;
            const int t = start + e % len;
            int* dst = sel + ((size_t)h * P.T + t) * P.topk;
            for (int i = 0; i < P.topk; ++i) dst[i] = (i == 0) ? c : -1;
        }
        return;
    }
    const int N = (c + 15) & ~15;  // MMA N: past blocks rounded up to 16 (c <= kMaxPast)
    const int split_bytes = N * D * 2;
    const uint32_t sm_base = smem_u32(smem);
    const uint32_t m_base = sm_base + L::kMeans;
    const uint32_t bar0 = sm_base + L::kBars(N);
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    const int B_QFULL = 0, B_QEMPTY = 1, B_SFULL = 2, B_SEMPTY = 4, B_FINAL = 6;

    // stage the split means of past blocks 0..c-1 (rows c..N-1 are zero)
    {
        const float* mg = means + ((size_t)s_first * P.hkv + g) * D;
        const size_t mstride = (size_t)P.hkv * D;
        for (int e = threadIdx.x; e < N * (D / 4); e += kThreads) {
            const int j = e / (D / 4), d0 = (e % (D / 4)) * 4;
            float4 m4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (j < c) m4 = __ldg(reinterpret_cast<const float4*>(mg + (size_t)j * mstride + d0));
            const float mv[4] = {m4.x, m4.y, m4.z, m4.w};
            uint32_t part[3][2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                float r0 = mv[2 * u], r1 = mv[2 * u + 1];
                __nv_bfloat16 h0[3], h1[3];
#pragma unroll
                for (int k = 0; k < 3; ++k) {
                    h0[k] = __float2bfloat16_rn(r0);
                    h1[k] = __float2bfloat16_rn(r1);
                    r0 -= __bfloat162float(h0[k]);
                    r1 -= __bfloat162float(h1[k]);
                    __nv_bfloat162 pr;
                    pr.x = h0[k];
                    pr.y = h1[k];
                    part[k][u] = *reinterpret_cast<uint32_t*>(&pr);
                }
            }
            // byte offset of (row j, column d0) in a K-major SWIZZLE_128B region of N rows
            const int half = d0 / 64, col = d0 % 64;
            const uint32_t off = (uint32_t)half * (uint32_t)(N * 128) + (uint32_t)j * 128u +
                                 (uint32_t)((((col / 8) ^ (j & 7)) << 4) + (col % 8) * 2);
#pragma unroll
            for (int k = 0; k < 3; ++k) {
                uint8_t* dst = smem + L::kMeans + k * split_bytes + off;
                *reinterpret_cast<uint2*>(dst) = make_uint2(part[k][0], part[k][1]);
            }
        }
    }
    fence_proxy_async();  // the MMAs read these shared-memory writes through the async proxy
    if (threadIdx.x == 0) {
        mbar_init(BAR(B_QFULL), 1);
        mbar_init(BAR(B_QEMPTY), 1);
        mbar_init(BAR(B_SFULL), 1);
        mbar_init(BAR(B_SFULL + 1), 1);
        mbar_init(BAR(B_SEMPTY), 128);
        mbar_init(BAR(B_SEMPTY + 1), 128);
        mbar_init(BAR(B_FINAL), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kWarpMMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                         smem_u32(&s_tmem)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    volatile int* abort_flag = &s_abort;
    int dummy_status = 0;
    int* st = status ? status : &dummy_status;

    if (warp == kWarpMMA) {
        const uint32_t idesc = idesc_bf16(N, false);
        for (int ti = 0; ti < ntiles; ++ti) {
            const int h = g * P.group + ti % P.group, qt = ti / P.group;
            if (ti > 0 && !wait_bar(BAR(B_QEMPTY), (uint32_t)(ti - 1) & 1u, abort_flag, st)) break;
            if (lane == 0) {
                mbar_arrive_tx(BAR(B_QFULL), (uint32_t)(kTileM * D * 2));
#pragma unroll
                for (int hh = 0; hh < D / 64; ++hh)
                    tma_load_3d(sm_base + L::kQ + hh * kHalfBytesQ, &tmap_q, BAR(B_QFULL), hh * 64, h,
                                start + qt * kTileM);
            }
            __syncwarp();
            const int sb = ti & 1;
            if (!wait_bar(BAR(B_QFULL), (uint32_t)ti & 1u, abort_flag, st)) break;
            if (ti >= 2 && !wait_bar(BAR(B_SEMPTY + sb), (uint32_t)((ti >> 1) - 1) & 1u, abort_flag, st))
                break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t s_tmem = tmem + (uint32_t)sb * kMaxPast;
#pragma unroll
                for (int k = 0; k < 3; ++k) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t aoff = (uint32_t)(kk >> 2) * kHalfBytesQ + (uint32_t)(kk & 3) * 32u;
                        const uint32_t boff = (uint32_t)k * split_bytes + (uint32_t)(kk >> 2) * (uint32_t)(N * 128) +
                                              (uint32_t)(kk & 3) * 32u;
                        mma_ss(s_tmem, smem_desc(sm_base + L::kQ + aoff, 16, 1024),
                               smem_desc(m_base + boff, 16, 1024), idesc, (k > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                mma_commit(BAR(B_SFULL + sb));
                mma_commit(BAR(B_QEMPTY));
            }
            __syncwarp();
        }
        if (lane == 0) mma_commit(BAR(B_FINAL));
        __syncwarp();
        drain_bar(BAR(B_FINAL), 0);
    } else {
        // warps 0-3: thread r owns row r of every tile
        const int r = threadIdx.x;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        for (int ti = 0; ti < ntiles; ++ti) {
            const int h = g * P.group + ti % P.group, qt = ti / P.group;
            const int sb = ti & 1;
            if (!wait_bar(BAR(B_SFULL + sb), (uint32_t)(ti >> 1) & 1u, abort_flag, st)) break;
            tc_fence_after();
            // two independent descending lists (even / odd columns) for instruction-level
            // parallelism, merged at the end; inside a list, columns arrive in increasing order
            // and an equal score never displaces an earlier (lower-index) block
            float val[KMAX], val2[KMAX];
            int idx[KMAX], idx2[KMAX];
#pragma unroll
            for (int i = 0; i < KMAX; ++i) {
                val[i] = val2[i] = -INFINITY;
                idx[i] = idx2[i] = INT_MAX;
            }
            const uint32_t s_tmem = tmem + lane_off + (uint32_t)sb * kMaxPast;
            for (int j0 = 0; j0 < c; j0 += 32) {
                float v[32];
                tmem_ld32(s_tmem + (uint32_t)j0, v);
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    insert_desc<KMAX>(val, idx, v[e], j0 + e, j0 + e < c);
                    insert_desc<KMAX>(val2, idx2, v[e + 1], j0 + e + 1, j0 + e + 1 < c);
                }
            }
            // merge: scores from the odd list enter with the full (score, lower index) order
#pragma unroll
            for (int i = 0; i < KMAX; ++i) insert_ordered<KMAX>(val, idx, val2[i], idx2[i]);
            tc_fence_before();
            mbar_arrive(BAR(B_SEMPTY + sb));
            const int rr = qt * kTileM + r;
            if (rr < len) {
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
                int* dst = sel + ((size_t)h * P.T + (start + rr)) * P.topk;
#pragma unroll
                for (int i = 0; i <= KMAX; ++i) {
                    if (i < P.topk) {
                        const int vo = (i < n_route) ? o[i < KMAX ? i : KMAX - 1] : (i == n_route ? c : -1);
                        dst[i] = vo;
                    }
                }
                for (int i = KMAX + 1; i < P.topk; ++i) dst[i] = -1;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMMA) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

template <int D, int KMAX>
cudaError_t launch_tc(const Problem& P, const __nv_bfloat16* q, const float* means, const int* cu,
                      int* sel, int* status, int n_max, cudaStream_t st) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    CUtensorMap mq;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)P.hq, (cuuint64_t)P.T};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)P.hq * D * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)kTileM};
    cuuint32_t estr[3] = {1, 1, 1};
    if (fn(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16*>(q), dims, strides,
           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const int smem = GateSmem<D>::kBytes(n_max);
    cudaError_t e = cudaFuncSetAttribute(gate_tc_kernel<D, KMAX>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(P.nb_cap, P.hkv);
    gate_tc_kernel<D, KMAX><<<grid, kThreads, smem, st>>>(mq, means, cu, P, sel, status, n_max);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_tc_k(const Problem& P, const __nv_bfloat16* q, const float* means,
                        const int* cu, int* sel, int* status, int n_max, cudaStream_t st) {
    const int need = P.topk - 1;
    if (need <= 2) return launch_tc<D, 2>(P, q, means, cu, sel, status, n_max, st);
    if (need <= 4) return launch_tc<D, 4>(P, q, means, cu, sel, status, n_max, st);
    if (need <= 8) return launch_tc<D, 8>(P, q, means, cu, sel, status, n_max, st);
    if (need <= 11) return launch_tc<D, 11>(P, q, means, cu, sel, status, n_max, st);
    if (need <= 16) return launch_tc<D, 16>(P, q, means, cu, sel, status, n_max, st);
    return launch_tc<D, 32>(P, q, means, cu, sel, status, n_max, st);
}

}  // namespace

// Tensor-core gate when every sequence has at most kMaxPast + 1 blocks (P.max_blocks, from the
// caller's max_seqlen, else the block-count bound of the whole call), else the fp32 CUDA-core
// gate.  Shared memory and the MMA's N are sized for the longest sequence's past blocks.
cudaError_t launch_gate_best(const Problem& P, const __nv_bfloat16* q, const float* means,
                             const int* cu_seqlens, int* sel, int* status, cudaStream_t st,
                             int* path) {
    if (P.nb_cap == 0) return cudaSuccess;
    const bool cuda_cores = P.max_blocks > kMaxPast + 1;
    if (path) *path = cuda_cores ? 2 : 1;
    if (cuda_cores) return launch_gate(P, q, means, cu_seqlens, sel, st);
    const int n_max = ((P.max_blocks - 1) + 15) & ~15;  // largest c is max_blocks - 1
    const int n_alloc = n_max < 16 ? 16 : n_max;
    if (P.d == 64) return launch_tc_k<64>(P, q, means, cu_seqlens, sel, status, n_alloc, st);
    return launch_tc_k<128>(P, q, means, cu_seqlens, sel, status, n_alloc, st);
}

}  // namespace moba
