// Steps 3-4 of the forward on the tensor cores: gate scores of 128-row query tiles against the
// block summaries by tcgen05 MMA, then the future-block mask, the forced own block and the
// hard top-k on the CUDA cores.
//
// The analysis page of the MoBA paper (§2.2-§2.3): s_j = <q, mean_j>; blocks after the row's
// own block c are masked to -inf, block c is always taken, the best topk-1 past blocks
// (j < c) are routed.  Ties keep the lower block index.  The same kernel runs the min/max
// (Quest-style) gate the analysis names as the stronger summary (§1.3, §5.1 item 6, §6.3):
// s_j = sum_i max(q_i kmin_ji, q_i kmax_ji).
//
// Both scores are contractions with exact bf16 operands and fp32 accumulation:
//   mean:    each fp32 mean is split exactly into three bf16 parts, m = hi + mid + lo
//            (|m - hi - mid - lo| <= 2^-24 |m|), and s = q.hi + q.mid + q.lo: three MMAs of
//            K = d into one accumulator, so the score is the fp32-accurate dot product (about
//            1e-6 absolute here), far inside the 1e-3 relative near-tie band, unlike a single
//            bf16 rounding of the means (about 2e-3 relative);
//   min/max: max(q_i lo_i, q_i hi_i) = q+_i hi_i + q-_i lo_i with q+ = max(q, 0) and
//            q- = min(q, 0), so s = q+.kmax + q-.kmin: two MMAs of K = d whose products are
//            exact (bf16 x bf16 in fp32); only the fp32 accumulation rounds.
//
// One CTA per (query block b, KV head g): it stages the summaries of the c past blocks of b's
// sequence in shared memory once (SWIZZLE_128B, K-major), then runs the 128-row tiles of block
// b for the query heads of g.  The last warp loads each Q tile by TMA (and, for the min/max
// gate, splits it into q+ and q-) and issues the MMAs (N = c rounded up to 16) into TMEM.  The
// top-(topk-1) is chosen by warpgroups that take whole tiles in turn, each with its own TMEM
// score buffer (four warpgroups while four buffers fit TMEM, i.e. up to 128 past blocks, and the
// lists are short; two otherwise, or two CTAs of two per SM when a CTA has few tiles and half an
// SM's shared memory holds it), thread = row = TMEM lane, in two passes over the row's
// scores: the first keeps the topk-1 largest values (a min/max merge network, no indices), the
// second marks the blocks scoring at least the smallest of them; when equal scores at the cut
// mark too many, the highest such blocks are dropped, so ties keep the lower block index.  The
// result is the exact top-k under the (score descending, lower index) order.  Rows with at
// most topk-1 past blocks take all of them without scoring.  Sequences longer than 257 blocks
// use the fp32 CUDA-core gate instead (gate.cu).
#include <climits>

#include "moba_internal.cuh"
#include "ptx.cuh"

namespace moba {

namespace {

using namespace ptx;

constexpr int kMaxPast = 256;   // past blocks scored in one MMA (N <= 256)
constexpr int kWords = kMaxPast / 32;  // a row's past blocks as a bit mask
constexpr int kMaxQBuf = 4;            // Q tile buffers (loads run ahead of the MMAs)
constexpr int kHalfSmLimit = 113 * 1024;  // dynamic shared memory of one of two CTAs per SM

// The K largest values seen so far, descending (-inf until K were seen).  Adding a pair is a
// merge with the sorted two-element list (a, b), a >= b: the i-th largest of the union is
// max(val[i], min(val[i-1], a), min(val[i-2], b)) with val[-1] = val[-2] = +inf.  Each position
// takes two mins and a three-input max of old values, so the K positions are independent and
// an insertion has no compares, selects or branches.
template <int K>
__device__ __forceinline__ void top_values_pair(float (&val)[K], float x0, float x1) {
    const float a = fmaxf(x0, x1), b = fminf(x0, x1);
#pragma unroll
    for (int i = K - 1; i >= 2; --i) val[i] = fmax3(val[i], fminf(val[i - 1], a), fminf(val[i - 2], b));
    if constexpr (K >= 2) val[1] = fmax3(val[1], fminf(val[0], a), b);
    val[0] = fmaxf(val[0], a);
}

// Top-k warpgroups, each ranking whole tiles in its own TMEM score buffer: four when the scores
// of a tile take at most 128 columns, two when they take 256 (TMEM holds 512 columns) or when
// the lists are long (topk - 1 > 16, for registers).
template <int NWG>
struct GateWarps {
    static constexpr int kNumWG = NWG;
    static constexpr int kThreads = kNumWG * 128 + 32;  // + the TMA / MMA warp
    static constexpr int kWarpMMA = kNumWG * 4;
};

__host__ __device__ constexpr int pow2_at_least(int x) {
    int p = 32;
    while (p < x) p *= 2;
    return p;
}

// TMEM plan of one launch (the same in every CTA): one buffer of NC columns (a power of two
// >= the largest N) per warpgroup.
__host__ __device__ inline int gate_cols(int n_alloc, int nwg) { return nwg * pow2_at_least(n_alloc); }

template <int D, bool MINMAX>
struct GateCfg {
    static constexpr int kPairs = MINMAX ? 2 : 3;     // (A, B) products accumulated per score
    static constexpr int kARegions = MINMAX ? 2 : 1;  // q (mean) or q+, q- (min/max)
    static constexpr int kTile = kTileM * D * 2;      // one [128 x D] bf16 tile
    // shared memory: NQ Q buffers, then kPairs B regions of [N x D] bf16, then barriers
    static constexpr int kQBytes(int nq) { return nq * kARegions * kTile; }
    static constexpr int kBars(int nq, int n) { return kQBytes(nq) + kPairs * n * D * 2; }
    static constexpr int kNumBars = 24;
    static constexpr int kBytes(int nq, int n) { return kBars(nq, n) + kNumBars * 8 + 16 + 1024; }
};

// q -> (q+, q-) in place: per bf16, q+ keeps positive values (and +0), q- negative ones.
__device__ __forceinline__ void split_sign(uint32_t x, uint32_t& pos, uint32_t& neg) {
    const uint32_t m = ((x >> 15) & 0x00010001u) * 0xFFFFu;  // 0xFFFF per negative half
    pos = x & ~m;
    neg = x & m;
}

template <int D, int KMAX, bool MINMAX, int NWG, int MINB>
__global__ void __launch_bounds__(GateWarps<NWG>::kThreads, MINB)
gate_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const float* __restrict__ means,
               const __nv_bfloat16* __restrict__ kmin, const __nv_bfloat16* __restrict__ kmax,
               const int* __restrict__ cu, Problem P, int* __restrict__ sel, int* status, int n_cap,
               int smem_bytes) {
    using C = GateCfg<D, MINMAX>;
    constexpr int kThreads = GateWarps<NWG>::kThreads;
    constexpr int kWarpMMA = GateWarps<NWG>::kWarpMMA;
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

    if (n_route == c || n_route == 0 || c > n_cap) {
        // nothing to choose: every past block is routed (c <= topk - 1), or none (topk = 1).
        // c > n_cap means the sequence is longer than the caller's max_seqlen promised: its rows
        // keep the own block only and the call's status word (when there is one) records the
        // broken promise.
        const bool broken = c > n_cap;
        if (broken && threadIdx.x == 0 && status) atomicExch(status, 1 /* INVALID_ARG */);
        for (int e = threadIdx.x; e < len * P.group; e += kThreads) {
            const int h = g * P.group + e / len;
            const int t = start + e % len;
            int* dst = sel + ((size_t)h * P.T + t) * P.topk;
            const int nr = broken ? 0 : n_route;
            for (int i = 0; i < P.topk; ++i) dst[i] = (i < nr) ? i : (i == nr ? c : -1);
        }
        return;
    }
    const int N = (c + 15) & ~15;  // MMA N: past blocks rounded up to 16 (c <= n_cap)
    const int split_bytes = N * D * 2;
    const int nc = pow2_at_least(n_cap);  // TMEM columns of one warpgroup's score buffer
    const int tmem_cols = gate_cols(n_cap, NWG);
    // Q buffers: as many as the launch's shared memory holds next to this CTA's summaries (at
    // most kMaxQBuf), so the Q loads run up to nq - 1 tiles ahead of the MMAs
    int nq = kMaxQBuf;
    while (nq > 1 && C::kBytes(nq, N) > smem_bytes) --nq;
    const uint32_t sm_base = smem_u32(smem);
    const uint32_t b_base = sm_base + C::kQBytes(nq);
    const uint32_t bar0 = sm_base + C::kBars(nq, N);
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    // per Q buffer: QFULL (loaded), QEMPTY (its MMAs are done); per warpgroup w: SFULL + w (its
    // scores are in TMEM), SEMPTY + w (it has read them)
    const int B_QFULL = 0, B_QEMPTY = kMaxQBuf, B_SFULL = 2 * kMaxQBuf, B_SEMPTY = B_SFULL + 4,
              B_FINAL = B_SEMPTY + 4;

    // stage the summaries of past blocks 0..c-1 as K-major SW128 rows (rows c..N-1 are zero)
    {
        const size_t mstride = (size_t)P.hkv * D;
        // byte offset of (row j, column d0) in a K-major SWIZZLE_128B region of N rows
        auto swz = [&](int j, int d0) {
            const int half = d0 / 64, col = d0 % 64;
            return (uint32_t)half * (uint32_t)(N * 128) + (uint32_t)j * 128u +
                   (uint32_t)((((col / 8) ^ (j & 7)) << 4) + (col % 8) * 2);
        };
        if constexpr (MINMAX) {
            const __nv_bfloat16* hi0 = kmax + ((size_t)s_first * P.hkv + g) * D;
            const __nv_bfloat16* lo0 = kmin + ((size_t)s_first * P.hkv + g) * D;
            for (int e = threadIdx.x; e < N * (D / 8); e += kThreads) {
                const int j = e / (D / 8), d0 = (e % (D / 8)) * 8;
                uint4 h4 = make_uint4(0u, 0u, 0u, 0u), l4 = h4;
                if (j < c) {
                    h4 = __ldg(reinterpret_cast<const uint4*>(hi0 + (size_t)j * mstride + d0));
                    l4 = __ldg(reinterpret_cast<const uint4*>(lo0 + (size_t)j * mstride + d0));
                }
                *reinterpret_cast<uint4*>(smem + C::kQBytes(nq) + swz(j, d0)) = h4;
                *reinterpret_cast<uint4*>(smem + C::kQBytes(nq) + split_bytes + swz(j, d0)) = l4;
            }
        } else {
            const float* mg = means + ((size_t)s_first * P.hkv + g) * D;
            for (int e = threadIdx.x; e < N * (D / 4); e += kThreads) {
                const int j = e / (D / 4), d0 = (e % (D / 4)) * 4;
                float4 m4 = make_float4(0.f, 0.f, 0.f, 0.f);
                if (j < c) m4 = __ldg(reinterpret_cast<const float4*>(mg + (size_t)j * mstride + d0));
                const float mv[4] = {m4.x, m4.y, m4.z, m4.w};
                uint32_t part[3][2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    float r0 = mv[2 * u], r1 = mv[2 * u + 1];
#pragma unroll
                    for (int k = 0; k < 3; ++k) {
                        const __nv_bfloat16 h0 = __float2bfloat16_rn(r0), h1 = __float2bfloat16_rn(r1);
                        r0 -= __bfloat162float(h0);
                        r1 -= __bfloat162float(h1);
                        __nv_bfloat162 pr;
                        pr.x = h0;
                        pr.y = h1;
                        part[k][u] = *reinterpret_cast<uint32_t*>(&pr);
                    }
                }
#pragma unroll
                for (int k = 0; k < 3; ++k)
                    *reinterpret_cast<uint2*>(smem + C::kQBytes(nq) + k * split_bytes + swz(j, d0)) =
                        make_uint2(part[k][0], part[k][1]);
            }
        }
    }
    fence_proxy_async();  // the MMAs read these shared-memory writes through the async proxy
    if (threadIdx.x == 0) {
        for (int i = 0; i < kMaxQBuf; ++i) {
            mbar_init(BAR(B_QFULL + i), 1);
            mbar_init(BAR(B_QEMPTY + i), 1);
        }
        for (int i = 0; i < NWG; ++i) {
            mbar_init(BAR(B_SFULL + i), 1);
            mbar_init(BAR(B_SEMPTY + i), 128);
        }
        mbar_init(BAR(B_FINAL), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kWarpMMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&s_tmem)), "r"(tmem_cols));
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
        // ---------------- Q tiles (TMA), q+ / q- split, MMA issue ----------------
        const uint32_t idesc = idesc_bf16(N, false);
        // tile ti is loaded into buffer ti % nq (its (ti / nq)-th use)
        auto load_q = [&](int ti) {
            const int h = g * P.group + ti % P.group, qt = ti / P.group;
            const int qb = ti % nq;
            const uint32_t qbase = sm_base + (uint32_t)qb * C::kARegions * C::kTile;
            if (lane == 0) {
                mbar_arrive_tx(BAR(B_QFULL + qb), (uint32_t)C::kTile);
#pragma unroll
                for (int hh = 0; hh < D / 64; ++hh)
                    tma_load_3d(qbase + hh * kHalfBytesQ, &tmap_q, BAR(B_QFULL + qb), hh * 64, h,
                                start + qt * kTileM);
            }
            __syncwarp();
        };
        int next_load = min(nq, ntiles), consumed = 0;
        for (int ti = 0; ti < next_load; ++ti) load_q(ti);
        for (int ti = 0; ti < ntiles; ++ti) {
            const int qb = ti % nq;
            const uint32_t uq = (uint32_t)(ti / nq);
            const uint32_t qbase = sm_base + (uint32_t)qb * C::kARegions * C::kTile;
            if (!wait_bar(BAR(B_QFULL + qb), uq & 1u, abort_flag, st)) break;
            consumed = ti + 1;
            if constexpr (MINMAX) {
                uint4* qp = reinterpret_cast<uint4*>(smem + (size_t)qb * C::kARegions * C::kTile);
                uint4* qm = qp + C::kTile / 16;
                for (int i = lane; i < C::kTile / 16; i += 32) {
                    const uint4 x = qp[i];
                    uint4 p4, n4;
                    split_sign(x.x, p4.x, n4.x);
                    split_sign(x.y, p4.y, n4.y);
                    split_sign(x.z, p4.z, n4.z);
                    split_sign(x.w, p4.w, n4.w);
                    qp[i] = p4;
                    qm[i] = n4;
                }
                fence_proxy_async();
                __syncwarp();
            }
            // tile ti goes to warpgroup ti % NWG (its u-th tile), into that warpgroup's buffer
            const int buf = ti % NWG;
            const uint32_t u = (uint32_t)(ti / NWG);
            if (u >= 1 && !wait_bar(BAR(B_SEMPTY + buf), (u - 1u) & 1u, abort_flag, st)) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t s_tmem = tmem + (uint32_t)(buf * nc);
#pragma unroll
                for (int p = 0; p < C::kPairs; ++p) {
                    const uint32_t abase = qbase + (uint32_t)(MINMAX ? p : 0) * C::kTile;
                    const uint32_t bbase = b_base + (uint32_t)p * (uint32_t)split_bytes;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t aoff = (uint32_t)(kk >> 2) * kHalfBytesQ + (uint32_t)(kk & 3) * 32u;
                        const uint32_t boff = (uint32_t)(kk >> 2) * (uint32_t)(N * 128) + (uint32_t)(kk & 3) * 32u;
                        mma_ss(s_tmem, smem_desc(abase + aoff, 16, 1024), smem_desc(bbase + boff, 16, 1024),
                               idesc, (p > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                mma_commit(BAR(B_SFULL + buf));
                mma_commit(BAR(B_QEMPTY + qb));
            }
            __syncwarp();
            // refill: tile next_load goes where tile next_load - nq was, once that tile's MMAs
            // are complete.  With several buffers that tile was issued before this one (so its
            // MMAs are done or nearly), which keeps the tensor pipe fed; with one buffer it is
            // this tile.
            if (next_load < ntiles && (nq == 1 || next_load - nq < ti)) {
                const int prev = next_load - nq;
                if (!wait_bar(BAR(B_QEMPTY + prev % nq), (uint32_t)(prev / nq) & 1u, abort_flag, st)) break;
                load_q(next_load++);
            }
        }
        // Q loads still in flight after an abort land before the CTA exits (bounded)
        for (int ti = consumed; ti < next_load; ++ti) drain_bar(BAR(B_QFULL + ti % nq), (uint32_t)(ti / nq) & 1u);
        if (lane == 0) mma_commit(BAR(B_FINAL));
        __syncwarp();
        drain_bar(BAR(B_FINAL), 0);
    } else {
        // ---------------- top-k: warpgroup wg takes tiles wg, wg + NWG, ...; thread = row ----------------
        const int wg = warp >> 2;
        const int r = threadIdx.x & 127;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t s_tmem = tmem + lane_off + (uint32_t)(wg * nc);
        for (int ti = wg; ti < ntiles; ti += NWG) {
            const int h = g * P.group + ti % P.group, qt = ti / P.group;
            const uint32_t u = (uint32_t)(ti / NWG);
            if (!wait_bar(BAR(B_SFULL + wg), u & 1u, abort_flag, st)) break;
            tc_fence_after();
            // pass 1: the n_route largest scores of the row, values only
            float val[KMAX];
#pragma unroll
            for (int i = 0; i < KMAX; ++i) val[i] = -INFINITY;
            for (int j0 = 0; j0 < c; j0 += 32) {
                float v[32];
                tmem_ld32(s_tmem + (uint32_t)j0, v);
                if (j0 + 32 > c) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = (j0 + e < c) ? v[e] : -INFINITY;
                }
#pragma unroll
                for (int e = 0; e < 32; e += 2) top_values_pair<KMAX>(val, v[e], v[e + 1]);
            }
            // vk = val[n_route - 1], the smallest of the first n_route (val is descending)
            float vk = val[0];
#pragma unroll
            for (int i = 1; i < KMAX; ++i) vk = fminf(vk, (i < n_route) ? val[i] : INFINITY);
            // pass 2: the blocks scoring at least vk, as a bit mask in block order
            uint32_t m[kWords];
            int cnt = 0;
#pragma unroll
            for (int w = 0; w < kWords; ++w) {
                m[w] = 0u;
                if (w * 32 < c) {
                    float v[32];
                    tmem_ld32(s_tmem + (uint32_t)(w * 32), v);
                    uint32_t mw = 0u;
#pragma unroll
                    for (int e = 0; e < 32; ++e) mw |= (v[e] >= vk) ? (1u << e) : 0u;
                    if (c - w * 32 < 32) mw &= (1u << (c - w * 32)) - 1u;
                    m[w] = mw;
                    cnt += __popc(mw);
                }
            }
            // scores equal to vk beyond the n_route places: the higher blocks drop out (ties
            // keep the lower block index)
            int excess = cnt - n_route;
            if (__any_sync(0xffffffffu, excess > 0)) {
#pragma unroll
                for (int w = kWords - 1; w >= 0; --w) {
                    if (w * 32 < c) {
                        float v[32];
                        tmem_ld32(s_tmem + (uint32_t)(w * 32), v);
                        uint32_t eq = 0u;
#pragma unroll
                        for (int e = 0; e < 32; ++e) eq |= (v[e] == vk) ? (1u << e) : 0u;
                        eq &= m[w];
                        while (excess > 0 && eq != 0u) {
                            const uint32_t top = 1u << (31 - __clz(eq));
                            m[w] &= ~top;
                            eq &= ~top;
                            --excess;
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(BAR(B_SEMPTY + wg));
            const int rr = qt * kTileM + r;
            if (rr < len) {
                // routed blocks ascending, then the own block (pos < n_route only when the
                // scores were not finite)
                int* dst = sel + ((size_t)h * P.T + (start + rr)) * P.topk;
                int pos = 0;
#pragma unroll
                for (int w = 0; w < kWords; ++w) {
                    uint32_t mw = m[w];
                    while (mw != 0u && pos < n_route) {
                        dst[pos++] = w * 32 + __ffs(mw) - 1;
                        mw &= mw - 1u;
                    }
                }
                dst[pos] = c;
                for (int i = pos + 1; i < P.topk; ++i) dst[i] = -1;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMMA) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tmem_cols));
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

// MINB CTAs per SM: with MINB = 2 the launch keeps to half an SM's shared memory (and the
// kernel to half its registers) so that a second CTA's loads overlap this one's compute.
template <int D, int KMAX, bool MINMAX, int NWG, int MINB>
cudaError_t launch_tc_w(const Problem& P, const CUtensorMap& mq, const GateSummary& s, const int* cu,
                        int* sel, int* status, int n_max, cudaStream_t st) {
    using C = GateCfg<D, MINMAX>;
    // as many Q buffers (up to kMaxQBuf) as fit next to the longest sequence's summaries; a CTA
    // with fewer past blocks fits more into the same allocation
    const int limit = MINB == 1 ? 227 * 1024 : kHalfSmLimit;
    int nq = MINB == 1 ? kMaxQBuf : 2;
    while (nq > 1 && C::kBytes(nq, n_max) > limit) --nq;
    const int smem = C::kBytes(nq, n_max);
    cudaError_t e = cudaFuncSetAttribute(gate_tc_kernel<D, KMAX, MINMAX, NWG, MINB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(P.nb_cap, P.hkv);
    gate_tc_kernel<D, KMAX, MINMAX, NWG, MINB><<<grid, GateWarps<NWG>::kThreads, smem, st>>>(
        mq, s.means, s.kmin, s.kmax, cu, P, sel, status, n_max, smem);
    return cudaGetLastError();
}

template <int D, int KMAX, bool MINMAX>
cudaError_t launch_tc(const Problem& P, const __nv_bfloat16* q, const GateSummary& s, const int* cu,
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
    using C = GateCfg<D, MINMAX>;
    if constexpr (KMAX <= 16) {
        // few query tiles per CTA (short blocks, small groups): each CTA is short and mostly
        // waits for its loads, so two CTAs of two warpgroups share an SM when half its shared
        // memory holds one
        const int tiles = (P.chunk + kTileM - 1) / kTileM * P.group;
        if (tiles <= 16 && C::kBytes(1, n_max) <= kHalfSmLimit)
            return launch_tc_w<D, KMAX, MINMAX, 2, 2>(P, mq, s, cu, sel, status, n_max, st);
        // four warpgroups while four score buffers fit TMEM and the lists are short (a longer
        // list needs more than the 120 registers a thread of 544 may have), else two
        if (pow2_at_least(n_max) <= 128)
            return launch_tc_w<D, KMAX, MINMAX, 4, 1>(P, mq, s, cu, sel, status, n_max, st);
    }
    return launch_tc_w<D, KMAX, MINMAX, 2, 1>(P, mq, s, cu, sel, status, n_max, st);
}

template <int D, bool MINMAX>
cudaError_t launch_tc_k(const Problem& P, const __nv_bfloat16* q, const GateSummary& s, const int* cu,
                        int* sel, int* status, int n_max, cudaStream_t st) {
    const int need = P.topk - 1;
    if (need <= 2) return launch_tc<D, 2, MINMAX>(P, q, s, cu, sel, status, n_max, st);
    if (need <= 4) return launch_tc<D, 4, MINMAX>(P, q, s, cu, sel, status, n_max, st);
    if (need <= 8) return launch_tc<D, 8, MINMAX>(P, q, s, cu, sel, status, n_max, st);
    if (need <= 11) return launch_tc<D, 11, MINMAX>(P, q, s, cu, sel, status, n_max, st);
    if (need <= 16) return launch_tc<D, 16, MINMAX>(P, q, s, cu, sel, status, n_max, st);
    return launch_tc<D, 32, MINMAX>(P, q, s, cu, sel, status, n_max, st);
}

}  // namespace

// Tensor-core gate when every sequence has at most kMaxPast + 1 blocks (P.max_blocks, from the
// caller's max_seqlen, else the block-count bound of the whole call), else the fp32 CUDA-core
// gate (mean gate only).  Shared memory, TMEM and the MMA's N are sized for the longest
// sequence's past blocks.
cudaError_t launch_gate_best(const Problem& P, const __nv_bfloat16* q, const GateSummary& s,
                             const int* cu_seqlens, int* sel, int* status, cudaStream_t st,
                             int* path) {
    if (P.nb_cap == 0) return cudaSuccess;
    const bool minmax = s.kmin != nullptr;
    const bool cuda_cores = P.max_blocks > kMaxPast + 1;
    if (path) *path = cuda_cores ? 2 : 1;
    if (cuda_cores) {
        if (minmax) return cudaErrorNotSupported;
        return launch_gate(P, q, s.means, cu_seqlens, sel, st);
    }
    const int n_max = ((P.max_blocks - 1) + 15) & ~15;  // largest c is max_blocks - 1
    const int n_alloc = n_max < 16 ? 16 : n_max;
    if (minmax) {
        if (P.d == 64) return launch_tc_k<64, true>(P, q, s, cu_seqlens, sel, status, n_alloc, st);
        return launch_tc_k<128, true>(P, q, s, cu_seqlens, sel, status, n_alloc, st);
    }
    if (P.d == 64) return launch_tc_k<64, false>(P, q, s, cu_seqlens, sel, status, n_alloc, st);
    return launch_tc_k<128, false>(P, q, s, cu_seqlens, sel, status, n_alloc, st);
}

}  // namespace moba
