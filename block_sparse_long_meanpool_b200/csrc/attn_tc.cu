// Step 5 of the forward on the 5th-generation tensor cores (tcgen05 + TMEM + TMA), sm_100a.
//
// The analysis page of the MoBA paper (§3.2): history blocks are attended without a causal
// mask (rule 1 of §2.3 already excluded every future block), the own block with a causal
// mask, and the partial softmax results are merged afterwards by their log-sum-exp.
//
// Work items (from the routing pass) are 128 query rows against one KV range: a history tile
// is up to 128 routed rows (any query heads of one KV head) against one whole block, a
// current-block tile is 128 consecutive tokens of one query head against the causal prefix
// of their block.  Two persistent CTAs per SM take items from an atomic cursor; each is a
// single-tile pipeline, and the two run out of phase so that one CTA's softmax overlaps the
// other's matrix products on the SM's tensor core.
//
// Warp roles per CTA (224 threads):
//   warps 0-3  softmax + epilogue, thread r owns query row r (TMEM lane r)
//   warp 4     K/V producer: TMA (SWIZZLE_128B, no multicast) into a 2-stage ring
//   warp 5     item fetch + Q gather: routed rows by cp.async into a swizzled K-major tile
//   warp 6     TMEM owner and single-thread MMA issuer
// Per 128-key chunk n: S_n = Q K_n^T (SS MMA, fp32 in TMEM); the softmax reads S_n twice with
// tcgen05.ld (row maximum, then p = 2^(s*scale*log2e - m)) and writes P_n as bf16 pairs over
// the S columns it has already read; then O += P_n V_n (TS MMA: A = P from TMEM, B = V
// MN-major from shared memory).  The MMA warp issues PV_{n-1} before QK_n, so the barrier
// that announces S_n also guarantees that O holds every earlier PV: the softmax may rescale
// O right away.  The running max is only raised (and O rescaled) when it grows by more than
// 2^8, so O is rarely touched.  TMEM per CTA: S/P 128 columns + O d columns (256 allocated).
//
// Every mbarrier wait is bounded: on expiry the kernel records MOBA_ERR_DEVICE_TIMEOUT in
// the workspace status word, all roles leave their loops, in-flight copies and MMAs are
// drained (bounded), TMEM is freed and the CTA returns.
#include <cuda.h>

#include <climits>

#include "moba_internal.cuh"
#include "ptx.cuh"

namespace moba {

namespace {

using namespace ptx;

constexpr int kBN = 128;       // keys per chunk
constexpr int kStages = 2;     // K/V ring depth
constexpr int kThreads = 224;  // 7 warps
constexpr int kWarpKV = 4, kWarpQ = 5, kWarpMMA = 6;
constexpr int kCtasPerSm = 2;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O is rescaled when max grows > 2^8

struct ItemSlot {
    int kind;  // -1 = no more work
    int g, key_start, key_end, nchunks;
    int pidx[kTileM];
    int tlim[kTileM];
};

template <int D>
struct SmemLayout {
    static constexpr int kTileBytes = kTileM * D * 2;  // 128 rows of bf16 (Q tile, K or V chunk)
    static constexpr int kQ = 0;                       // one Q buffer
    static constexpr int kKV = kTileBytes;             // kStages K/V buffers
    static constexpr int kSlots = kKV + kStages * kTileBytes;
    static constexpr int kBars = kSlots + 2 * (int)sizeof(ItemSlot);
    static constexpr int kNumBars = 16;
    static constexpr int kMisc = kBars + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16 + 1024;  // + slack for 1024-byte alignment
};

// One butterfly stage of an 8x8 transpose of float4 elements across the 8 lanes of a lane
// group: lanes i and i^DIST exchange the element pairs whose index bit DIST differs from
// their lane bit.  After stages 4, 2, 1, lane i holds a[j] = original a[i] of lane j.
template <int DIST>
__device__ __forceinline__ void transpose8x8(float4 (&a)[8], int lane) {
    const bool up = (lane & DIST) != 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        if (j & DIST) continue;
        const float4 send = up ? a[j] : a[j | DIST];
        float4 recv;
        recv.x = __shfl_xor_sync(0xffffffffu, send.x, DIST);
        recv.y = __shfl_xor_sync(0xffffffffu, send.y, DIST);
        recv.z = __shfl_xor_sync(0xffffffffu, send.z, DIST);
        recv.w = __shfl_xor_sync(0xffffffffu, send.w, DIST);
        if (up) a[j] = recv; else a[j | DIST] = recv;
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
               const __nv_bfloat16* __restrict__ q, Problem P, Workspace ws, int t0, int t1) {
    using L = SmemLayout<D>;
    constexpr int kHalves = D / 64;           // 128-byte swizzle atoms along d
    constexpr int kHalfBytes = kTileM * 128;  // one [128 rows x 64 bf16] swizzled half
    constexpr uint32_t kChunkBytes = kTileM * D * 2;
    constexpr int kKSteps = D / 16;           // QK^T k-steps (16 bf16 each)
    constexpr uint32_t kIdescQK = idesc_bf16(kBN, false);
    constexpr uint32_t kIdescPV = idesc_bf16(D, true);
    constexpr uint32_t kColS = 0, kColO = kBN;  // TMEM: S (P over its first 64 columns), O
    constexpr uint32_t kTmemCols = 256;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    ItemSlot* slots = reinterpret_cast<ItemSlot*>(smem + L::kSlots);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

    const uint32_t sm_base = smem_u32(smem);
    const uint32_t bar0 = sm_base + L::kBars;
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    const int B_INFO = 0, B_ITEM_EMPTY = 2, B_QFULL = 4, B_QEMPTY = 5, B_KV_FULL = 6,
              B_KV_EMPTY = 6 + kStages, B_SFULL = 6 + 2 * kStages, B_PFULL = B_SFULL + 1,
              B_OFULL = B_PFULL + 1, B_OEMPTY = B_OFULL + 1, B_FINAL = B_OEMPTY + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int* status = &ws.hdr->status;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(BAR(B_INFO + i), 32);
            mbar_init(BAR(B_ITEM_EMPTY + i), 128);
        }
        for (int i = 0; i < kStages; ++i) {
            mbar_init(BAR(B_KV_FULL + i), 1);
            mbar_init(BAR(B_KV_EMPTY + i), 1);
        }
        mbar_init(BAR(B_QFULL), 32);
        mbar_init(BAR(B_QEMPTY), 1);
        mbar_init(BAR(B_SFULL), 1);
        mbar_init(BAR(B_PFULL), 128);
        mbar_init(BAR(B_OFULL), 1);
        mbar_init(BAR(B_OEMPTY), 128);
        mbar_init(BAR(B_FINAL), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kWarpMMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)), "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kWarpQ) {
        // ---------------- item fetch + Q gather ----------------
        const int n_items = ws.hdr->n_items;
        constexpr int CK = D / 8;  // 16-byte chunks per row
        for (int it = 0;; ++it) {
            const int s = it & 1;
            const uint32_t ph = (uint32_t)(it >> 1) & 1u;
            if (it >= 2 && !wait_bar(BAR(B_ITEM_EMPTY + s), ph ^ 1u, abort_flag, status)) break;
            int idx = 0;
            if (lane == 0) idx = (int)atomicAdd(&ws.hdr->work_counter, 1u);
            idx = __shfl_sync(0xffffffffu, idx, 0);
            ItemSlot& sl = slots[s];
            if (idx >= n_items) {
                if (lane == 0) sl.kind = -1;
                __syncwarp();
                mbar_arrive(BAR(B_INFO + s));
                break;
            }
            const WorkItem w = ws.items[idx];
            int g, key_start, key_end;
            long long qoff[kTileM / 32];
            if (w.kind == 0) {
                g = w.a / P.nb_cap;
                const int b = w.a - g * P.nb_cap;
                key_start = ws.blk_start[b];
                key_end = key_start + ws.blk_len[b];
#pragma unroll
                for (int i = 0; i < kTileM / 32; ++i) {
                    const int r = lane + 32 * i;
                    int pidx = -1;
                    long long off = -1;
                    if (r < w.c) {
                        pidx = ws.entries[w.b + r];
                        const int rid = pidx / P.topk;
                        const int t = t0 + rid / P.hq;
                        const int h = rid - (rid / P.hq) * P.hq;
                        off = ((long long)t * P.hq + h) * D;
                    }
                    sl.pidx[r] = pidx;
                    sl.tlim[r] = INT_MAX;
                    qoff[i] = off;
                }
            } else {
                const int b = w.a, h = w.b, qt = w.c;
                g = h / P.group;
                key_start = ws.blk_start[b];
                const int len = ws.blk_len[b];
                key_end = key_start + min((qt + 1) * kTileM, len);
#pragma unroll
                for (int i = 0; i < kTileM / 32; ++i) {
                    const int r = lane + 32 * i;
                    const int rr = qt * kTileM + r;
                    const int t = key_start + rr;
                    const bool ok = rr < len && t >= t0 && t < t1;
                    sl.pidx[r] = ok ? ((t - t0) * P.hq + h) * P.topk : -1;
                    sl.tlim[r] = ok ? t : INT_MAX;
                    qoff[i] = ok ? ((long long)t * P.hq + h) * D : -1;
                }
            }
            if (lane == 0) {
                sl.kind = w.kind;
                sl.g = g;
                sl.key_start = key_start;
                sl.key_end = key_end;
                sl.nchunks = (key_end - key_start + kBN - 1) / kBN;
            }
            __syncwarp();
            mbar_arrive(BAR(B_INFO + s));
            // the single Q buffer is free once every QK^T of the previous item has completed
            if (it >= 1 && !wait_bar(BAR(B_QEMPTY), (uint32_t)(it - 1) & 1u, abort_flag, status)) break;
            const uint32_t qbuf = sm_base + L::kQ;
#pragma unroll
            for (int i = 0; i < kTileM / 32; ++i) {
                const int r = lane + 32 * i;
                const long long off = qoff[i];
                const __nv_bfloat16* src = off >= 0 ? q + off : q;
#pragma unroll
                for (int c = 0; c < CK; ++c) {
                    const uint32_t dst = qbuf + (uint32_t)(c >> 3) * kHalfBytes + (uint32_t)r * 128u +
                                         (uint32_t)(((c & 7) ^ (r & 7)) << 4);
                    cp_async16(dst, src + (off >= 0 ? c * 8 : 0), off >= 0);
                }
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
            asm volatile("cp.async.wait_group 0;" ::: "memory");
            fence_proxy_async();
            mbar_arrive(BAR(B_QFULL));
        }
    } else if (warp == kWarpKV) {
        // ---------------- K/V producer (TMA), in MMA consumption order K0 V0 K1 V1 ... ----------
        uint32_t c = 0;  // ring position
        for (int it = 0;; ++it) {
            const int s = it & 1;
            if (!wait_bar(BAR(B_INFO + s), (uint32_t)(it >> 1) & 1u, abort_flag, status)) break;
            const ItemSlot& sl = slots[s];
            if (sl.kind < 0) break;
            const int g = sl.g, key_start = sl.key_start, N = sl.nchunks;
            bool ok = true;
            for (int j = 0; j < 2 * N && ok; ++j) {
                const bool is_v = (j & 1) != 0;
                const int chunk = j >> 1;
                const uint32_t st = c % kStages;
                if (c >= kStages &&
                    !wait_bar(BAR(B_KV_EMPTY + st), ((c / kStages) - 1u) & 1u, abort_flag, status)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    const uint32_t dst = sm_base + L::kKV + st * L::kTileBytes;
                    mbar_arrive_tx(BAR(B_KV_FULL + st), kChunkBytes);
                    const void* tm = is_v ? (const void*)&tmap_v : (const void*)&tmap_k;
#pragma unroll
                    for (int hh = 0; hh < kHalves; ++hh)
                        tma_load_3d(dst + hh * kHalfBytes, tm, BAR(B_KV_FULL + st), hh * 64, g,
                                    key_start + chunk * kBN);
                }
                __syncwarp();
                ++c;
            }
            if (!ok) break;
        }
        // drain: every issued load must land before the CTA exits
        const uint32_t issued = c;
        for (uint32_t k = (issued > kStages ? issued - kStages : 0); k < issued; ++k)
            drain_bar(BAR(B_KV_FULL + k % kStages), (k / kStages) & 1u);
    } else if (warp == kWarpMMA) {
        // ---------------- MMA issuer: QK0, then per n >= 1: PV_{n-1}, QK_n; finally PV_{N-1} ----
        uint32_t c = 0;     // ring position
        uint32_t glob = 0;  // global chunk counter (S / P barrier phases)
        bool ok = true;
        const uint32_t s_tmem = tmem + kColS, o_tmem = tmem + kColO;
        auto wait_stage = [&]() -> uint32_t {
            const uint32_t st = c % kStages;
            if (!wait_bar(BAR(B_KV_FULL + st), (c / kStages) & 1u, abort_flag, status)) return ~0u;
            tc_fence_after();
            return st;
        };
        for (int it = 0; ok; ++it) {
            const int s = it & 1;
            if (!wait_bar(BAR(B_INFO + s), (uint32_t)(it >> 1) & 1u, abort_flag, status)) break;
            const ItemSlot& sl = slots[s];
            if (sl.kind < 0) break;
            const int N = sl.nchunks;
            if (!wait_bar(BAR(B_QFULL), (uint32_t)it & 1u, abort_flag, status)) break;
            tc_fence_after();
            const uint32_t qbuf = sm_base + L::kQ;
            for (int n = 0; n <= N && ok; ++n) {
                if (n > 0) {
                    // PV_{n-1}: P from TMEM (16 keys = 8 packed columns per step), V MN-major
                    const uint32_t pg = glob + (uint32_t)(n - 1);
                    if (!wait_bar(BAR(B_PFULL), pg & 1u, abort_flag, status)) { ok = false; break; }
                    if (n == 1 && it >= 1 &&
                        !wait_bar(BAR(B_OEMPTY), (uint32_t)(it - 1) & 1u, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = wait_stage();
                    if (st == ~0u) { ok = false; break; }
                    const uint32_t vbuf = sm_base + L::kKV + st * L::kTileBytes;
                    if (lane == 0) {
#pragma unroll
                        for (int kk = 0; kk < kBN / 16; ++kk)
                            mma_ts(o_tmem, s_tmem + (uint32_t)kk * 8u,
                                   smem_desc(vbuf + (uint32_t)kk * 2048u, (uint32_t)kHalfBytes, 1024),
                                   kIdescPV, (n > 1 || kk > 0) ? 1u : 0u);
                        mma_commit(BAR(B_KV_EMPTY + st));
                        if (n == N) mma_commit(BAR(B_OFULL));
                    }
                    __syncwarp();
                    ++c;
                }
                if (n < N) {
                    // QK_n into S (after PV_{n-1} in issue order, so P_{n-1} has been read)
                    const uint32_t st = wait_stage();
                    if (st == ~0u) { ok = false; break; }
                    const uint32_t kbuf = sm_base + L::kKV + st * L::kTileBytes;
                    if (lane == 0) {
#pragma unroll
                        for (int kk = 0; kk < kKSteps; ++kk) {
                            const uint32_t koff = (uint32_t)(kk >> 2) * kHalfBytes + (uint32_t)(kk & 3) * 32u;
                            mma_ss(s_tmem, smem_desc(qbuf + koff, 16, 1024),
                                   smem_desc(kbuf + koff, 16, 1024), kIdescQK, kk > 0 ? 1u : 0u);
                        }
                        mma_commit(BAR(B_KV_EMPTY + st));
                        mma_commit(BAR(B_SFULL));
                        if (n == N - 1) mma_commit(BAR(B_QEMPTY));
                    }
                    __syncwarp();
                    ++c;
                }
            }
            glob += (uint32_t)N;
        }
        // drain the tensor pipe before TMEM is freed
        if (lane == 0) mma_commit(BAR(B_FINAL));
        __syncwarp();
        drain_bar(BAR(B_FINAL), 0);
    } else {
        // ---------------- softmax + epilogue (warps 0-3), thread = query row ----------------
        const int row = warp * 32 + lane;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const uint32_t s_tmem = tmem + lane_off + kColS, o_tmem = tmem + lane_off + kColO;
        uint32_t glob = 0;
        const float ln2 = 0.69314718055994531f;
        const float sl2 = P.scale_log2;
        bool ok = true;
        for (int it = 0; ok; ++it) {
            const int s = it & 1;
            if (!wait_bar(BAR(B_INFO + s), (uint32_t)(it >> 1) & 1u, abort_flag, status)) break;
            const ItemSlot& sl = slots[s];
            if (sl.kind < 0) break;
            const int N = sl.nchunks, key_start = sl.key_start, key_end = sl.key_end;
            const int pidx = sl.pidx[row];
            const int tl = sl.tlim[row];
            float m = -INFINITY;  // running row maximum, log2 units
            float l = 0.f;        // running row sum of p
            for (int n = 0; n < N; ++n) {
                const uint32_t cg = glob + (uint32_t)n;
                if (!wait_bar(BAR(B_SFULL), cg & 1u, abort_flag, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // keys past the block / after the row (current-block tiles only)
                const int lim = min(key_end - 1, tl) - (key_start + n * kBN);
                const bool masked = __any_sync(0xffffffffu, lim < kBN - 1);
                // pass 1: row maximum of the raw scores
                float mh = -INFINITY;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float x[64];
                    tmem_ld64(s_tmem + 64u * hh, x);
                    if (masked) {
#pragma unroll
                        for (int j = 0; j < 64; ++j) x[j] = (64 * hh + j <= lim) ? x[j] : -INFINITY;
                    }
                    float mx[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) mx[j] = x[j];
#pragma unroll
                    for (int j = 8; j < 64; ++j) mx[j & 7] = fmaxf(mx[j & 7], x[j]);
                    mh = fmaxf(mh, fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                         fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))));
                }
                const float mloc = mh * sl2;
                if (n == 0) {
                    m = mloc;
                } else if (__any_sync(0xffffffffu, mloc > m + kRescaleThreshold)) {
                    // S_n was committed after PV_{n-1}: O already holds every earlier PV
                    const float mn = fmaxf(m, mloc);
                    const float alpha = ex2(m - mn);
#pragma unroll
                    for (int j = 0; j < D / 32; ++j) {
                        float v[32];
                        tmem_ld32(o_tmem + 32u * j, v);
                        uint32_t w[32];
#pragma unroll
                        for (int e = 0; e < 32; ++e) w[e] = __float_as_uint(v[e] * alpha);
                        tmem_st32(o_tmem + 32u * j, w);
                    }
                    tmem_st_wait();
                    l *= alpha;
                    m = mn;
                }
                // pass 2: p = 2^(s * scale * log2(e) - m) as bf16 pairs over the read S columns
                const float negm = -m;
                float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float x[64];
                    tmem_ld64(s_tmem + 64u * hh, x);
                    if (masked) {
#pragma unroll
                        for (int j = 0; j < 64; ++j) x[j] = (64 * hh + j <= lim) ? x[j] : -INFINITY;
                    }
                    uint32_t w[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float p0 = ex2(fmaf(x[2 * e], sl2, negm));
                        const float p1 = ex2(fmaf(x[2 * e + 1], sl2, negm));
                        rs0 += p0;
                        rs1 += p1;
                        w[e] = pack_bf16(p0, p1);
                    }
                    tmem_st32(s_tmem + 32u * hh, w);
                }
                l += rs0 + rs1;
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(BAR(B_PFULL));
            }
            if (!ok) break;
            // epilogue: O after the last PV, normalise, write the partial (o, lse)
            if (!wait_bar(BAR(B_OFULL), (uint32_t)it & 1u, abort_flag, status)) break;
            tc_fence_after();
            const float inv = 1.f / l;
            // Rows are 512-byte partial-output records at scattered addresses.  A thread owns a
            // row, so storing straight from registers would touch 32 cache lines per warp
            // store.  Instead each group of 8 lanes transposes 8x8 blocks of float4 by shuffles
            // and every store instruction writes 128 contiguous bytes of 4 rows.
            int prow[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) prow[jj] = __shfl_sync(0xffffffffu, pidx, (lane & ~7) + jj);
            const int seg = lane & 7;
#pragma unroll
            for (int j = 0; j < D / 32; ++j) {
                float v[32];
                tmem_ld32(o_tmem + 32u * j, v);
                float4 a[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    a[e] = make_float4(v[4 * e] * inv, v[4 * e + 1] * inv, v[4 * e + 2] * inv,
                                       v[4 * e + 3] * inv);
                transpose8x8<4>(a, lane);
                transpose8x8<2>(a, lane);
                transpose8x8<1>(a, lane);
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
                    if (prow[jj] >= 0)
                        *reinterpret_cast<float4*>(ws.part_o + (size_t)prow[jj] * D + 32 * j + 4 * seg) = a[jj];
            }
            if (pidx >= 0) ws.part_lse[pidx] = m * ln2 + logf(l);
            tc_fence_before();
            mbar_arrive(BAR(B_OEMPTY));
            mbar_arrive(BAR(B_ITEM_EMPTY + s));
            glob += (uint32_t)N;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMMA) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

// ---------------------------------------------------------------------------------------
// Host side: tensor maps through the driver entry point (no libcuda link dependency)

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
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

// [T, Hkv, d] bf16 as a 3-D tensor (d, Hkv, T); box (64, 1, 128) with 128-byte swizzle.
cudaError_t make_kv_map(CUtensorMap* m, const void* base, const Problem& P) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return cudaErrorNotSupported;
    cuuint64_t dims[3] = {(cuuint64_t)P.d, (cuuint64_t)P.hkv, (cuuint64_t)P.T};
    cuuint64_t strides[2] = {(cuuint64_t)P.d * 2, (cuuint64_t)P.hkv * P.d * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)kTileM};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D>
cudaError_t launch_tc_d(const Problem& P, const __nv_bfloat16* q, const __nv_bfloat16* k,
                        const __nv_bfloat16* v, const Workspace& ws, int t0, int t1, int num_sms,
                        cudaStream_t st) {
    CUtensorMap mk, mv;
    cudaError_t e = make_kv_map(&mk, k, P);
    if (e != cudaSuccess) return e;
    e = make_kv_map(&mv, v, P);
    if (e != cudaSuccess) return e;
    const int smem = SmemLayout<D>::kBytes;
    e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_tc_kernel<D><<<num_sms * kCtasPerSm, kThreads, smem, st>>>(mk, mv, q, P, ws, t0, t1);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const Problem& P, const __nv_bfloat16* q, const __nv_bfloat16* k,
                             const __nv_bfloat16* v, const Workspace& ws, int t0, int t1,
                             int num_sms, cudaStream_t st) {
    if (P.d == 64) return launch_tc_d<64>(P, q, k, v, ws, t0, t1, num_sms, st);
    return launch_tc_d<128>(P, q, k, v, ws, t0, t1, num_sms, st);
}

}  // namespace moba
