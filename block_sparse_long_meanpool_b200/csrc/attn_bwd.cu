// Backward pass of the MoBA attention (dQ, dK, dV) on the 5th-generation tensor cores, sm_100a.
//
// The analysis page of the MoBA paper: the gate has no parameters (§2.5) and routes by hard
// top-k (§2.2), so the selection is piecewise constant in q and K and the gradient reaches q,
// k and v only through the softmax attention over the selected union (§2.2-§2.3), with the
// forward's selection held fixed.  Per row (t, h) with attended keys U, logits
// z_u = scale q.k_u, p_u = exp(z_u - lse) and out = sum_u p_u v_u:
//   dv_u += p_u dO,   dp_u = dO . v_u,   dz_u = p_u (dp_u - Dp),  Dp = <dO, out> - dlse,
//   dq = scale sum_u dz_u k_u,   dk_u += scale dz_u q.
// The rows attending a key are those of the (KV head, block) routing list of the key's block
// (history rows: the whole block) and the block's own rows at or after the key (causal).
//
// Kernels (after the routing pass of the forward, run over all rows at once):
//   bwd_rowstats_kernel  per row: lse * log2(e) and Dp (reads dO and out; HBM stream)
//   bwd_dkdv_kernel      one CTA per (KV head, block, 128-key tile).  It streams every query
//                        row attending the tile in 64-row tiles (routed rows of the block's
//                        list, then the block's own rows of the group's heads; three warps,
//                        one per stage of a 3-stage ring, gather row tiles in turn, Q and dO
//                        together, by cp.async) and computes, with the keys on the TMEM lanes:
//                          S^T = K Q^T, dP^T = V dO^T            (SS MMA, M = 128 keys, N = 64)
//                          P^T, dS^T                             (8 warps, thread = key)
//                          dV += P^T dO, dK += dS^T Q            (TS MMA, A from TMEM)
//                        dK and dV stay in TMEM over the whole stream and are written once.
//   bwd_dq_kernel        persistent, over the forward's work items (up to two 128-row query
//                        tiles against one block's keys), per 64-key chunk:
//                          S = Q K^T, dP = dO V^T                (SS MMA, M = 128 rows, N = 64)
//                          dS                                    (8 warps, thread = row)
//                          dQ += dS K                            (TS MMA, A from TMEM)
//                        then scale * dQ of each row is added to an fp32 accumulator row with
//                        vector reductions (one per row and selected block).
//   bwd_dq_convert_kernel  fp32 accumulator -> bf16 dq.
// P and dS enter the MMAs as bf16 (as the forward's P does); every accumulation is fp32.
// Splitting dQ from dK/dV costs a recomputation of S and dP (7 tile products per (row tile,
// key tile) instead of 5) but needs no reduction per key tile and keeps dK/dV deterministic.
//
// Every mbarrier wait is bounded; on expiry the kernel records MOBA_ERR_DEVICE_TIMEOUT in the
// workspace status word, every role leaves its loop, in-flight copies and MMAs are drained
// (bounded), TMEM is freed and the CTA returns.
#include <cuda.h>

#include <climits>

#include "moba_internal.cuh"
#include "ptx.cuh"

namespace moba {

namespace {

using namespace ptx;

constexpr int kThreads = 384;  // 12 warps: 0-7 softmax-like work, 8-11 loads and MMA issue
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------------------
// Row statistics: rs[h * T + t] = (lse * log2 e, <dO, out> - dlse).  A half-warp per row.

template <int D>
__global__ void __launch_bounds__(256)
bwd_rowstats_kernel(const __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ dout,
                    const float* __restrict__ lse, const float* __restrict__ dlse, Problem P,
                    float2* __restrict__ rs) {
    constexpr int V = D / 16;  // channels per lane
    const unsigned full = 0xffffffffu;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hl = lane & 15, half = lane >> 4;
    const long long n = (long long)P.T * P.hq;
    const long long stride = (long long)gridDim.x * 16;
    for (long long base = ((long long)blockIdx.x * 8 + warp) * 2; base < n; base += stride) {
        const long long r = base + half;
        const bool valid = r < n;
        float acc = 0.f;
        if (valid) {
            const __nv_bfloat16* o = out + r * D + hl * V;
            const __nv_bfloat16* g = dout + r * D + hl * V;
            uint32_t wo[V / 2], wg[V / 2];
            if constexpr (V == 8) {
                const uint4 a = __ldcs(reinterpret_cast<const uint4*>(o));
                const uint4 b = __ldcs(reinterpret_cast<const uint4*>(g));
                wo[0] = a.x; wo[1] = a.y; wo[2] = a.z; wo[3] = a.w;
                wg[0] = b.x; wg[1] = b.y; wg[2] = b.z; wg[3] = b.w;
            } else {
                const uint2 a = __ldcs(reinterpret_cast<const uint2*>(o));
                const uint2 b = __ldcs(reinterpret_cast<const uint2*>(g));
                wo[0] = a.x; wo[1] = a.y;
                wg[0] = b.x; wg[1] = b.y;
            }
#pragma unroll
            for (int e = 0; e < V / 2; ++e) {
                const float2 fo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wo[e]));
                const float2 fg = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wg[e]));
                acc = fmaf(fo.x, fg.x, acc);
                acc = fmaf(fo.y, fg.y, acc);
            }
        }
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) acc += __shfl_xor_sync(full, acc, off);
        if (valid && hl == 0) {
            const int t = (int)(r / P.hq), h = (int)(r % P.hq);
            const size_t i = (size_t)h * P.T + t;
            rs[i] = make_float2(lse[i] * kLog2e, acc - (dlse ? dlse[i] : 0.f));
        }
    }
}

// ---------------------------------------------------------------------------------------
// dK, dV

constexpr int kQRows = 64;   // query rows per tile of the dK/dV stream (MMA N)
constexpr int kStages = 3;   // ring of (Q, dO, row info) tiles
static_assert(kStages == 3, "one dK/dV gather warp per ring stage (warps 8, 10 and 11)");

struct RowInfo {
    float lse2;  // lse * log2 e
    float dp;    // <dO, out> - dlse
    int tok;     // last key the row may see (INT_MAX for routed rows), -1 = no row
    int pad;
};

template <int D>
struct DkdvSmem {
    static constexpr int kKV = kTileM * D * 2;     // K or V tile, 128 keys
    static constexpr int kQT = kQRows * D * 2;     // Q or dO tile, 64 rows
    static constexpr int kK = 0, kV = kKV;
    static constexpr int kRing = 2 * kKV;          // stage s: Q at kRing + 2 s kQT, dO at + kQT
    static constexpr int kRows = kRing + kStages * 2 * kQT;
    static constexpr int kBars = kRows + kStages * kQRows * (int)sizeof(RowInfo);
    static constexpr int kNumBars = 16;
    static constexpr int kMisc = kBars + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16 + 1024;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ dout,
                const float2* __restrict__ rs, Problem P, Workspace ws,
                __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv) {
    using L = DkdvSmem<D>;
    constexpr int kHalfKV = kTileM * 128;   // [128 keys x 64] swizzled half of a K / V tile
    constexpr int kHalfQ = kQRows * 128;    // [64 rows x 64] swizzled half of a Q / dO tile
    constexpr uint32_t kIdescS = idesc_bf16(kQRows, false);
    constexpr uint32_t kIdescKV = idesc_bf16(D, true);
    constexpr uint32_t kColDV = 256, kColDK = 256 + D;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    RowInfo* rinfo = reinterpret_cast<RowInfo*>(smem + L::kRows);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    const uint32_t sm_base = smem_u32(smem);
    const uint32_t bar0 = sm_base + L::kBars;
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    constexpr int B_KV = 0, B_FULL = 1, B_EMPTY = B_FULL + kStages, B_SFULL = B_EMPTY + kStages,
                  B_PREADY = B_SFULL + 2, B_FINAL = B_PREADY + 2;
    static_assert(B_FINAL < L::kNumBars, "barrier area too small");

    // the item: KV head g, block b, key tile kt
    const int nkt = P.chunk / kTileM;
    int idx = blockIdx.x;
    const int kt = idx % nkt;
    idx /= nkt;
    const int b = idx % P.nb_cap;
    const int g = idx / P.nb_cap;
    if (b >= ws.hdr->nb_total) return;
    const int len = ws.blk_len[b];
    if (kt * kTileM >= len) return;
    const int bstart = ws.blk_start[b];
    const int ks = bstart + kt * kTileM;
    const int ke = bstart + min(len, (kt + 1) * kTileM);
    const int list = g * P.nb_cap + b;
    const int cnt = ws.counts[list], off = ws.offsets[list];
    const int n_hist = (cnt + kQRows - 1) / kQRows;
    const int n_cur_h = (len - kt * kTileM + kQRows - 1) / kQRows;  // own-block tiles per head
    const int n_tiles = n_hist + P.group * n_cur_h;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int* status = &ws.hdr->status;

    if (threadIdx.x == 0) {
        mbar_init(BAR(B_KV), 1);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(BAR(B_FULL + i), 32);  // the gather warp of the tile
            mbar_init(BAR(B_EMPTY + i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(BAR(B_SFULL + i), 1);
            mbar_init(BAR(B_PREADY + i), 256);
        }
        mbar_init(BAR(B_FINAL), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 9) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                         smem_u32(tmem_slot)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // Row r (0..63) of tile i of the stream: its (token, head) and causal limit.
    auto row_of = [&](int i, int r, int& t, int& h, int& tok) -> bool {
        if (i < n_hist) {
            const int e = i * kQRows + r;
            if (e >= cnt) return false;
            const int row = ws.entries[off + e] / P.topk;  // one wave from token 0: t * Hq + h
            t = row / P.hq;
            h = row - t * P.hq;
            tok = INT_MAX;
            return true;
        }
        const int ci = i - n_hist;
        const int hh = ci / n_cur_h, hi = ci - hh * n_cur_h;
        const int lr = kt * kTileM + hi * kQRows + r;
        if (lr >= len) return false;
        t = bstart + lr;
        h = g * P.group + hh;
        tok = t;
        return true;
    };
    // cp.async gather of the 64 rows of tile i, Q and dO, into [64 x D] K-major SW128 tiles at
    // q_tile and q_tile + kQT, with the rows' statistics (one warp; each row is resolved once)
    auto gather = [&](uint32_t q_tile, int i) {
        constexpr int CK = D / 8;
#pragma unroll 1
        for (int r = lane; r < kQRows; r += 32) {
            int t = 0, h = 0, tok = -1;
            const bool valid = row_of(i, r, t, h, tok);
            const long long ro = valid ? ((long long)t * P.hq + h) * D : 0;
            const uint32_t rbase = q_tile + (uint32_t)r * 128u;
#pragma unroll
            for (int cc = 0; cc < CK; ++cc) {
                const uint32_t dst = rbase + (uint32_t)(cc >> 3) * kHalfQ + (uint32_t)(((cc & 7) ^ (r & 7)) << 4);
                cp_async16(dst, q + ro + (valid ? cc * 8 : 0), valid);
                cp_async16(dst + (uint32_t)L::kQT, dout + ro + (valid ? cc * 8 : 0), valid);
            }
            RowInfo ri;
            if (valid) {
                const float2 st = rs[(size_t)h * P.T + t];
                ri.lse2 = st.x;
                ri.dp = st.y;
                ri.tok = tok;
            } else {
                ri.lse2 = 0.f;
                ri.dp = 0.f;
                ri.tok = -1;
            }
            ri.pad = 0;
            rinfo[(i % kStages) * kQRows + r] = ri;
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        fence_proxy_async();
    };

    if (warp >= 8) {
        if (warp == 8 || warp == 10 || warp == 11) {
            // ---------------- K / V tile (warp 10, once) and the Q / dO row stream ----------------
            // three gather warps, one per ring stage: warp 8 takes tiles 0, 3, 6, ..., warp 10
            // tiles 1, 4, ..., warp 11 tiles 2, 5, ...
            if (warp == 10) {
                if (lane == 0) {
                    mbar_arrive_tx(BAR(B_KV), 2u * L::kKV);
#pragma unroll
                    for (int hh = 0; hh < D / 64; ++hh) {
                        tma_load_3d(sm_base + L::kK + hh * kHalfKV, &tmap_k, BAR(B_KV), hh * 64, g, ks);
                        tma_load_3d(sm_base + L::kV + hh * kHalfKV, &tmap_v, BAR(B_KV), hh * 64, g, ks);
                    }
                }
                __syncwarp();
            }
            const int first = warp == 8 ? 0 : (warp == 10 ? 1 : 2);
            for (int i = first; i < n_tiles; i += kStages) {
                const int s = i % kStages;
                if (i >= kStages &&
                    !wait_bar(BAR(B_EMPTY + s), (uint32_t)((i / kStages) - 1) & 1u, abort_flag, status))
                    break;
                gather(sm_base + L::kRing + (uint32_t)s * 2u * L::kQT, i);
                mbar_arrive(BAR(B_FULL + s));
            }
            if (warp == 10) drain_bar(BAR(B_KV), 0);  // the K / V tile must land before the CTA exits
        } else if (warp == 9) {
            // ---------------- MMA issuer (one thread) ----------------
            if (lane == 0) {
                bool ok = wait_bar1(BAR(B_KV), 0u, abort_flag, status);
                auto kdesc = [&](int kk, uint32_t base) {
                    return smem_desc(base + (uint32_t)(kk >> 2) * kHalfKV + (uint32_t)(kk & 3) * 32u, 16, 1024);
                };
                auto qdesc = [&](int kk, uint32_t base) {
                    return smem_desc(base + (uint32_t)(kk >> 2) * kHalfQ + (uint32_t)(kk & 3) * 32u, 16, 1024);
                };
                auto issue_sdp = [&](int i) {
                    const int s = i % kStages;
                    const uint32_t bb = (uint32_t)(i & 1);
                    const uint32_t qt = sm_base + L::kRing + (uint32_t)s * 2u * L::kQT;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        mma_ss(tmem + 128u * bb, kdesc(kk, sm_base + L::kK), qdesc(kk, qt), kIdescS, kk > 0 ? 1u : 0u);
                        mma_ss(tmem + 128u * bb + 64u, kdesc(kk, sm_base + L::kV), qdesc(kk, qt + L::kQT), kIdescS,
                               kk > 0 ? 1u : 0u);
                    }
                    mma_commit(BAR(B_SFULL + (int)bb));
                };
                auto issue_dkv = [&](int i) {
                    const int s = i % kStages;
                    const uint32_t bb = (uint32_t)(i & 1);
                    const uint32_t qt = sm_base + L::kRing + (uint32_t)s * 2u * L::kQT;
#pragma unroll
                    for (int kk = 0; kk < kQRows / 16; ++kk) {
                        // P^T / dS^T of rows 16kk..16kk+15: packed columns of the row half kk / 2
                        const uint32_t acol = (uint32_t)(kk >> 1) * 32u + (uint32_t)(kk & 1) * 8u;
                        const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
                        mma_ts(tmem + kColDV, tmem + 128u * bb + acol,
                               smem_desc(qt + L::kQT + (uint32_t)kk * 2048u, kHalfQ, 1024), kIdescKV, acc);
                        mma_ts(tmem + kColDK, tmem + 128u * bb + 64u + acol,
                               smem_desc(qt + (uint32_t)kk * 2048u, kHalfQ, 1024), kIdescKV, acc);
                    }
                    mma_commit(BAR(B_EMPTY + s));
                };
                if (ok && n_tiles > 0) {
                    ok = wait_bar1(BAR(B_FULL), 0u, abort_flag, status);
                    if (ok) {
                        tc_fence_after();
                        issue_sdp(0);
                    }
                }
                for (int i = 0; ok && i < n_tiles; ++i) {
                    if (i + 1 < n_tiles) {
                        const int s1 = (i + 1) % kStages;
                        if (!wait_bar1(BAR(B_FULL + s1), (uint32_t)((i + 1) / kStages) & 1u, abort_flag, status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_sdp(i + 1);
                    }
                    if (!wait_bar1(BAR(B_PREADY + (i & 1)), (uint32_t)(i >> 1) & 1u, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_dkv(i);
                }
                mma_commit(BAR(B_FINAL));
                drain_bar(BAR(B_FINAL), 0);
            }
            __syncwarp();
        }
    } else {
        // ---------------- P^T, dS^T (thread = key), then the dK / dV epilogue ----------------
        const int wg = warp >> 2, quad = warp & 3;
        const int key = ks + quad * 32 + lane;
        const bool key_ok = key < ke;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const float sl2 = P.scale_log2;
        bool ok = true;
        for (int i = 0; i < n_tiles; ++i) {
            const uint32_t bb = (uint32_t)(i & 1);
            // the row statistics of stage i % kStages come from the gather warp: acquire them
            // from its FULL arrival (the slot cannot turn over before this tile's PREADY)
            if (!wait_bar(BAR(B_FULL + i % kStages), (uint32_t)(i / kStages) & 1u, abort_flag, status) ||
                !wait_bar(BAR(B_SFULL + (int)bb), (uint32_t)(i >> 1) & 1u, abort_flag, status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sr[32], dr[32];
            const uint32_t scol = tmem + lane_off + 128u * bb + 32u * (uint32_t)wg;
            tmem_ld32_nowait(scol, sr);
            tmem_ld32_nowait(scol + 64u, dr);
            tmem_ld_wait();
            const RowInfo* ri = rinfo + (i % kStages) * kQRows + 32 * wg;
            uint32_t pw[16], dw[16];
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                const RowInfo r0 = ri[j], r1 = ri[j + 1];
                const float s0 = __uint_as_float(sr[j]), s1 = __uint_as_float(sr[j + 1]);
                const float e0 = ex2(fmaf(s0, sl2, -r0.lse2)), e1 = ex2(fmaf(s1, sl2, -r1.lse2));
                const float p0 = (key_ok && r0.tok >= key) ? e0 : 0.f;
                const float p1 = (key_ok && r1.tok >= key) ? e1 : 0.f;
                const float d0 = p0 * (__uint_as_float(dr[j]) - r0.dp);
                const float d1 = p1 * (__uint_as_float(dr[j + 1]) - r1.dp);
                pw[j >> 1] = pack_bf16(p0, p1);
                dw[j >> 1] = pack_bf16(d0, d1);
            }
            tmem_st16(scol, pw);         // P^T over the S^T columns this warp has read
            tmem_st16(scol + 64u, dw);   // dS^T over the dP^T columns this warp has read
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(BAR(B_PREADY + (int)bb));
        }
        if (ok && wait_bar(BAR(B_FINAL), 0u, abort_flag, status)) {
            tc_fence_after();
            // warpgroup 0 writes dV, warpgroup 1 writes scale * dK
            const float mul = wg ? P.scale : 1.f;
            __nv_bfloat16* dst = (wg ? dk : dv) + ((size_t)key * P.hkv + g) * D;
#pragma unroll
            for (int j = 0; j < D / 32; ++j) {
                float v[32];
                if (n_tiles > 0) {
                    tmem_ld32(tmem + lane_off + (wg ? kColDK : kColDV) + 32u * j, v);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = 0.f;
                }
                if (key_ok) {
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        const uint4 w = make_uint4(pack_bf16(v[e] * mul, v[e + 1] * mul), pack_bf16(v[e + 2] * mul, v[e + 3] * mul),
                                                   pack_bf16(v[e + 4] * mul, v[e + 5] * mul), pack_bf16(v[e + 6] * mul, v[e + 7] * mul));
                        *reinterpret_cast<uint4*>(dst + 32 * j + e) = w;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
    }
}

// ---------------------------------------------------------------------------------------
// dQ

constexpr int kBN = 64;       // keys per chunk of the dQ kernel (MMA N)
constexpr int kKVStages = 3;  // ring of (K chunk, V chunk)

struct DqSlot {
    int kind;  // -1 = no more work
    int ntiles;
    int g;     // KV head
    int key_start[2], key_end[2], nchunks[2];
    int rowoff[kItemRows];  // t * Hq + h of each row, -1 = no row
    int tok[kItemRows];     // last key the row may see (INT_MAX for routed rows)
    float lse2[kItemRows];
    float dp[kItemRows];
};

template <int D>
struct DqSmem {
    static constexpr int kTile = kTileM * D * 2;   // Q or dO tile, 128 rows
    static constexpr int kChunk = kBN * D * 2;     // K or V chunk, 64 keys
    static constexpr int kQ = 0, kDO = kTile;
    static constexpr int kKV = 2 * kTile;          // stage s: K at kKV + 2 s kChunk, V at + kChunk
    static constexpr int kSlots = kKV + kKVStages * 2 * kChunk;
    static constexpr int kBars = kSlots + 2 * (int)sizeof(DqSlot);
    static constexpr int kNumBars = 24;
    static constexpr int kMisc = kBars + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16 + 1024;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
bwd_dq_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
              const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ dout,
              const float2* __restrict__ rs, Problem P, Workspace ws, float* __restrict__ dq_acc) {
    using L = DqSmem<D>;
    constexpr int kHalfT = kTileM * 128;   // [128 rows x 64] swizzled half of a Q / dO tile
    constexpr int kHalfC = kBN * 128;      // [64 keys x 64] swizzled half of a K / V chunk
    constexpr uint32_t kIdescS = idesc_bf16(kBN, false);
    constexpr uint32_t kIdescDQ = idesc_bf16(D, true);
    constexpr uint32_t kColDQ = 256;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    DqSlot* slots = reinterpret_cast<DqSlot*>(smem + L::kSlots);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    const uint32_t sm_base = smem_u32(smem);
    const uint32_t bar0 = sm_base + L::kBars;
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    constexpr int B_INFO = 0, B_ITEM_EMPTY = 2, B_QFULL = 4, B_QEMPTY = 5, B_KV_FULL = 6,
                  B_KV_EMPTY = B_KV_FULL + kKVStages, B_SFULL = B_KV_EMPTY + kKVStages,
                  B_PREADY = B_SFULL + 2, B_DQFULL = B_PREADY + 2, B_DQEMPTY = B_DQFULL + 1,
                  B_FINAL = B_DQEMPTY + 1;
    static_assert(B_FINAL < L::kNumBars, "barrier area too small");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int* status = &ws.hdr->status;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(BAR(B_INFO + i), 32);
            mbar_init(BAR(B_ITEM_EMPTY + i), 256 + 32);  // softmax threads + the dO gather warp
            mbar_init(BAR(B_SFULL + i), 1);
            mbar_init(BAR(B_PREADY + i), 256);
        }
        mbar_init(BAR(B_QFULL), 64);
        mbar_init(BAR(B_QEMPTY), 1);
        for (int i = 0; i < kKVStages; ++i) {
            mbar_init(BAR(B_KV_FULL + i), 1);
            mbar_init(BAR(B_KV_EMPTY + i), 1);
        }
        mbar_init(BAR(B_DQFULL), 1);
        mbar_init(BAR(B_DQEMPTY), 256);
        mbar_init(BAR(B_FINAL), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 9) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                         smem_u32(tmem_slot)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // cp.async gather of the 128 rows of tile u of an item into a K-major SW128 tile (one warp)
    auto gather = [&](const __nv_bfloat16* src_base, uint32_t dst_tile, const DqSlot& sl, int u) {
        constexpr int CK = D / 8;
#pragma unroll 1
        for (int r = lane; r < kTileM; r += 32) {
            const int ro = sl.rowoff[u * kTileM + r];
            const bool valid = ro >= 0;
            const __nv_bfloat16* src = valid ? src_base + (long long)ro * D : src_base;
            const uint32_t rbase = dst_tile + (uint32_t)r * 128u;
#pragma unroll
            for (int cc = 0; cc < CK; ++cc) {
                const uint32_t dst = rbase + (uint32_t)(cc >> 3) * kHalfT + (uint32_t)(((cc & 7) ^ (r & 7)) << 4);
                cp_async16(dst, src + (valid ? cc * 8 : 0), valid);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        fence_proxy_async();
    };

    if (warp >= 8) {
        if (warp == 8) {
            // ---------------- item fetch, row table and the Q gather ----------------
            const int n_items = ws.hdr->n_items;
            uint32_t tiles = 0;  // tiles gathered so far (Q buffer phase)
            for (int it = 0;; ++it) {
                const int s = it & 1;
                if (it >= 2 && !wait_bar(BAR(B_ITEM_EMPTY + s), (uint32_t)((it >> 1) - 1) & 1u, abort_flag, status)) break;
                int idx = 0;
                if (lane == 0) idx = (int)atomicAdd(&ws.hdr->work_counter, 1u);
                idx = __shfl_sync(0xffffffffu, idx, 0);
                DqSlot& sl = slots[s];
                if (idx >= n_items) {
                    if (lane == 0) sl.kind = -1;
                    __syncwarp();
                    mbar_arrive(BAR(B_INFO + s));
                    break;
                }
                const WorkItem w = ws.items[idx];
                int ntiles;
                if (w.kind == 0) {
                    const int g = w.a / P.nb_cap, b = w.a - g * P.nb_cap;
                    const int kstart = ws.blk_start[b], klen = ws.blk_len[b];
                    ntiles = w.c > kTileM ? 2 : 1;
                    for (int r = lane; r < kItemRows; r += 32) {
                        int ro = -1;
                        if (r < w.c) ro = ws.entries[w.b + r] / P.topk;  // t * Hq + h
                        sl.rowoff[r] = ro;
                        sl.tok[r] = INT_MAX;
                        const float2 st = ro >= 0 ? rs[(size_t)(ro % P.hq) * P.T + ro / P.hq] : make_float2(0.f, 0.f);
                        sl.lse2[r] = st.x;
                        sl.dp[r] = st.y;
                    }
                    if (lane == 0) {
                        for (int u = 0; u < 2; ++u) {
                            sl.key_start[u] = kstart;
                            sl.key_end[u] = kstart + klen;
                            sl.nchunks[u] = (klen + kBN - 1) / kBN;
                        }
                    }
                } else {
                    const int b = w.a;
                    const int kstart = ws.blk_start[b], klen = ws.blk_len[b];
                    int h0 = w.b, h1 = w.b, qt0 = w.c, qt1 = w.c;
                    ntiles = 1;
                    if (w.kind == 2) {
                        h1 = h0 + 1;
                        ntiles = 2;
                    } else if (w.kind == 3) {
                        qt0 = (klen + kTileM - 1) / kTileM - 1 - w.c;
                        ntiles = 2;
                    }
                    for (int r = lane; r < kItemRows; r += 32) {
                        const int u = r / kTileM;
                        const int rr = (u ? qt1 : qt0) * kTileM + (r - u * kTileM);
                        const int tok = kstart + rr;
                        const bool okr = u < ntiles && rr < klen;
                        const int ro = okr ? tok * P.hq + (u ? h1 : h0) : -1;
                        sl.rowoff[r] = ro;
                        sl.tok[r] = okr ? tok : -1;
                        const float2 st = okr ? rs[(size_t)(u ? h1 : h0) * P.T + tok] : make_float2(0.f, 0.f);
                        sl.lse2[r] = st.x;
                        sl.dp[r] = st.y;
                    }
                    if (lane == 0) {
                        for (int u = 0; u < 2; ++u) {
                            const int qt = u ? qt1 : qt0;
                            const int kend = kstart + min((qt + 1) * kTileM, klen);
                            sl.key_start[u] = kstart;
                            sl.key_end[u] = kend;
                            sl.nchunks[u] = (kend - kstart + kBN - 1) / kBN;
                        }
                    }
                }
                if (lane == 0) {
                    sl.kind = w.kind;
                    sl.ntiles = ntiles;
                    sl.g = (w.kind == 0) ? w.a / P.nb_cap : w.b / P.group;
                }
                __syncwarp();
                mbar_arrive(BAR(B_INFO + s));
                bool okq = true;
                for (int u = 0; u < ntiles; ++u, ++tiles) {
                    if (tiles > 0 && !wait_bar(BAR(B_QEMPTY), (tiles - 1u) & 1u, abort_flag, status)) {
                        okq = false;
                        break;
                    }
                    gather(q, sm_base + L::kQ, sl, u);
                    mbar_arrive(BAR(B_QFULL));
                }
                if (!okq) break;
            }
        } else if (warp == 11) {
            // ---------------- dO gather ----------------
            uint32_t tiles = 0;
            bool okd = true;
            for (int it = 0; okd; ++it) {
                const int s = it & 1;
                if (!wait_bar(BAR(B_INFO + s), (uint32_t)(it >> 1) & 1u, abort_flag, status)) break;
                const DqSlot& sl = slots[s];
                if (sl.kind < 0) break;
                for (int u = 0; u < sl.ntiles; ++u, ++tiles) {
                    if (tiles > 0 && !wait_bar(BAR(B_QEMPTY), (tiles - 1u) & 1u, abort_flag, status)) {
                        okd = false;
                        break;
                    }
                    gather(dout, sm_base + L::kDO, sl, u);
                    mbar_arrive(BAR(B_QFULL));
                }
                mbar_arrive(BAR(B_ITEM_EMPTY + s));
            }
        } else if (warp == 10) {
            // ---------------- K / V chunk producer (TMA) ----------------
            uint32_t c = 0;  // chunks issued so far
            bool okp = true;
            for (int it = 0; okp; ++it) {
                const int s = it & 1;
                if (!wait_bar(BAR(B_INFO + s), (uint32_t)(it >> 1) & 1u, abort_flag, status)) break;
                const DqSlot& sl = slots[s];
                if (sl.kind < 0) break;
                const int ntiles = sl.ntiles;
                const int g = sl.g;
                for (int u = 0; okp && u < ntiles; ++u) {
                    const int kstart = sl.key_start[u], N = sl.nchunks[u];
                    for (int n = 0; n < N; ++n, ++c) {
                        const uint32_t st = c % kKVStages;
                        if (c >= kKVStages &&
                            !wait_bar(BAR(B_KV_EMPTY + st), ((c / kKVStages) - 1u) & 1u, abort_flag, status)) {
                            okp = false;
                            break;
                        }
                        if (lane == 0) {
                            const uint32_t dst = sm_base + L::kKV + st * 2u * L::kChunk;
                            mbar_arrive_tx(BAR(B_KV_FULL + st), 2u * L::kChunk);
#pragma unroll
                            for (int hh = 0; hh < D / 64; ++hh) {
                                tma_load_3d(dst + hh * kHalfC, &tmap_k, BAR(B_KV_FULL + st), hh * 64, g, kstart + n * kBN);
                                tma_load_3d(dst + L::kChunk + hh * kHalfC, &tmap_v, BAR(B_KV_FULL + st), hh * 64, g,
                                            kstart + n * kBN);
                            }
                        }
                        __syncwarp();
                    }
                }
            }
            const uint32_t issued = c;
            for (uint32_t k = (issued > kKVStages ? issued - kKVStages : 0); k < issued; ++k)
                drain_bar(BAR(B_KV_FULL + k % kKVStages), (k / kKVStages) & 1u);
        } else {
            // ---------------- MMA issuer (warp 9, one thread) ----------------
            if (lane == 0) {
                uint32_t cc = 0, tiles = 0;
                bool ok = true;
                auto tdesc = [&](int kk, uint32_t base) {
                    return smem_desc(base + (uint32_t)(kk >> 2) * kHalfT + (uint32_t)(kk & 3) * 32u, 16, 1024);
                };
                auto cdesc = [&](int kk, uint32_t base) {
                    return smem_desc(base + (uint32_t)(kk >> 2) * kHalfC + (uint32_t)(kk & 3) * 32u, 16, 1024);
                };
                for (int it = 0; ok; ++it) {
                    const int s = it & 1;
                    if (!wait_bar1(BAR(B_INFO + s), (uint32_t)(it >> 1) & 1u, abort_flag, status)) break;
                    const DqSlot& sl = slots[s];
                    if (sl.kind < 0) break;
                    const int ntiles = sl.ntiles;
                    for (int u = 0; ok && u < ntiles; ++u) {
                        const int N = sl.nchunks[u];
                        if (!wait_bar1(BAR(B_QFULL), tiles & 1u, abort_flag, status)) {
                            ok = false;
                            break;
                        }
                        for (int n = 0; n <= N; ++n) {
                            if (n < N) {
                                const uint32_t c = cc + (uint32_t)n, st = c % kKVStages, bb = c & 1u;
                                if (!wait_bar1(BAR(B_KV_FULL + st), (c / kKVStages) & 1u, abort_flag, status)) {
                                    ok = false;
                                    break;
                                }
                                tc_fence_after();
                                const uint32_t kb = sm_base + L::kKV + st * 2u * L::kChunk;
#pragma unroll
                                for (int kk = 0; kk < D / 16; ++kk) {
                                    mma_ss(tmem + 128u * bb, tdesc(kk, sm_base + L::kQ), cdesc(kk, kb), kIdescS,
                                           kk > 0 ? 1u : 0u);
                                    mma_ss(tmem + 128u * bb + 64u, tdesc(kk, sm_base + L::kDO), cdesc(kk, kb + L::kChunk),
                                           kIdescS, kk > 0 ? 1u : 0u);
                                }
                                mma_commit(BAR(B_SFULL + (int)bb));
                                if (n == N - 1) mma_commit(BAR(B_QEMPTY));
                            }
                            if (n >= 1) {
                                const uint32_t c1 = cc + (uint32_t)(n - 1), st1 = c1 % kKVStages, bb1 = c1 & 1u;
                                if (!wait_bar1(BAR(B_PREADY + (int)bb1), (c1 >> 1) & 1u, abort_flag, status)) {
                                    ok = false;
                                    break;
                                }
                                if (n == 1 && tiles > 0 &&
                                    !wait_bar1(BAR(B_DQEMPTY), (tiles - 1u) & 1u, abort_flag, status)) {
                                    ok = false;
                                    break;
                                }
                                tc_fence_after();
                                const uint32_t kb = sm_base + L::kKV + st1 * 2u * L::kChunk;
#pragma unroll
                                for (int kk = 0; kk < kBN / 16; ++kk) {
                                    // dS of keys 16kk..16kk+15: packed columns of the key half kk / 2
                                    const uint32_t acol = (uint32_t)(kk >> 1) * 32u + (uint32_t)(kk & 1) * 8u;
                                    mma_ts(tmem + kColDQ, tmem + 128u * bb1 + acol,
                                           smem_desc(kb + (uint32_t)kk * 2048u, kHalfC, 1024), kIdescDQ,
                                           (n > 1 || kk > 0) ? 1u : 0u);
                                }
                                mma_commit(BAR(B_KV_EMPTY + (int)st1));
                            }
                        }
                        if (!ok) break;
                        mma_commit(BAR(B_DQFULL));
                        cc += (uint32_t)N;
                        ++tiles;
                    }
                }
                mma_commit(BAR(B_FINAL));
                drain_bar(BAR(B_FINAL), 0);
            }
            __syncwarp();
        }
    } else {
        // ---------------- dS (thread = row), then the dQ epilogue ----------------
        const int wg = warp >> 2, quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const float sl2 = P.scale_log2;
        uint32_t cc = 0, tiles = 0;
        bool ok = true;
        for (int it = 0; ok; ++it) {
            const int s = it & 1;
            if (!wait_bar(BAR(B_INFO + s), (uint32_t)(it >> 1) & 1u, abort_flag, status)) break;
            const DqSlot& sl = slots[s];
            if (sl.kind < 0) break;
            const int ntiles = sl.ntiles;
            for (int u = 0; u < ntiles; ++u) {
                const int ro = sl.rowoff[u * kTileM + row];
                const int tok = sl.tok[u * kTileM + row];
                const float lse2 = sl.lse2[u * kTileM + row], dpr = sl.dp[u * kTileM + row];
                const int N = sl.nchunks[u], kstart = sl.key_start[u], kend = sl.key_end[u];
                const int lim = min(kend - 1, tok);  // last key the row sees
                for (int n = 0; n < N; ++n) {
                    const uint32_t c = cc + (uint32_t)n, bb = c & 1u;
                    if (!wait_bar(BAR(B_SFULL + (int)bb), (c >> 1) & 1u, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint32_t sr[32], dr[32];
                    const uint32_t scol = tmem + lane_off + 128u * bb + 32u * (uint32_t)wg;
                    tmem_ld32_nowait(scol, sr);
                    tmem_ld32_nowait(scol + 64u, dr);
                    tmem_ld_wait();
                    const int k0 = kstart + n * kBN + 32 * wg;
                    uint32_t dw[16];
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        const float e0 = ex2(fmaf(__uint_as_float(sr[j]), sl2, -lse2));
                        const float e1 = ex2(fmaf(__uint_as_float(sr[j + 1]), sl2, -lse2));
                        const float p0 = (ro >= 0 && k0 + j <= lim) ? e0 : 0.f;
                        const float p1 = (ro >= 0 && k0 + j + 1 <= lim) ? e1 : 0.f;
                        dw[j >> 1] = pack_bf16(p0 * (__uint_as_float(dr[j]) - dpr),
                                               p1 * (__uint_as_float(dr[j + 1]) - dpr));
                    }
                    tmem_st16(scol, dw);  // dS over the S columns this warp has read
                    tmem_st_wait();
                    tc_fence_before();
                    mbar_arrive(BAR(B_PREADY + (int)bb));
                }
                if (!ok) break;
                cc += (uint32_t)N;
                // epilogue: scale * dQ of this row added to the fp32 accumulator
                if (!wait_bar(BAR(B_DQFULL), tiles & 1u, abort_flag, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int j = 0; j < D / 64; ++j) {
                    const int col = wg * (D / 2) + 32 * j;
                    float v[32];
                    tmem_ld32(tmem + lane_off + kColDQ + (uint32_t)col, v);
                    if (ro >= 0) {
                        float* dst = dq_acc + (size_t)ro * D + col;
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            red_add_v4(dst + e, v[e] * P.scale, v[e + 1] * P.scale, v[e + 2] * P.scale,
                                       v[e + 3] * P.scale);
                    }
                }
                tc_fence_before();
                mbar_arrive(BAR(B_DQEMPTY));
                ++tiles;
            }
            if (!ok) break;
            mbar_arrive(BAR(B_ITEM_EMPTY + s));
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
    }
}

// fp32 accumulator -> bf16 dq, 8 values per thread.
__global__ void __launch_bounds__(256)
bwd_dq_convert_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq, long long n8) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
         i += (long long)gridDim.x * blockDim.x) {
        const float4 a = __ldcs(reinterpret_cast<const float4*>(acc) + 2 * i);
        const float4 b = __ldcs(reinterpret_cast<const float4*>(acc) + 2 * i + 1);
        reinterpret_cast<uint4*>(dq)[i] =
            make_uint4(pack_bf16(a.x, a.y), pack_bf16(a.z, a.w), pack_bf16(b.x, b.y), pack_bf16(b.z, b.w));
    }
}

// ---------------------------------------------------------------------------------------
// Host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [T, Hkv, d] bf16 as a 3-D tensor (d, Hkv, T); box (64, 1, rows) with 128-byte swizzle.
cudaError_t make_map(CUtensorMap* m, const void* base, const Problem& P, int rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    cuuint64_t dims[3] = {(cuuint64_t)P.d, (cuuint64_t)P.hkv, (cuuint64_t)P.T};
    cuuint64_t strides[2] = {(cuuint64_t)P.d * 2, (cuuint64_t)P.hkv * P.d * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)rows};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D>
cudaError_t launch_bwd_d(const Problem& P, const BwdArgs& a, const Workspace& ws, int num_sms,
                         cudaStream_t st, int* launches) {
    const long long rows = (long long)P.T * P.hq;
    {
        long long grid = (rows + 15) / 16;
        if (grid > 148 * 32) grid = 148 * 32;
        bwd_rowstats_kernel<D><<<(int)(grid < 1 ? 1 : grid), 256, 0, st>>>(a.out, a.dout, a.lse, a.dlse, P, a.rs);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        ++*launches;
    }
    CUtensorMap mk128, mv128, mk64, mv64;
    cudaError_t e = make_map(&mk128, a.k, P, kTileM);
    if (e == cudaSuccess) e = make_map(&mv128, a.v, P, kTileM);
    if (e == cudaSuccess) e = make_map(&mk64, a.k, P, kBN);
    if (e == cudaSuccess) e = make_map(&mv64, a.v, P, kBN);
    if (e != cudaSuccess) return e;
    {
        const int smem = DkdvSmem<D>::kBytes;
        e = cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        const long long grid = (long long)P.hkv * P.nb_cap * (P.chunk / kTileM);
        bwd_dkdv_kernel<D><<<(unsigned)grid, kThreads, smem, st>>>(mk128, mv128, a.q, a.dout, a.rs, P, ws, a.dk, a.dv);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        ++*launches;
    }
    {
        const int smem = DqSmem<D>::kBytes;
        e = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        bwd_dq_kernel<D><<<num_sms, kThreads, smem, st>>>(mk64, mv64, a.q, a.dout, a.rs, P, ws, a.dq_acc);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        ++*launches;
    }
    {
        const long long n8 = rows * P.d / 8;
        long long grid = (n8 + 255) / 256;
        if (grid > 148 * 64) grid = 148 * 64;
        bwd_dq_convert_kernel<<<(int)(grid < 1 ? 1 : grid), 256, 0, st>>>(a.dq_acc, a.dq, n8);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        ++*launches;
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_backward(const Problem& P, const BwdArgs& a, const Workspace& ws, int num_sms,
                            cudaStream_t st, int* launches) {
    if (P.d == 64) return launch_bwd_d<64>(P, a, ws, num_sms, st, launches);
    return launch_bwd_d<128>(P, a, ws, num_sms, st, launches);
}

}  // namespace moba
