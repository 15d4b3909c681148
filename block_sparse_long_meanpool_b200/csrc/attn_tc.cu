// Step 5 of the forward on the 5th-generation tensor cores (tcgen05 + TMEM + TMA), sm_100a.
//
// The analysis page of the MoBA paper (§3.2): history blocks are attended without a causal
// mask (rule 1 of §2.3 already excluded every future block), the own block with a causal
// mask, and the partial softmax results are merged afterwards by their log-sum-exp.
//
// Work items (from the routing pass) hold up to two 128-row query tiles against one KV range
// of one KV head: a history item is up to 256 routed rows (any query heads of that KV head)
// against one whole block; a current-block item is one or two 128-token query tiles (two heads
// of that KV head, or two tiles of one head) against the causal prefix of their block.  Every
// K/V chunk loaded into shared memory serves both tiles (a shorter tile stops early).  One
// persistent CTA per SM takes items from an atomic cursor.
//
// Warp roles (384 threads; setmaxnreg gives the softmax warps 192 registers, enough to hold a
// whole 128-score row, and the other warpgroup 120):
//   warps 0-3   softmax + epilogue of tile 0, thread r owns row r (TMEM lane r)
//   warps 4-7   softmax + epilogue of tile 1
//   warp 8      item fetch + Q gather of tile 0 (cp.async into a swizzled K-major tile)
//   warp 9      TMEM owner and single-thread MMA issuer
//   warp 10     K/V producer: TMA (SWIZZLE_128B, no multicast) into a 2-slot ring
//   warp 11     Q gather of tile 1
// TMEM (512 columns): S_0, S_1 (128 each; P_t as bf16 pairs over the first 64 columns of S_t),
// O_0, O_1 (d each).  Per 128-key chunk n the MMA warp issues, tile by tile,
//   PV_t(n-1): O_t += P_t(n-1) V(n-1)   (TS MMA: A = P from TMEM, B = V MN-major in smem)
//   QK_t(n):   S_t  = Q_t K(n)^T        (SS MMA, fp32 accumulate)
// so the tensor core works on one tile while the other tile's softmax runs.  Each tile's
// PV_t(n-1) and QK_t(n) go out as one uninterrupted run of MMAs.  The tensor pipe drains
// whenever the issuing thread stops issuing (and a commit holds the thread until the queued
// MMAs are dispatched), so the run's operands come in one ring slot -- step n of an item
// loads K(n) and V(n-1) together, behind one barrier, two steps ahead -- and tile 1's waits
// are done while tile 0's MMAs are still queued, before tile 0's commits.  PV_t(n-1) is
// issued before QK_t(n), so the barrier announcing S_t(n) also guarantees that O_t holds every
// earlier PV and that no MMA touches O_t until P_t(n) is announced: the softmax may rescale O_t
// in between.  The softmax reads its row of S once (tcgen05.ld), takes the maximum with
// three-input max, computes p = 2^(s*scale*log2e - m) with packed two-lane FMAs and the SFU, and
// raises the running maximum m (rescaling O_t) only when it grows by more than 2^8.  The
// epilogue writes the normalised partial output as bf16 (with its fp32 log-sum-exp).
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
constexpr int kSlots = 2;      // K/V ring: step j of an item loads K(j) and V(j-1) into one slot
constexpr int kThreads = 384;  // 12 warps
constexpr int kWarpFetch = 8, kWarpMMA = 9, kWarpKV = 10, kWarpQ1 = 11;
constexpr int kRegsSoftmax = 192, kRegsOther = 120;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O is rescaled when max grows > 2^8

// launched with 65536 / 384 -> 168 registers per thread; the split must not exceed that
static_assert(8 * 32 * kRegsSoftmax + 4 * 32 * kRegsOther <= 168 * kThreads,
              "setmaxnreg split exceeds the registers the CTA is launched with");

struct ItemSlot {
    int kind;    // -1 = no more work
    int ntiles;  // 1 or 2
    int g, key_start, key_end;
    int nchunks;          // K/V chunks of the item (= n[0])
    int n[2];             // chunks of each tile (n[1] <= n[0]; 0 when tile 1 is idle)
    int pidx[kItemRows];  // partial-output index of each row (-1 = no row)
    int tlim[kItemRows];  // last key a row may see (current-block items), else INT_MAX
};

template <int D>
struct SmemLayout {
    static constexpr int kTileBytes = kTileM * D * 2;  // 128 rows of bf16 (Q tile, K or V chunk)
    static constexpr int kQ = 0;                       // Q_0, Q_1
    static constexpr int kKV = 2 * kTileBytes;         // kSlots x (K chunk, V chunk)
    static constexpr int kItems = kKV + kSlots * 2 * kTileBytes;
    static constexpr int kBars = kItems + 2 * (int)sizeof(ItemSlot);
    static constexpr int kNumBars = 26;
    static constexpr int kMisc = kBars + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16 + 1024;  // + slack for 1024-byte alignment
};

// One butterfly stage of a 4x4 transpose of uint4 elements across the 4 lanes of a lane group:
// lanes i and i^DIST exchange the element pairs whose index bit DIST differs from their lane
// bit.  After stages 2 and 1, lane i holds a[j] = original a[i] of lane j.
template <int DIST>
__device__ __forceinline__ void transpose4x4(uint4 (&a)[4], int lane) {
    const bool up = (lane & DIST) != 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (j & DIST) continue;
        const uint4 send = up ? a[j] : a[j | DIST];
        uint4 recv;
        recv.x = __shfl_xor_sync(0xffffffffu, send.x, DIST);
        recv.y = __shfl_xor_sync(0xffffffffu, send.y, DIST);
        recv.z = __shfl_xor_sync(0xffffffffu, send.z, DIST);
        recv.w = __shfl_xor_sync(0xffffffffu, send.w, DIST);
        if (up) a[j] = recv; else a[j | DIST] = recv;
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
               const __nv_bfloat16* __restrict__ q, Problem P, Workspace ws, int t0, int t1) {
    using L = SmemLayout<D>;
    constexpr int kHalves = D / 64;           // 128-byte swizzle atoms along d
    constexpr int kHalfBytes = kTileM * 128;  // one [128 rows x 64 bf16] swizzled half
    constexpr uint32_t kChunkBytes = kTileM * D * 2;
    constexpr int kKSteps = D / 16;           // QK^T k-steps (16 bf16 each)
    constexpr uint32_t kIdescQK = idesc_bf16(kBN, false);
    constexpr uint32_t kIdescPV = idesc_bf16(D, true);
    constexpr uint32_t kColO = 2 * kBN;       // TMEM: S_0 at 0, S_1 at 128, O_0, O_1 from 256
    constexpr uint32_t kTmemCols = 512;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    ItemSlot* slots = reinterpret_cast<ItemSlot*>(smem + L::kItems);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

    const uint32_t sm_base = smem_u32(smem);
    const uint32_t bar0 = sm_base + L::kBars;
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    constexpr int B_INFO = 0, B_ITEM_EMPTY = 2, B_QFULL = 4, B_QEMPTY = 6, B_KV_FULL = 8,
                  B_KV_EMPTY = B_KV_FULL + kSlots, B_SFULL = B_KV_EMPTY + kSlots,
                  B_PFULL = B_SFULL + 2, B_OFULL = B_PFULL + 2, B_OEMPTY = B_OFULL + 2,
                  B_FINAL = B_OEMPTY + 2;
    static_assert(B_FINAL < L::kNumBars, "barrier area too small");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int* status = &ws.hdr->status;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(BAR(B_INFO + i), 32);
            mbar_init(BAR(B_ITEM_EMPTY + i), 2 * kTileM + 32);  // softmax threads + warp 11
            mbar_init(BAR(B_SFULL + i), 1);
            mbar_init(BAR(B_PFULL + i), kTileM);
            mbar_init(BAR(B_OFULL + i), 1);
            mbar_init(BAR(B_OEMPTY + i), kTileM);
            mbar_init(BAR(B_QFULL + i), 32);
            mbar_init(BAR(B_QEMPTY + i), 1);
        }
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(BAR(B_KV_FULL + i), 1);
            mbar_init(BAR(B_KV_EMPTY + i), 1);
        }
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
    // Gathers the rows of tile t of an item into Q_t by cp.async (called by one whole warp);
    // a row's partial index encodes ((token - t0) * Hq + head) * topk + slot.
    auto gather_q = [&](const ItemSlot& sl, int t) {
        constexpr int CK = D / 8;  // 16-byte chunks per row
#pragma unroll 1
        for (int rr = lane; rr < kTileM; rr += 32) {
            const int pi = sl.pidx[t * kTileM + rr];
            const bool valid = pi >= 0;
            const __nv_bfloat16* src = valid ? q + ((long long)t0 * P.hq + pi / P.topk) * D : q;
            const uint32_t rbase = sm_base + L::kQ + (uint32_t)t * L::kTileBytes + (uint32_t)rr * 128u;
#pragma unroll
            for (int cc = 0; cc < CK; ++cc) {
                const uint32_t dst = rbase + (uint32_t)(cc >> 3) * kHalfBytes +
                                     (uint32_t)(((cc & 7) ^ (rr & 7)) << 4);
                cp_async16(dst, src + (valid ? cc * 8 : 0), valid);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        fence_proxy_async();
    };

    if (warp >= 8) {
        // loads and MMA issue: few registers
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
        if (warp == kWarpFetch) {
            // ---------------- item fetch + Q gather of tile 0 ----------------
            const int n_items = ws.hdr->n_items;
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
                int g, key_start, key_end, ntiles, n0, n1;
                if (w.kind == 0) {
                    g = w.a / P.nb_cap;
                    const int b = w.a - g * P.nb_cap;
                    key_start = ws.blk_start[b];
                    key_end = key_start + ws.blk_len[b];
                    ntiles = w.c > kTileM ? 2 : 1;
                    n0 = (key_end - key_start + kBN - 1) / kBN;
                    n1 = ntiles == 2 ? n0 : 0;
                    for (int r = lane; r < kItemRows; r += 32) {
                        sl.pidx[r] = (r < w.c) ? ws.entries[w.b + r] : -1;
                        sl.tlim[r] = INT_MAX;
                    }
                } else {
                    // tile 0 covers (head h0, query tile qt0), tile 1 (h1, qt1); qt0 >= qt1
                    const int b = w.a;
                    key_start = ws.blk_start[b];
                    const int len = ws.blk_len[b];
                    int h0 = w.b, h1 = w.b, qt0 = w.c, qt1 = w.c;
                    ntiles = 1;
                    if (w.kind == 2) {
                        h1 = h0 + 1;
                        ntiles = 2;
                    } else if (w.kind == 3) {
                        qt0 = (len + kTileM - 1) / kTileM - 1 - w.c;
                        ntiles = 2;
                    }
                    g = h0 / P.group;
                    key_end = key_start + min((qt0 + 1) * kTileM, len);
                    n0 = qt0 + 1;
                    n1 = ntiles == 2 ? qt1 + 1 : 0;
                    for (int r = lane; r < kItemRows; r += 32) {
                        const int tt = r / kTileM;
                        const int rr = (tt ? qt1 : qt0) * kTileM + (r - tt * kTileM);
                        const int tok = key_start + rr;
                        const bool ok = tt < ntiles && rr < len && tok >= t0 && tok < t1;
                        sl.pidx[r] = ok ? ((tok - t0) * P.hq + (tt ? h1 : h0)) * P.topk : -1;
                        sl.tlim[r] = ok ? tok : INT_MAX;
                    }
                }
                if (lane == 0) {
                    sl.kind = w.kind;
                    sl.ntiles = ntiles;
                    sl.g = g;
                    sl.key_start = key_start;
                    sl.key_end = key_end;
                    sl.nchunks = n0;
                    sl.n[0] = n0;
                    sl.n[1] = n1;
                }
                __syncwarp();
                mbar_arrive(BAR(B_INFO + s));
                // Q_0 is free once every QK^T of tile 0 of the previous item has completed
                if (it >= 1 && !wait_bar(BAR(B_QEMPTY), (uint32_t)(it - 1) & 1u, abort_flag, status)) break;
                gather_q(sl, 0);
                mbar_arrive(BAR(B_QFULL));
            }
        } else if (warp == kWarpQ1) {
            // ---------------- Q gather of tile 1 ----------------
            uint32_t uses1 = 0;  // earlier items with tile 1 active
            for (int it = 0;; ++it) {
                const int s = it & 1;
                if (!wait_bar(BAR(B_INFO + s), (uint32_t)(it >> 1) & 1u, abort_flag, status)) break;
                const ItemSlot& sl = slots[s];
                if (sl.kind < 0) break;
                if (sl.ntiles == 2) {
                    if (uses1 >= 1 && !wait_bar(BAR(B_QEMPTY + 1), (uses1 - 1u) & 1u, abort_flag, status)) break;
                    gather_q(sl, 1);
                    mbar_arrive(BAR(B_QFULL + 1));
                    ++uses1;
                }
                // the slot may be reused only after this warp is done with it
                mbar_arrive(BAR(B_ITEM_EMPTY + s));
            }
        } else if (warp == kWarpKV) {
            // ---------------- K/V producer (TMA) ----------------
            // step j = 0..N of an item fills ring slot (CTA step count) % 2 with K(j) (j < N)
            // and V(j-1) (j > 0): exactly the operands of the MMA runs of step j
            uint32_t c = 0;  // steps issued so far
            for (int it = 0;; ++it) {
                const int s = it & 1;
                if (!wait_bar(BAR(B_INFO + s), (uint32_t)(it >> 1) & 1u, abort_flag, status)) break;
                const ItemSlot& sl = slots[s];
                if (sl.kind < 0) break;
                const int g = sl.g, key_start = sl.key_start, N = sl.nchunks;
                bool ok = true;
                for (int j = 0; j <= N; ++j) {
                    const uint32_t st = c % kSlots;
                    if (c >= kSlots &&
                        !wait_bar(BAR(B_KV_EMPTY + st), ((c / kSlots) - 1u) & 1u, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        const uint32_t dst = sm_base + L::kKV + st * 2u * L::kTileBytes;
                        mbar_arrive_tx(BAR(B_KV_FULL + st),
                                       (j < N ? kChunkBytes : 0u) + (j > 0 ? kChunkBytes : 0u));
#pragma unroll
                        for (int hh = 0; hh < kHalves; ++hh) {
                            if (j < N)
                                tma_load_3d(dst + hh * kHalfBytes, &tmap_k, BAR(B_KV_FULL + st), hh * 64, g,
                                            key_start + j * kBN);
                            if (j > 0)
                                tma_load_3d(dst + L::kTileBytes + hh * kHalfBytes, &tmap_v, BAR(B_KV_FULL + st),
                                            hh * 64, g, key_start + (j - 1) * kBN);
                        }
                    }
                    __syncwarp();
                    ++c;
                }
                if (!ok) break;
            }
            // drain: every issued load must land before the CTA exits
            const uint32_t issued = c;
            for (uint32_t k = (issued > kSlots ? issued - kSlots : 0); k < issued; ++k)
                drain_bar(BAR(B_KV_FULL + k % kSlots), (k / kSlots) & 1u);
        } else if (warp == kWarpMMA) {
            // ---------------- MMA issuer ----------------
            // step n = 0..N of an item, tile by tile: PV_t(n-1) then QK_t(n) as one run of MMAs
            // (tile t runs while n <= n_t; n_1 <= n_0 = N).  One thread runs this role (waits
            // without warp votes, no warp syncs between runs).
            if (lane == 0) {
                uint32_t cs = 0;              // CTA step index of the current item's step 0
                uint32_t glob[2] = {0u, 0u};  // chunks done per tile (S / P barrier phases)
                uint32_t uses[2] = {0u, 0u};  // items done per tile (Q / O barrier phases)
                bool ok = true;
                // Shared-memory matrix descriptors: one base per operand form; an operand's
                // descriptor is the base plus its byte offset / 16 (shared addresses stay below
                // 2^18 bytes, so the 14-bit start-address field never carries).
                const uint64_t desc_kmaj = smem_desc(sm_base, 16, 1024);                     // Q, K
                const uint64_t desc_mnmaj = smem_desc(sm_base, (uint32_t)kHalfBytes, 1024);  // V
                // the waits of tile t's run at step n (besides its ring slot)
                auto run_waits = [&](int t, int n) -> bool {
                    if (n > 0) {
                        if (!wait_bar1(BAR(B_PFULL + t), (glob[t] + (uint32_t)(n - 1)) & 1u, abort_flag, status))
                            return false;
                        if (n == 1 && uses[t] > 0 &&
                            !wait_bar1(BAR(B_OEMPTY + t), (uses[t] - 1u) & 1u, abort_flag, status))
                            return false;
                    } else if (!wait_bar1(BAR(B_QFULL + t), uses[t] & 1u, abort_flag, status)) {
                        return false;
                    }
                    return true;
                };
                auto run_mmas = [&](int t, int n, int Nt, uint32_t slot) {
                    const uint32_t s_col = tmem + (uint32_t)(kBN * t);
                    const uint32_t o_col = tmem + kColO + (uint32_t)(D * t);
                    if (n > 0) {
                        // PV_t(n-1): P_t from TMEM (16 keys = 8 packed columns per step), V(n-1)
                        // MN-major from the slot (16 keys = 2048 bytes per step)
                        const uint64_t vdesc = desc_mnmaj + ((uint32_t)(L::kKV + (2u * slot + 1u) * L::kTileBytes) >> 4);
                        mma_ts(o_col, s_col, vdesc, kIdescPV, n > 1 ? 1u : 0u);
#pragma unroll
                        for (int kk = 1; kk < kBN / 16; ++kk)
                            mma_ts(o_col, s_col + (uint32_t)kk * 8u, vdesc + (uint64_t)(kk * 128), kIdescPV, 1u);
                    }
                    if (n < Nt) {
                        // QK_t(n) into S_t (after PV_t(n-1) in issue order: P_t has been read);
                        // 16 d-columns per step: 32 bytes inside a 128-byte swizzle row, then the
                        // next [128 x 64] half
                        const uint64_t qdesc = desc_kmaj + ((uint32_t)(L::kQ + t * L::kTileBytes) >> 4);
                        const uint64_t kdesc = desc_kmaj + ((uint32_t)(L::kKV + 2u * slot * L::kTileBytes) >> 4);
#pragma unroll
                        for (int kk = 0; kk < kKSteps; ++kk) {
                            const uint64_t koff = (uint64_t)((kk >> 2) * (kHalfBytes >> 4) + (kk & 3) * 2);
                            mma_ss(s_col, qdesc + koff, kdesc + koff, kIdescQK, kk > 0 ? 1u : 0u);
                        }
                    }
                };
                auto run_commits = [&](int t, int n, int Nt, uint32_t slot, bool release) {
                    if (n < Nt) {
                        mma_commit(BAR(B_SFULL + t));
                        if (n == Nt - 1) mma_commit(BAR(B_QEMPTY + t));
                    }
                    if (n > 0 && n == Nt) mma_commit(BAR(B_OFULL + t));
                    if (release) mma_commit(BAR(B_KV_EMPTY + slot));  // the slot's last reader
                };
                for (int it = 0; ok; ++it) {
                    const int s = it & 1;
                    if (!wait_bar1(BAR(B_INFO + s), (uint32_t)(it >> 1) & 1u, abort_flag, status)) break;
                    const ItemSlot& sl = slots[s];
                    if (sl.kind < 0) break;
                    const int N = sl.nchunks;
                    const int N1 = sl.ntiles == 2 ? sl.n[1] : 0;
                    for (int n = 0; n <= N; ++n) {
                        const uint32_t step = cs + (uint32_t)n, slot = step % kSlots;
                        const bool act1 = N1 > 0 && n <= N1;
                        if (!wait_bar1(BAR(B_KV_FULL + slot), (step / kSlots) & 1u, abort_flag, status) ||
                            !run_waits(0, n)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        run_mmas(0, n, N, slot);
                        // tile 1's waits while tile 0's MMAs are still queued
                        if (act1 && !run_waits(1, n)) {
                            ok = false;
                            break;
                        }
                        run_commits(0, n, N, slot, !act1);
                        if (act1) {
                            tc_fence_after();
                            run_mmas(1, n, N1, slot);
                            run_commits(1, n, N1, slot, true);
                        }
                    }
                    cs += (uint32_t)N + 1u;
                    glob[0] += (uint32_t)N;
                    uses[0] += 1u;
                    if (N1 > 0) {
                        glob[1] += (uint32_t)N1;
                        uses[1] += 1u;
                    }
                }
                // drain the tensor pipe before TMEM is freed
                mma_commit(BAR(B_FINAL));
                drain_bar(BAR(B_FINAL), 0);
            }
            __syncwarp();
        }
    } else {
        // softmax: a whole row of S in registers
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        // ---------------- softmax + epilogue of tile t, thread = query row ----------------
        const int t = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t s_tmem = tmem + lane_off + (uint32_t)(kBN * t);
        const uint32_t o_tmem = tmem + lane_off + kColO + (uint32_t)(D * t);
        uint32_t glob = 0, uses = 0;
        const float ln2 = 0.69314718055994531f;
        const float sl2 = P.scale_log2;
        const float2 sl2x2 = make_float2(sl2, sl2);
        bool ok = true;
        for (int it = 0; ok; ++it) {
            const int s = it & 1;
            if (!wait_bar(BAR(B_INFO + s), (uint32_t)(it >> 1) & 1u, abort_flag, status)) break;
            const ItemSlot& sl = slots[s];
            if (sl.kind < 0) break;
            if (t >= sl.ntiles) {  // this tile is idle for the item
                mbar_arrive(BAR(B_ITEM_EMPTY + s));
                continue;
            }
            const int N = sl.n[t], key_start = sl.key_start, key_end = sl.key_end;
            const int pidx = sl.pidx[t * kTileM + row];
            const int tl = sl.tlim[t * kTileM + row];
            float m = -INFINITY;  // running row maximum, log2 units
            float l = 0.f;        // running row sum of p
            for (int n = 0; n < N; ++n) {
                if (!wait_bar(BAR(B_SFULL + t), (glob + (uint32_t)n) & 1u, abort_flag, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // keys past the block / after the row (current-block items only)
                const int lim = min(key_end - 1, tl) - (key_start + n * kBN);
                const bool masked = __any_sync(0xffffffffu, lim < kBN - 1);
                float x[kBN];
                tmem_ld128(s_tmem, x);
                if (masked) {
#pragma unroll
                    for (int j = 0; j < kBN; ++j) x[j] = (j <= lim) ? x[j] : -INFINITY;
                }
                // row maximum: 8 chains of three-input max over x[u + 8k]
                float mx[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    float a = fmax3(x[u], x[u + 8], x[u + 16]);
#pragma unroll
                    for (int k = 3; k < 15; k += 2) a = fmax3(a, x[u + 8 * k], x[u + 8 * k + 8]);
                    mx[u] = fmaxf(a, x[u + 120]);
                }
                const float mloc =
                    fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * sl2;
                float alpha = 1.f;
                if (n == 0) {
                    m = mloc;
                } else if (__any_sync(0xffffffffu, mloc > m + kRescaleThreshold)) {
                    const float mn = fmaxf(m, mloc);
                    alpha = ex2(m - mn);
                    m = mn;
                }
                // p = 2^(s * scale * log2(e) - m), two lanes per FMA / add; bf16 pairs over the
                // first 64 S columns (every score is already in registers)
                const float2 negm = make_float2(-m, -m);
                float2 acc[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) acc[u] = make_float2(0.f, 0.f);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t w[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int j = 64 * hh + 2 * e;
                        const float2 tt = __ffma2_rn(make_float2(x[j], x[j + 1]), sl2x2, negm);
                        const float2 pr = make_float2(ex2(tt.x), ex2(tt.y));
                        acc[e & 3] = __fadd2_rn(acc[e & 3], pr);
                        w[e] = pack_bf16(pr.x, pr.y);
                    }
                    tmem_st32(s_tmem + 32u * hh, w);
                }
                const float2 a03 = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
                if (n > 0 && __any_sync(0xffffffffu, alpha < 1.f)) {
                    // no MMA touches O_t between the barriers of S_t(n) and P_t(n)
#pragma unroll
                    for (int j = 0; j < D / 32; ++j) {
                        float v[32];
                        tmem_ld32(o_tmem + 32u * j, v);
                        uint32_t w[32];
#pragma unroll
                        for (int e = 0; e < 32; ++e) w[e] = __float_as_uint(v[e] * alpha);
                        tmem_st32(o_tmem + 32u * j, w);
                    }
                }
                l = fmaf(l, alpha, a03.x + a03.y);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(BAR(B_PFULL + t));
            }
            if (!ok) break;
            // epilogue: O_t after its last PV, normalise, write the partial (o, lse)
            if (!wait_bar(BAR(B_OFULL + t), uses & 1u, abort_flag, status)) break;
            tc_fence_after();
            const float inv = 1.f / l;
            // Rows are 2d-byte bf16 partial-output records at scattered addresses.  A thread owns
            // a row, so storing straight from registers would touch 32 rows per warp store.
            // Instead each group of 4 lanes transposes 4x4 blocks of 16-byte pieces by shuffles
            // and every store instruction writes 64 contiguous bytes of each of 8 rows.
            int prow[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) prow[jj] = __shfl_sync(0xffffffffu, pidx, (lane & ~3) + jj);
            const int sub = lane & 3;
#pragma unroll
            for (int j = 0; j < D / 32; ++j) {
                float v[32];
                tmem_ld32(o_tmem + 32u * j, v);
                uint4 a[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    a[e] = make_uint4(pack_bf16(v[8 * e] * inv, v[8 * e + 1] * inv),
                                      pack_bf16(v[8 * e + 2] * inv, v[8 * e + 3] * inv),
                                      pack_bf16(v[8 * e + 4] * inv, v[8 * e + 5] * inv),
                                      pack_bf16(v[8 * e + 6] * inv, v[8 * e + 7] * inv));
                transpose4x4<2>(a, lane);
                transpose4x4<1>(a, lane);
#pragma unroll
                for (int jj = 0; jj < 4; ++jj)
                    if (prow[jj] >= 0)
                        *reinterpret_cast<uint4*>(ws.part_o + (size_t)prow[jj] * D + 32 * j + 8 * sub) = a[jj];
            }
            if (pidx >= 0) ws.part_lse[pidx] = m * ln2 + logf(l);
            tc_fence_before();
            mbar_arrive(BAR(B_OEMPTY + t));
            mbar_arrive(BAR(B_ITEM_EMPTY + s));
            glob += (uint32_t)N;
            ++uses;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMMA) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

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
    attn_tc_kernel<D><<<num_sms, kThreads, smem, st>>>(mk, mv, q, P, ws, t0, t1);
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
