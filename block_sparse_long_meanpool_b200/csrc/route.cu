// Block table and the MoE-style dispatch of query rows to (KV head, block) lists.
//
// The analysis page of the MoBA paper (§3.2) computes the history blocks by regrouping the
// queries per selected KV block, as in mixture-of-experts dispatch, and computes the
// current block separately with a causal mask.  Here, per wave of query tokens [t0, t1):
//
//   route_count    histogram of routed rows per (KV head g, global block b)
//   route_plan     exclusive scans -> list offsets and each list's first work item; the
//                  current-block items (one 128-token query tile for one head, or for two heads
//                  of the same KV head), largest first, after the history items
//   route_items    the history items (<= 256 rows of one list each), one thread per item
//   route_scatter  writes each routed row's partial-output index into its list
//
// A routed entry is the row's partial-output index ((t - t0) * Hq + h) * topk + slot, where
// slot 0 is the own block and slots 1.. are the routed history blocks in row order.
#include "moba_internal.cuh"

namespace moba {

namespace {

constexpr int kPlanThreads = 1024;

// Block-wide exclusive scan of one value per thread (kPlanThreads threads).  Returns the
// exclusive prefix; *total receives the sum over the block.
__device__ int block_exclusive_scan(int v, int* s_warp, int* total) {
    const unsigned full = 0xffffffffu;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(full, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = (lane < kPlanThreads / 32) ? s_warp[lane] : 0;
        int wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(full, wi, off);
            if (lane >= off) wi += y;
        }
        if (lane < kPlanThreads / 32) s_warp[lane] = wi - w;
        if (lane == 31) s_warp[32] = wi;
    }
    __syncthreads();
    const int res = s_warp[warp] + incl - v;
    *total = s_warp[32];
    __syncthreads();
    return res;
}

__global__ void __launch_bounds__(kPlanThreads)
plan_blocks_kernel(const int* __restrict__ cu, Problem P, Workspace ws) {
    __shared__ int s_total;
    if (threadIdx.x == 0) {
        int run = 0;
        for (int i = 0; i < P.batch; ++i) {
            ws.cu_blocks[i] = run;
            const int n = cu[i + 1] - cu[i];
            run += (n + P.chunk - 1) / P.chunk;
        }
        ws.cu_blocks[P.batch] = run;
        ws.hdr->nb_total = run;
        ws.hdr->status = 0;
        s_total = run;
    }
    __syncthreads();
    const int nb = s_total;
    for (int b = threadIdx.x; b < nb; b += blockDim.x) {
        int lo = 0, hi = P.batch;  // last sequence i with cu_blocks[i] <= b
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (ws.cu_blocks[mid] <= b) lo = mid; else hi = mid;
        }
        const int i = lo;
        const int local = b - ws.cu_blocks[i];
        const int start = cu[i] + local * P.chunk;
        ws.blk_start[b] = start;
        ws.blk_len[b] = min(P.chunk, cu[i + 1] - start);
        ws.blk_seq[b] = i;
        ws.blk_local[b] = local;
    }
}

// Rows of the wave are processed in CTA-sized ranges of consecutive (t, h) rows.  All the
// lists a range can touch are (g, b) with b in [first block of the range's first sequence,
// own block of its last row), so a CTA counts its entries in a shared-memory histogram over
// that span and touches each global list counter once (kScatter = false), or reserves one
// contiguous range per list with one global atomic and hands out positions from shared
// memory (kScatter = true).  Spans too wide for shared memory fall back to one global atomic
// per entry.  Positions inside a list depend on timing, results do not: every row's partial
// output index travels with it.
constexpr int kRouteThreads = 256;
constexpr int kRouteRows = 4096;        // query rows per CTA
constexpr int kRouteSmemLists = 12288;  // shared-memory histogram capacity (48 KB)

struct RowRef {
    int t, h, g, c, first;
    const int* row;
};

__device__ __forceinline__ RowRef row_ref(const int* __restrict__ cu, const int* __restrict__ sel,
                                          const Problem& P, const Workspace& ws, int t0,
                                          long long r) {
    RowRef x;
    x.t = t0 + (int)(r / P.hq);
    x.h = (int)(r % P.hq);
    const int i = seq_of_token(cu, P.batch, x.t);
    x.c = (x.t - __ldg(cu + i)) / P.chunk;
    x.first = ws.cu_blocks[i];
    x.g = x.h / P.group;
    x.row = sel + ((size_t)x.h * P.T + x.t) * P.topk;
    return x;
}

template <bool kScatter, int K>
__global__ void __launch_bounds__(kRouteThreads)
route_rows_kernel(const int* __restrict__ cu, const int* __restrict__ sel, Problem P,
                  Workspace ws, int t0, int t1) {
    __shared__ int hist[kRouteSmemLists];
    const long long n = (long long)(t1 - t0) * P.hq;
    const long long r0 = (long long)blockIdx.x * kRouteRows;
    if (r0 >= n) return;
    const long long r1 = min(n, r0 + kRouteRows);
    // block span of the lists this range can touch
    const RowRef a = row_ref(cu, sel, P, ws, t0, r0);
    const RowRef z = row_ref(cu, sel, P, ws, t0, r1 - 1);
    const int b_lo = a.first;
    const int b_hi = z.first + z.c;  // exclusive: history blocks are strictly before c
    const int span = b_hi - b_lo;
    if (span <= 0) {  // no row of the range routes anything: one slot (the own block) each
        if (!kScatter)
            for (long long r = r0 + threadIdx.x; r < r1; r += kRouteThreads) ws.nslots[r] = 1;
        return;
    }
    const bool in_smem = (long long)P.hkv * span <= kRouteSmemLists;
    if (!in_smem) {
        for (long long r = r0 + threadIdx.x; r < r1; r += kRouteThreads) {
            const RowRef x = row_ref(cu, sel, P, ws, t0, r);
            const int pbase = (int)(r * P.topk);
            const int nr = for_each_routed<K>(x.row, P.topk, x.c, [&](int slot, int j) {
                int* ctr = (kScatter ? ws.cursor : ws.counts) + (size_t)x.g * P.nb_cap + x.first + j;
                const int pos = atomicAdd(ctr, 1);
                if (kScatter) ws.entries[pos] = pbase + slot;
            });
            if (!kScatter) ws.nslots[r] = (unsigned char)(1 + nr);
        }
        return;
    }
    const int nl = P.hkv * span;
    for (int i = threadIdx.x; i < nl; i += kRouteThreads) hist[i] = 0;
    __syncthreads();
    for (long long r = r0 + threadIdx.x; r < r1; r += kRouteThreads) {
        const RowRef x = row_ref(cu, sel, P, ws, t0, r);
        const int nr = for_each_routed<K>(x.row, P.topk, x.c, [&](int, int j) {
            atomicAdd(&hist[x.g * span + (x.first + j - b_lo)], 1);
        });
        if (!kScatter) ws.nslots[r] = (unsigned char)(1 + nr);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nl; i += kRouteThreads) {
        const int cnt = hist[i];
        if (cnt == 0) continue;
        const int g = i / span, bb = i - g * span;
        int* ctr = (kScatter ? ws.cursor : ws.counts) + (size_t)g * P.nb_cap + b_lo + bb;
        const int base = atomicAdd(ctr, cnt);
        if (kScatter) hist[i] = base;
    }
    if (!kScatter) return;
    __syncthreads();
    for (long long r = r0 + threadIdx.x; r < r1; r += kRouteThreads) {
        const RowRef x = row_ref(cu, sel, P, ws, t0, r);
        const int pbase = (int)(r * P.topk);
        for_each_routed<K>(x.row, P.topk, x.c, [&](int slot, int j) {
            const int pos = atomicAdd(&hist[x.g * span + (x.first + j - b_lo)], 1);
            ws.entries[pos] = pbase + slot;
        });
    }
}

__global__ void __launch_bounds__(kPlanThreads)
route_plan_kernel(Problem P, Workspace ws, int t0, int t1) {
    __shared__ int s_warp[33];
    const int n_lists = P.hkv * P.nb_cap;
    // 1. list offsets
    int carry = 0;
    for (int base = 0; base < n_lists; base += kPlanThreads) {
        const int L = base + threadIdx.x;
        const int cnt = (L < n_lists) ? ws.counts[L] : 0;
        int tot;
        const int ex = block_exclusive_scan(cnt, s_warp, &tot);
        if (L < n_lists) {
            ws.offsets[L] = carry + ex;
            ws.cursor[L] = carry + ex;
        }
        carry += tot;
    }
    if (threadIdx.x == 0) ws.offsets[n_lists] = carry;
    // 2. history items (up to two tiles of routed rows), list by list: only each list's first
    //    item index here; route_items_kernel writes the items themselves on the whole GPU
    int tcarry = 0;
    for (int base = 0; base < n_lists; base += kPlanThreads) {
        const int L = base + threadIdx.x;
        const int cnt = (L < n_lists) ? ws.counts[L] : 0;
        const int nt = (cnt + kItemRows - 1) / kItemRows;
        int tot;
        const int ex = block_exclusive_scan(nt, s_warp, &tot);
        if (L < n_lists) ws.item_off[L] = tcarry + ex;
        tcarry += tot;
    }
    if (threadIdx.x == 0) ws.item_off[n_lists] = tcarry;
    const int n_past = tcarry;
    // 3. current-block items of the blocks overlapping [t0, t1), by decreasing tile index
    //    (tile q has q + 1 key tiles of work)
    const int nb = ws.hdr->nb_total;
    int lo = 0, hi = nb;  // first block whose end is > t0
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (ws.blk_start[mid] + ws.blk_len[mid] <= t0) lo = mid + 1; else hi = mid;
    }
    const int b_lo = lo;
    lo = b_lo;
    hi = nb;  // first block whose start is >= t1
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (ws.blk_start[mid] < t1) lo = mid + 1; else hi = mid;
    }
    const int b_hi = lo;
    const int levels = (P.chunk + kTileM - 1) / kTileM;
    // does query tile qt of block b (a block of length len) hold a token of [t0, t1)?
    auto overlaps = [&](int b, int len, int qt) {
        const int r0 = qt * kTileM;
        if (r0 >= len) return false;
        const int a = ws.blk_start[b] + r0;
        const int e = ws.blk_start[b] + min(r0 + kTileM, len);
        return a < t1 && e > t0;
    };
    int dcarry = n_past;
    if (P.group > 1) {
        // heads of one KV head go in pairs (same keys and values); largest query tile first
        // (tile qt has qt + 1 key chunks of work)
        const int per_block = P.hkv * ((P.group + 1) / 2);  // items per query tile
        for (int qt = levels - 1; qt >= 0; --qt) {
            for (int base = b_lo; base < b_hi; base += kPlanThreads) {
                const int b = base + threadIdx.x;
                const int has = (b < b_hi && overlaps(b, ws.blk_len[b], qt)) ? 1 : 0;
                int tot;
                const int ex = block_exclusive_scan(has, s_warp, &tot);
                if (has) {
                    int k = 0;
                    for (int g = 0; g < P.hkv; ++g) {
                        for (int j = 0; j < P.group; j += 2) {
                            WorkItem it;
                            it.a = b;
                            it.b = g * P.group + j;
                            it.c = qt;
                            it.kind = (j + 1 < P.group) ? 2 : 1;
                            ws.items[dcarry + ex * per_block + k] = it;
                            ++k;
                        }
                    }
                }
                dcarry += tot * per_block;
            }
        }
    } else {
        // one query head per KV head: query tiles lv-1-p and p of the same head and block go
        // together (same keys and values; every pair spans lv + 1 key chunks)
        for (int p = 0; p < (levels + 1) / 2; ++p) {
            for (int base = b_lo; base < b_hi; base += kPlanThreads) {
                const int b = base + threadIdx.x;
                int kind = -1, qt = 0;
                if (b < b_hi) {
                    const int len = ws.blk_len[b];
                    const int lv = (len + kTileM - 1) / kTileM;
                    if (p < (lv + 1) / 2) {
                        const int qa = lv - 1 - p;
                        const bool ha = overlaps(b, len, qa);
                        const bool hb = p != qa && overlaps(b, len, p);
                        if (ha && hb) {
                            kind = 3;
                            qt = p;
                        } else if (ha || hb) {
                            kind = 1;
                            qt = ha ? qa : p;
                        }
                    }
                }
                const int has = kind >= 0 ? 1 : 0;
                int tot;
                const int ex = block_exclusive_scan(has, s_warp, &tot);
                if (has) {
                    for (int h = 0; h < P.hq; ++h) {
                        WorkItem it;
                        it.a = b;
                        it.b = h;
                        it.c = qt;
                        it.kind = kind;
                        ws.items[dcarry + ex * P.hq + h] = it;
                    }
                }
                dcarry += tot * P.hq;
            }
        }
    }
    if (threadIdx.x == 0) {
        ws.hdr->n_items = dcarry;
        ws.hdr->n_past_items = n_past;
        ws.hdr->work_counter = 0u;
    }
}

// History work items of the wave, one thread per item: item i belongs to the last list L with
// item_off[L] <= i (empty lists share their successor's offset), as its (i - item_off[L])-th
// tile of up to kItemRows routed rows.
__global__ void __launch_bounds__(256)
route_items_kernel(Problem P, Workspace ws) {
    const int n_lists = P.hkv * P.nb_cap;
    const int n_past = ws.item_off[n_lists];
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_past; i += gridDim.x * blockDim.x) {
        int lo = 0, hi = n_lists;  // answer in [lo, hi): item_off[lo] <= i < item_off[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(ws.item_off + mid) <= i) lo = mid; else hi = mid;
        }
        const int k = i - __ldg(ws.item_off + lo);
        WorkItem it;
        it.a = lo;
        it.b = __ldg(ws.offsets + lo) + k * kItemRows;
        it.c = min(kItemRows, __ldg(ws.counts + lo) - k * kItemRows);
        it.kind = 0;
        ws.items[i] = it;
    }
}

template <bool kScatter>
void launch_rows(const Problem& P, const int* cu, const int* sel, const Workspace& ws, int t0,
                 int t1, int grid, cudaStream_t st) {
    if (P.topk <= 4)
        route_rows_kernel<kScatter, 4><<<grid, kRouteThreads, 0, st>>>(cu, sel, P, ws, t0, t1);
    else if (P.topk <= 8)
        route_rows_kernel<kScatter, 8><<<grid, kRouteThreads, 0, st>>>(cu, sel, P, ws, t0, t1);
    else if (P.topk <= 16)
        route_rows_kernel<kScatter, 16><<<grid, kRouteThreads, 0, st>>>(cu, sel, P, ws, t0, t1);
    else
        route_rows_kernel<kScatter, 32><<<grid, kRouteThreads, 0, st>>>(cu, sel, P, ws, t0, t1);
}

int rows_grid(long long n) {
    long long g = (n + kRouteRows - 1) / kRouteRows;
    return (int)(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_plan_blocks(const Problem& P, const int* cu_seqlens, const Workspace& ws,
                               cudaStream_t st) {
    plan_blocks_kernel<<<1, kPlanThreads, 0, st>>>(cu_seqlens, P, ws);
    return cudaGetLastError();
}

cudaError_t launch_route_count(const Problem& P, const int* cu_seqlens, const int* sel,
                               const Workspace& ws, int t0, int t1, cudaStream_t st) {
    const long long n = (long long)(t1 - t0) * P.hq;
    launch_rows<false>(P, cu_seqlens, sel, ws, t0, t1, rows_grid(n), st);
    return cudaGetLastError();
}

cudaError_t launch_route_plan(const Problem& P, const Workspace& ws, int t0, int t1,
                              cudaStream_t st) {
    route_plan_kernel<<<1, kPlanThreads, 0, st>>>(P, ws, t0, t1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    route_items_kernel<<<4 * 148, 256, 0, st>>>(P, ws);
    return cudaGetLastError();
}

cudaError_t launch_route_scatter(const Problem& P, const int* cu_seqlens, const int* sel,
                                 const Workspace& ws, int t0, int t1, cudaStream_t st) {
    const long long n = (long long)(t1 - t0) * P.hq;
    launch_rows<true>(P, cu_seqlens, sel, ws, t0, t1, rows_grid(n), st);
    return cudaGetLastError();
}

}  // namespace moba
