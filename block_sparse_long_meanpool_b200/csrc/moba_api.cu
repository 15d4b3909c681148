// Host side of the C ABI declared in include/moba.h: argument checks, workspace layout,
// and the launch sequence of the MoBA prefill forward.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "moba.h"
#include "moba_internal.cuh"
#include "ptx.cuh"

using namespace moba;

namespace {

// Named NVTX range over a scope.  Without a profiler attached each push/pop is a no-op after a
// one-time check; under nsys or ncu every launch is attributed to its entry point and stage,
// e.g. `ncu --clock-control none --nvtx --nvtx-include "moba_attn_fwd/wave/attention/"` captures the attention
// launches only.
struct NvtxScope {
    explicit NvtxScope(const char* name) { nvtxRangePushA(name); }
    ~NvtxScope() { nvtxRangePop(); }
    NvtxScope(const NvtxScope&) = delete;
    NvtxScope& operator=(const NvtxScope&) = delete;
};

thread_local std::string g_last_error;

moba_status fail(moba_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
moba_status fail(moba_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

moba_status cuda_fail(cudaError_t e, const char* what) {
    return fail(MOBA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t x) { return (x + 255) & ~size_t(255); }

// Shape checks common to every entry point.
moba_status check_params(const moba_params* p) {
    if (!p) return fail(MOBA_ERR_INVALID_ARG, "params is NULL");
    if (p->batch < 1) return fail(MOBA_ERR_INVALID_ARG, "batch must be >= 1 (got %d)", p->batch);
    if (p->total_tokens < 0)
        return fail(MOBA_ERR_INVALID_ARG, "total_tokens must be >= 0 (got %d)", p->total_tokens);
    if (p->num_q_heads < 1 || p->num_kv_heads < 1)
        return fail(MOBA_ERR_INVALID_ARG, "head counts must be >= 1");
    if (p->num_q_heads % p->num_kv_heads)
        return fail(MOBA_ERR_INVALID_ARG, "num_q_heads (%d) %% num_kv_heads (%d) != 0",
                    p->num_q_heads, p->num_kv_heads);
    if (p->topk < 1) return fail(MOBA_ERR_INVALID_ARG, "topk must be >= 1 (got %d)", p->topk);
    if (p->chunk_size < 1)
        return fail(MOBA_ERR_INVALID_ARG, "chunk_size must be >= 1 (got %d)", p->chunk_size);
    if (p->head_dim < 1) return fail(MOBA_ERR_INVALID_ARG, "head_dim must be >= 1");
    if (p->wave_tokens < 0) return fail(MOBA_ERR_INVALID_ARG, "wave_tokens must be >= 0");
    if (p->gate != MOBA_GATE_MEAN && p->gate != MOBA_GATE_MINMAX)
        return fail(MOBA_ERR_INVALID_ARG, "gate must be MOBA_GATE_MEAN or MOBA_GATE_MINMAX (got %d)",
                    p->gate);
    if (p->max_seqlen < 0)
        return fail(MOBA_ERR_INVALID_ARG, "max_seqlen must be >= 0 (got %d)", p->max_seqlen);
    if (p->max_seqlen > 0 &&
        (p->max_seqlen > p->total_tokens || (long long)p->batch * p->max_seqlen < p->total_tokens))
        return fail(MOBA_ERR_INVALID_ARG,
                    "max_seqlen %d inconsistent with %d tokens in %d sequences", p->max_seqlen,
                    p->total_tokens, p->batch);
    if (!(p->softmax_scale == p->softmax_scale) || std::isinf(p->softmax_scale))
        return fail(MOBA_ERR_INVALID_ARG, "softmax_scale must be finite");
    if (p->head_dim != 64 && p->head_dim != 128)
        return fail(MOBA_ERR_UNSUPPORTED, "head_dim %d unsupported (64 or 128)", p->head_dim);
    if (p->chunk_size % kTileM)
        return fail(MOBA_ERR_UNSUPPORTED, "chunk_size %d unsupported (multiple of %d)",
                    p->chunk_size, kTileM);
    if (p->topk > 32) return fail(MOBA_ERR_UNSUPPORTED, "topk %d unsupported (<= 32)", p->topk);
    if (p->wave_tokens % kTileM)
        return fail(MOBA_ERR_UNSUPPORTED, "wave_tokens %d must be a multiple of %d",
                    p->wave_tokens, kTileM);
    if ((long long)p->num_q_heads * p->topk > (1 << 20))
        return fail(MOBA_ERR_UNSUPPORTED, "num_q_heads * topk too large");
    return MOBA_OK;
}

long long blocks_bound(const moba_params& p) {
    if (p.total_tokens == 0) return 0;
    long long nb = (p.total_tokens + (long long)p.chunk_size - 1) / p.chunk_size + p.batch - 1;
    return nb < p.total_tokens ? nb : p.total_tokens;
}

struct Layout {
    size_t hdr, cu_blocks, blk_start, blk_len, blk_seq, blk_local, means, sel, counts, offsets,
        cursor, item_off, entries, items, part_o, part_lse, nslots, total;
    int wave;
    long long nb_cap, max_items;
};

Layout make_layout(const moba_params& p) {
    Layout L{};
    const long long T = p.total_tokens;
    L.nb_cap = blocks_bound(p);
    L.wave = (p.wave_tokens > 0 && p.wave_tokens < T) ? p.wave_tokens : (int)T;
    const long long W = L.wave;
    // Work items of one wave (route_plan_kernel), bounded from above:
    //  - history: a list of n routed rows gives ceil(n / 256) items <= n / 256 + 1, so all lists
    //    give at most routed / 256 + min(lists, routed);
    //  - current block: at most Hq items per 128-row query tile that overlaps the wave (head
    //    pairs give Hkv * ceil(group / 2) <= Hq, MHA tile pairs fewer).  Blocks start on their
    //    sequence's 128-token grid and only a sequence's last block is partial, so the tiles
    //    overlapping W tokens number at most W / 128 + (partial blocks) + 2 (the blocks that
    //    straddle the wave's ends), within W / 128 + min(NB, W) + 4.
    const long long lists = (long long)p.num_kv_heads * L.nb_cap;
    const long long routed = W * p.num_q_heads * (p.topk - 1);
    const long long past_items = routed / kTileM + (lists < routed ? lists : routed) + 1;
    const long long blk_in_wave = L.nb_cap < W ? L.nb_cap : W;
    const long long diag_items = (long long)p.num_q_heads * (W / kTileM + blk_in_wave + 4);
    L.max_items = past_items + diag_items;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = align_up(o + bytes);
        return at;
    };
    L.hdr = take(sizeof(WsHeader));
    L.cu_blocks = take(4ull * (p.batch + 1));
    L.blk_start = take(4ull * L.nb_cap);
    L.blk_len = take(4ull * L.nb_cap);
    L.blk_seq = take(4ull * L.nb_cap);
    L.blk_local = take(4ull * L.nb_cap);
    L.means = take(4ull * L.nb_cap * p.num_kv_heads * p.head_dim);
    L.sel = take(4ull * p.num_q_heads * T * p.topk);
    L.counts = take(4ull * lists);
    L.offsets = take(4ull * (lists + 1));
    L.cursor = take(4ull * lists);
    L.item_off = take(4ull * (lists + 1));
    L.entries = take(4ull * routed);
    L.items = take(sizeof(WorkItem) * L.max_items);
    L.part_o = take(2ull * W * p.num_q_heads * p.topk * p.head_dim);  // bf16
    L.part_lse = take(4ull * W * p.num_q_heads * p.topk);
    L.nslots = take(1ull * W * p.num_q_heads);
    L.total = o;
    return L;
}

Problem make_problem(const moba_params& p, long long nb_cap) {
    Problem P;
    P.batch = p.batch;
    P.T = p.total_tokens;
    P.hq = p.num_q_heads;
    P.hkv = p.num_kv_heads;
    P.d = p.head_dim;
    P.chunk = p.chunk_size;
    P.topk = p.topk;
    P.group = p.num_q_heads / p.num_kv_heads;
    P.nb_cap = (int)nb_cap;
    P.max_blocks = (int)nb_cap;
    if (p.max_seqlen > 0) {
        const long long mb = (p.max_seqlen + (long long)p.chunk_size - 1) / p.chunk_size;
        if (mb < nb_cap) P.max_blocks = (int)mb;
    }
    P.scale = p.softmax_scale > 0.f ? p.softmax_scale : 1.0f / sqrtf((float)p.head_dim);
    P.scale_log2 = P.scale * 1.4426950408889634f;
    return P;
}

int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}

// The min/max gate runs on the tensor cores only: every sequence must have <= 257 blocks.
moba_status check_minmax_gate(const Problem& P) {
    if (P.max_blocks > 257)
        return fail(MOBA_ERR_UNSUPPORTED,
                    "the min/max gate needs every sequence to have <= 257 blocks (%d possible; "
                    "give max_seqlen)", P.max_blocks);
    return MOBA_OK;
}

// Index-range limits of the 32-bit indices used on the device.
moba_status check_ranges(const moba_params& p, const Layout& L) {
    const long long lim = 0x7fffffffLL;
    if ((long long)L.wave * p.num_q_heads * p.topk > lim)
        return fail(MOBA_ERR_UNSUPPORTED,
                    "wave_tokens * num_q_heads * topk exceeds 2^31; set a smaller wave_tokens");
    if (L.max_items > lim || (long long)p.num_kv_heads * L.nb_cap > lim)
        return fail(MOBA_ERR_UNSUPPORTED, "too many blocks for 32-bit work indices");
    return MOBA_OK;
}

}  // namespace

namespace moba {
// Lets other translation units of the library report a failure through moba_last_error().
void set_error_message(const char* msg) { g_last_error = msg; }
}  // namespace moba

extern "C" {

int moba_num_blocks_bound(const moba_params* p) {
    if (check_params(p) != MOBA_OK) return -1;
    return (int)blocks_bound(*p);
}

size_t moba_workspace_size(const moba_params* p) {
    if (check_params(p) != MOBA_OK) return 0;
    return make_layout(*p).total;
}

moba_status moba_meanpool(const moba_params* p, const void* k, const int* cu_seqlens,
                          float* k_mean, void* stream) {
    NvtxScope range("moba_meanpool");
    moba_status s = check_params(p);
    if (s != MOBA_OK) return s;
    if (p->total_tokens == 0) return MOBA_OK;
    if (!k || !cu_seqlens || !k_mean) return fail(MOBA_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned16(k) || !aligned16(k_mean))
        return fail(MOBA_ERR_INVALID_ARG, "k and k_mean must be 16-byte aligned");
    const Problem P = make_problem(*p, blocks_bound(*p));
    cudaError_t e = launch_meanpool(P, static_cast<const __nv_bfloat16*>(k), cu_seqlens, k_mean,
                                    static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "meanpool launch");
    return MOBA_OK;
}

moba_status moba_minmaxpool(const moba_params* p, const void* k, const int* cu_seqlens,
                            void* k_min, void* k_max, void* stream) {
    NvtxScope range("moba_minmaxpool");
    moba_status s = check_params(p);
    if (s != MOBA_OK) return s;
    if (p->total_tokens == 0) return MOBA_OK;
    if (!k || !cu_seqlens || !k_min || !k_max) return fail(MOBA_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned16(k) || !aligned16(k_min) || !aligned16(k_max))
        return fail(MOBA_ERR_INVALID_ARG, "k, k_min and k_max must be 16-byte aligned");
    const Problem P = make_problem(*p, blocks_bound(*p));
    cudaError_t e = launch_minmaxpool(P, static_cast<const __nv_bfloat16*>(k), cu_seqlens,
                                      static_cast<__nv_bfloat16*>(k_min), static_cast<__nv_bfloat16*>(k_max),
                                      static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "minmaxpool launch");
    return MOBA_OK;
}

moba_status moba_gate_topk(const moba_params* p, const void* q, const float* k_mean,
                           const int* cu_seqlens, int* sel, void* stream) {
    NvtxScope range("moba_gate_topk");
    moba_status s = check_params(p);
    if (s != MOBA_OK) return s;
    if (p->total_tokens == 0) return MOBA_OK;
    if (!q || !k_mean || !cu_seqlens || !sel)
        return fail(MOBA_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned16(q) || !aligned16(k_mean))
        return fail(MOBA_ERR_INVALID_ARG, "q and k_mean must be 16-byte aligned");
    const Problem P = make_problem(*p, blocks_bound(*p));
    cudaError_t e = launch_gate_best(P, static_cast<const __nv_bfloat16*>(q),
                                     GateSummary{k_mean, nullptr, nullptr}, cu_seqlens, sel, nullptr,
                                     static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "gate launch");
    return MOBA_OK;
}

moba_status moba_gate_minmax_topk(const moba_params* p, const void* q, const void* k_min,
                                  const void* k_max, const int* cu_seqlens, int* sel, void* stream) {
    NvtxScope range("moba_gate_minmax_topk");
    moba_status s = check_params(p);
    if (s != MOBA_OK) return s;
    if (p->total_tokens == 0) return MOBA_OK;
    if (!q || !k_min || !k_max || !cu_seqlens || !sel)
        return fail(MOBA_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned16(q) || !aligned16(k_min) || !aligned16(k_max))
        return fail(MOBA_ERR_INVALID_ARG, "q, k_min and k_max must be 16-byte aligned");
    const Problem P = make_problem(*p, blocks_bound(*p));
    s = check_minmax_gate(P);
    if (s != MOBA_OK) return s;
    cudaError_t e = launch_gate_best(P, static_cast<const __nv_bfloat16*>(q),
                                     GateSummary{nullptr, static_cast<const __nv_bfloat16*>(k_min),
                                                 static_cast<const __nv_bfloat16*>(k_max)},
                                     cu_seqlens, sel, nullptr, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "gate launch");
    return MOBA_OK;
}

moba_status moba_attn_fwd(const moba_params* p, const void* q, const void* k, const void* v,
                          const int* cu_seqlens, const int* sel_in, int* sel_out,
                          void* workspace, size_t workspace_bytes, void* out, float* lse,
                          moba_run_info* info, void* stream) {
    NvtxScope range("moba_attn_fwd");
    moba_status s = check_params(p);
    if (s != MOBA_OK) return s;
    if (info) {
        info->launches = 0;
        info->waves = 0;
        info->gate_path = MOBA_GATE_PATH_NONE;
    }
    if (p->total_tokens == 0) return MOBA_OK;
    if (!q || !k || !v || !cu_seqlens || !out || !lse)
        return fail(MOBA_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return fail(MOBA_ERR_INVALID_ARG, "q, k, v and out must be 16-byte aligned");
    const Layout L = make_layout(*p);
    s = check_ranges(*p, L);
    if (s != MOBA_OK) return s;
    if (!workspace || workspace_bytes < L.total)
        return fail(MOBA_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", L.total,
                    workspace ? workspace_bytes : (size_t)0);
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
        return fail(MOBA_ERR_WORKSPACE, "workspace must be 256-byte aligned");

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Problem P = make_problem(*p, L.nb_cap);
    if (!sel_in && p->gate == MOBA_GATE_MINMAX) {
        s = check_minmax_gate(P);
        if (s != MOBA_OK) return s;
    }
    char* base = static_cast<char*>(workspace);
    Workspace ws;
    ws.hdr = reinterpret_cast<WsHeader*>(base + L.hdr);
    ws.cu_blocks = reinterpret_cast<int*>(base + L.cu_blocks);
    ws.blk_start = reinterpret_cast<int*>(base + L.blk_start);
    ws.blk_len = reinterpret_cast<int*>(base + L.blk_len);
    ws.blk_seq = reinterpret_cast<int*>(base + L.blk_seq);
    ws.blk_local = reinterpret_cast<int*>(base + L.blk_local);
    ws.means = reinterpret_cast<float*>(base + L.means);
    ws.sel = reinterpret_cast<int*>(base + L.sel);
    ws.counts = reinterpret_cast<int*>(base + L.counts);
    ws.offsets = reinterpret_cast<int*>(base + L.offsets);
    ws.cursor = reinterpret_cast<int*>(base + L.cursor);
    ws.item_off = reinterpret_cast<int*>(base + L.item_off);
    ws.entries = reinterpret_cast<int*>(base + L.entries);
    ws.items = reinterpret_cast<WorkItem*>(base + L.items);
    ws.part_o = reinterpret_cast<__nv_bfloat16*>(base + L.part_o);
    ws.part_lse = reinterpret_cast<float*>(base + L.part_lse);
    ws.nslots = reinterpret_cast<unsigned char*>(base + L.nslots);

    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q);
    const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(k);
    const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(v);
    int launches = 0;
    auto record = [&](int idx) -> cudaError_t {
        if (info && info->events && idx < info->n_events && info->events[idx])
            return cudaEventRecord(static_cast<cudaEvent_t>(info->events[idx]), st);
        return cudaSuccess;
    };
    cudaError_t e;
#define MOBA_TRY(expr, what)                      \
    do {                                          \
        e = (expr);                               \
        if (e != cudaSuccess) return cuda_fail(e, what); \
    } while (0)

    // the block summary of the gate: fp32 means, or the bf16 min/max pair in the same bytes
    const bool minmax = p->gate == MOBA_GATE_MINMAX;
    const size_t summ_elems = (size_t)L.nb_cap * P.hkv * P.d;
    __nv_bfloat16* kmin_ws = reinterpret_cast<__nv_bfloat16*>(ws.means);
    __nv_bfloat16* kmax_ws = kmin_ws + summ_elems;
    const GateSummary summary = minmax ? GateSummary{nullptr, kmin_ws, kmax_ws}
                                       : GateSummary{ws.means, nullptr, nullptr};
    MOBA_TRY(record(MOBA_EV_BEGIN), "event record");
    {
        NvtxScope stage("means");
        MOBA_TRY(launch_plan_blocks(P, cu_seqlens, ws, st), "block table launch");
        if (minmax)
            MOBA_TRY(launch_minmaxpool(P, kb, cu_seqlens, kmin_ws, kmax_ws, st), "minmaxpool launch");
        else
            MOBA_TRY(launch_meanpool(P, kb, cu_seqlens, ws.means, st), "meanpool launch");
    }
    launches += 2;
    MOBA_TRY(record(MOBA_EV_MEANS_DONE), "event record");
    const int* sel_use = sel_in;
    if (!sel_use) {
        NvtxScope stage("gate");
        int* dst = sel_out ? sel_out : ws.sel;
        int path = MOBA_GATE_PATH_NONE;
        MOBA_TRY(launch_gate_best(P, qb, summary, cu_seqlens, dst, &ws.hdr->status, st, &path),
                 "gate launch");
        if (info) info->gate_path = path;
        ++launches;
        sel_use = dst;
    }
    MOBA_TRY(record(MOBA_EV_GATE_DONE), "event record");

    const int num_sms = device_sm_count();
    const int T = p->total_tokens;
    int w = 0;
    for (int t0 = 0; t0 < T; t0 += L.wave, ++w) {
        const int t1 = (T - t0 > L.wave) ? t0 + L.wave : T;
        const int ev = MOBA_EV_WAVE0 + 4 * w;
        NvtxScope wave("wave");
        MOBA_TRY(record(ev), "event record");
        {
            NvtxScope stage("route");
            MOBA_TRY(cudaMemsetAsync(ws.counts, 0, 4ull * P.hkv * L.nb_cap, st), "memset");
            MOBA_TRY(launch_route_count(P, cu_seqlens, sel_use, ws, t0, t1, st), "route count launch");
            MOBA_TRY(launch_route_plan(P, ws, t0, t1, st), "route plan launch");
            MOBA_TRY(launch_route_scatter(P, cu_seqlens, sel_use, ws, t0, t1, st), "route scatter launch");
        }
        MOBA_TRY(record(ev + 1), "event record");
        {
            NvtxScope stage("attention");
            MOBA_TRY(launch_attention(P, qb, kb, vb, ws, t0, t1, num_sms, st), "attention launch");
        }
        MOBA_TRY(record(ev + 2), "event record");
        {
            NvtxScope stage("merge");
            MOBA_TRY(launch_merge(P, cu_seqlens, sel_use, ws, t0, t1,
                                  static_cast<__nv_bfloat16*>(out), lse, st),
                     "merge launch");
        }
        MOBA_TRY(record(ev + 3), "event record");
        launches += 6;  // route count, plan, items, scatter; attention; merge
    }
#undef MOBA_TRY
    if (info) {
        info->launches = launches;
        info->waves = w;
    }
    return MOBA_OK;
}

// ---- backward -------------------------------------------------------------------------

namespace {

struct BwdLayout {
    size_t hdr, cu_blocks, blk_start, blk_len, blk_seq, blk_local, counts, offsets, cursor,
        item_off, entries, items, nslots, rs, dq_acc, total;
    long long nb_cap, max_items;
};

// The backward routes every row at once (one wave from token 0) and keeps no partial outputs:
// the block table, the routing lists and work items of all T tokens, per-row statistics and
// an fp32 dq accumulator.
BwdLayout make_bwd_layout(const moba_params& p) {
    moba_params one = p;
    one.wave_tokens = 0;
    const Layout F = make_layout(one);  // work-item bound of a single wave over all tokens
    BwdLayout L{};
    const long long T = p.total_tokens;
    L.nb_cap = F.nb_cap;
    L.max_items = F.max_items;
    const long long lists = (long long)p.num_kv_heads * L.nb_cap;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = align_up(o + bytes);
        return at;
    };
    L.hdr = take(sizeof(WsHeader));
    L.cu_blocks = take(4ull * (p.batch + 1));
    L.blk_start = take(4ull * L.nb_cap);
    L.blk_len = take(4ull * L.nb_cap);
    L.blk_seq = take(4ull * L.nb_cap);
    L.blk_local = take(4ull * L.nb_cap);
    L.counts = take(4ull * lists);
    L.offsets = take(4ull * (lists + 1));
    L.cursor = take(4ull * lists);
    L.item_off = take(4ull * (lists + 1));
    L.entries = take(4ull * T * p.num_q_heads * (p.topk - 1));
    L.items = take(sizeof(WorkItem) * L.max_items);
    L.nslots = take(1ull * T * p.num_q_heads);
    L.rs = take(8ull * T * p.num_q_heads);
    L.dq_acc = take(4ull * T * p.num_q_heads * p.head_dim);
    L.total = o;
    return L;
}

}  // namespace

size_t moba_bwd_workspace_size(const moba_params* p) {
    if (check_params(p) != MOBA_OK) return 0;
    return make_bwd_layout(*p).total;
}

moba_status moba_attn_bwd(const moba_params* p, const void* q, const void* k, const void* v,
                          const void* out, const float* lse, const void* d_out, const float* d_lse,
                          const int* cu_seqlens, const int* sel, void* workspace,
                          size_t workspace_bytes, void* dq, void* dk, void* dv, void* stream) {
    NvtxScope range("moba_attn_bwd");
    moba_status s = check_params(p);
    if (s != MOBA_OK) return s;
    if (p->total_tokens == 0) return MOBA_OK;
    if (!q || !k || !v || !out || !lse || !d_out || !cu_seqlens || !sel || !dq || !dk || !dv)
        return fail(MOBA_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(d_out) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return fail(MOBA_ERR_INVALID_ARG, "q, k, v, out, d_out, dq, dk and dv must be 16-byte aligned");
    if ((long long)p->total_tokens * p->num_q_heads * p->topk > 0x7fffffffLL)
        return fail(MOBA_ERR_UNSUPPORTED, "total_tokens * num_q_heads * topk exceeds 2^31");
    const BwdLayout L = make_bwd_layout(*p);
    if (L.max_items > 0x7fffffffLL || (long long)p->num_kv_heads * L.nb_cap > 0x7fffffffLL)
        return fail(MOBA_ERR_UNSUPPORTED, "too many blocks for 32-bit work indices");
    if ((long long)p->num_kv_heads * L.nb_cap * (p->chunk_size / kTileM) > 0x7fffffffLL)
        return fail(MOBA_ERR_UNSUPPORTED, "too many key tiles for one launch");
    if (!workspace || workspace_bytes < L.total)
        return fail(MOBA_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", L.total,
                    workspace ? workspace_bytes : (size_t)0);
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
        return fail(MOBA_ERR_WORKSPACE, "workspace must be 256-byte aligned");

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Problem P = make_problem(*p, L.nb_cap);
    char* base = static_cast<char*>(workspace);
    Workspace ws{};
    ws.hdr = reinterpret_cast<WsHeader*>(base + L.hdr);
    ws.cu_blocks = reinterpret_cast<int*>(base + L.cu_blocks);
    ws.blk_start = reinterpret_cast<int*>(base + L.blk_start);
    ws.blk_len = reinterpret_cast<int*>(base + L.blk_len);
    ws.blk_seq = reinterpret_cast<int*>(base + L.blk_seq);
    ws.blk_local = reinterpret_cast<int*>(base + L.blk_local);
    ws.counts = reinterpret_cast<int*>(base + L.counts);
    ws.offsets = reinterpret_cast<int*>(base + L.offsets);
    ws.cursor = reinterpret_cast<int*>(base + L.cursor);
    ws.item_off = reinterpret_cast<int*>(base + L.item_off);
    ws.entries = reinterpret_cast<int*>(base + L.entries);
    ws.items = reinterpret_cast<WorkItem*>(base + L.items);
    ws.nslots = reinterpret_cast<unsigned char*>(base + L.nslots);
    BwdArgs a;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.k = static_cast<const __nv_bfloat16*>(k);
    a.v = static_cast<const __nv_bfloat16*>(v);
    a.out = static_cast<const __nv_bfloat16*>(out);
    a.dout = static_cast<const __nv_bfloat16*>(d_out);
    a.lse = lse;
    a.dlse = d_lse;
    a.rs = reinterpret_cast<float2*>(base + L.rs);
    a.dq_acc = reinterpret_cast<float*>(base + L.dq_acc);
    a.dq = static_cast<__nv_bfloat16*>(dq);
    a.dk = static_cast<__nv_bfloat16*>(dk);
    a.dv = static_cast<__nv_bfloat16*>(dv);

    const int T = p->total_tokens;
    int launches = 0;
    cudaError_t e;
#define MOBA_TRY(expr, what)                             \
    do {                                                 \
        e = (expr);                                      \
        if (e != cudaSuccess) return cuda_fail(e, what); \
    } while (0)
    {
        NvtxScope stage("route");
        MOBA_TRY(launch_plan_blocks(P, cu_seqlens, ws, st), "block table launch");
        MOBA_TRY(cudaMemsetAsync(ws.counts, 0, 4ull * P.hkv * L.nb_cap, st), "memset");
        MOBA_TRY(launch_route_count(P, cu_seqlens, sel, ws, 0, T, st), "route count launch");
        MOBA_TRY(launch_route_plan(P, ws, 0, T, st), "route plan launch");
        MOBA_TRY(launch_route_scatter(P, cu_seqlens, sel, ws, 0, T, st), "route scatter launch");
        MOBA_TRY(cudaMemsetAsync(a.dq_acc, 0, 4ull * T * P.hq * P.d, st), "memset");
    }
    {
        NvtxScope stage("attention");
        MOBA_TRY(launch_backward(P, a, ws, device_sm_count(), st, &launches), "backward launch");
    }
#undef MOBA_TRY
    return MOBA_OK;
}

// ---- decode step ----------------------------------------------------------------------

namespace {

struct DecodeLayout {
    size_t sel, nsl, part_o, part_lse, total;
};

DecodeLayout make_decode_layout(const moba_params& p) {
    DecodeLayout L;
    const size_t rows = (size_t)p.batch * p.num_q_heads;
    const size_t parts = (size_t)p.topk * decode_splits(p.batch, p.num_q_heads, p.topk, p.chunk_size);
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = align_up(o + bytes);
        return at;
    };
    L.sel = take(4 * rows * p.topk);
    L.nsl = take(4 * rows);
    L.part_o = take(4 * rows * parts * p.head_dim);
    L.part_lse = take(4 * rows * parts);
    L.total = o;
    return L;
}

}  // namespace

size_t moba_decode_workspace_size(const moba_params* p) {
    if (check_params(p) != MOBA_OK) return 0;
    return make_decode_layout(*p).total;
}

namespace {

// The decode step with either block summary (gate.means, or gate.kmin and gate.kmax).
moba_status decode_fwd(const moba_params* p, const void* q, const void* k, const void* v,
                       const int* cu_seqlens, const DecodeGate& gate, void* workspace,
                       size_t ws_bytes, void* out, float* lse, void* stream) {
    moba_status s = check_params(p);
    if (s != MOBA_OK) return s;
    if (p->batch > 65535)
        return fail(MOBA_ERR_UNSUPPORTED, "decode batch %d unsupported (<= 65535)", p->batch);
    const bool summary = gate.means || (gate.kmin && gate.kmax);
    if (!q || !cu_seqlens || !workspace || !out || !lse || (p->total_tokens > 0 && (!k || !v || !summary)))
        return fail(MOBA_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned16(q) || !aligned16(out) || !aligned16(workspace) ||
        (p->total_tokens > 0 && (!aligned16(k) || !aligned16(v) || !aligned16(gate.means) ||
                                 !aligned16(gate.kmin) || !aligned16(gate.kmax))))
        return fail(MOBA_ERR_INVALID_ARG, "q, k, v, the block summary, out and workspace must be 16-byte aligned");
    const DecodeLayout L = make_decode_layout(*p);
    if (ws_bytes < L.total)
        return fail(MOBA_ERR_WORKSPACE, "decode workspace too small: %zu < %zu bytes", ws_bytes, L.total);
    const Problem P = make_problem(*p, blocks_bound(*p));
    uint8_t* base = static_cast<uint8_t*>(workspace);
    DecodeWorkspace ws;
    ws.sel = reinterpret_cast<int*>(base + L.sel);
    ws.nsl = reinterpret_cast<int*>(base + L.nsl);
    ws.part_o = reinterpret_cast<float*>(base + L.part_o);
    ws.part_lse = reinterpret_cast<float*>(base + L.part_lse);
    ws.splits = decode_splits(p->batch, p->num_q_heads, p->topk, p->chunk_size);
    cudaError_t e = launch_decode(P, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                                  static_cast<const __nv_bfloat16*>(v), cu_seqlens, gate, ws,
                                  static_cast<__nv_bfloat16*>(out), lse, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    return MOBA_OK;
}

}  // namespace

moba_status moba_decode_fwd(const moba_params* p, const void* q, const void* k, const void* v,
                            const int* cu_seqlens, const float* k_mean, void* workspace,
                            size_t ws_bytes, void* out, float* lse, void* stream) {
    NvtxScope range("moba_decode_fwd");
    return decode_fwd(p, q, k, v, cu_seqlens, DecodeGate{k_mean, nullptr, nullptr}, workspace, ws_bytes,
                      out, lse, stream);
}

moba_status moba_decode_minmax_fwd(const moba_params* p, const void* q, const void* k, const void* v,
                                   const int* cu_seqlens, const void* k_min, const void* k_max,
                                   void* workspace, size_t ws_bytes, void* out, float* lse,
                                   void* stream) {
    NvtxScope range("moba_decode_minmax_fwd");
    return decode_fwd(p, q, k, v, cu_seqlens,
                      DecodeGate{nullptr, static_cast<const __nv_bfloat16*>(k_min),
                                 static_cast<const __nv_bfloat16*>(k_max)},
                      workspace, ws_bytes, out, lse, stream);
}

moba_status moba_device_status(const moba_params* p, const void* workspace, void* stream) {
    moba_status s = check_params(p);
    if (s != MOBA_OK) return s;
    if (!workspace) return fail(MOBA_ERR_WORKSPACE, "workspace is NULL");
    int word = 0;
    const WsHeader* hdr = static_cast<const WsHeader*>(workspace);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&word, &hdr->status, sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "status read");
    if (word == 0) return MOBA_OK;
    return fail((moba_status)word, "device status word %d", word);
}

// ---------------------------------------------------------------------------------------
// Self-test of the bounded device waits (no counterpart in the pages).  One warp waits on an
// mbarrier that nothing completes, through the same bounded wait the attention and gate
// kernels use, with a short poll limit: the wait must give up, raise the CTA's abort flag and
// record MOBA_ERR_DEVICE_TIMEOUT in the status word.  A wait that wrongly succeeds writes -1.

namespace {

__global__ void __launch_bounds__(32, 1) timeout_probe_kernel(int* status, uint32_t polls) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        moba::ptx::mbar_init(moba::ptx::smem_u32(&bar), 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    const bool ok = moba::ptx::wait_bar(moba::ptx::smem_u32(&bar), 0u,
                                        reinterpret_cast<volatile int*>(&abort_flag), status, polls);
    if (ok && threadIdx.x == 0) atomicExch(status, -1);
}

}  // namespace

extern "C" moba_status moba_selftest_timeout(int* status_dev, unsigned polls, void* stream) {
    if (!status_dev) return fail(MOBA_ERR_INVALID_ARG, "status word is NULL");
    if (polls == 0 || polls > (1u << 20)) return fail(MOBA_ERR_INVALID_ARG, "polls must be in [1, 2^20]");
    timeout_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status_dev, polls);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "timeout probe launch");
    return MOBA_OK;
}

const char* moba_status_string(moba_status s) {
    switch (s) {
        case MOBA_OK: return "MOBA_OK";
        case MOBA_ERR_INVALID_ARG: return "MOBA_ERR_INVALID_ARG";
        case MOBA_ERR_UNSUPPORTED: return "MOBA_ERR_UNSUPPORTED";
        case MOBA_ERR_WORKSPACE: return "MOBA_ERR_WORKSPACE";
        case MOBA_ERR_CUDA: return "MOBA_ERR_CUDA";
        case MOBA_ERR_DEVICE_TIMEOUT: return "MOBA_ERR_DEVICE_TIMEOUT";
    }
    return "MOBA_ERR_UNKNOWN";
}

const char* moba_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
