// Decode step: one new query per sequence against its KV cache.
//
// The analysis page of the MoBA paper (§2.2-§2.3) applied to the query of each sequence's
// last cache row t = L-1 (the new token's key and value are that row): its own block
// c = (L-1) / B is forced and attended whole (every cached token of it precedes or equals t),
// the topk-1 best earlier blocks by q . mean_j are routed, and softmax attention runs over the
// union; per-block partial results are merged by their log-sum-exp (§3.2).  The means are the
// cached fp32 block means of moba_meanpool over the same caches.  The gate may instead score
// with the min/max block summary of moba_minmaxpool: the Quest variant the analysis names
// (§1.3, §5.1 item 6), s_j = sum_i max(q_i kmin_ji, q_i kmax_ji), the largest q . x over the
// block's bounding box.  There is one query row per (sequence, head), so the step streams
// whole K/V blocks and is HBM-bound: it runs on the CUDA cores.
//   decode_gate_kernel   one warp per (sequence, query head): fp32 scores, top-(k-1)
//   decode_attn_kernel   one CTA per (slot, key range, query head, sequence): a selected
//                        block's keys in tiles (a block is cut into several ranges when there
//                        are too few (sequence, head, block) tasks to fill the GPU)
//   decode_merge_kernel  one warp per (sequence, query head)
#include <climits>

#include "moba_internal.cuh"

namespace moba {

namespace {

constexpr int kGateWarps = 8;
constexpr int kAttnThreads = 256;
constexpr int kKeyTile = 64;

// Global index of sequence `seq`'s block 0: the sum of ceil(L_i / chunk) over i < seq (the
// block order of moba_meanpool).  Called by all 32 lanes; every lane gets the answer.
__device__ __forceinline__ int seq_block_base(const int* __restrict__ cu, int seq, int chunk) {
    const int lane = threadIdx.x & 31;
    int base = 0;
    for (int i0 = 0; i0 < seq; i0 += 32) {
        const int i = i0 + lane;
        int n = 0;
        if (i < seq) n = (__ldg(cu + i + 1) - __ldg(cu + i) + chunk - 1) / chunk;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) n += __shfl_xor_sync(0xffffffffu, n, off);
        base += n;
    }
    return base;
}

// Gate score of one block summary row (global block x KV head) for the fp32 query qs[D].
// Mean gate (analysis §2.2): q . mean, fp32 means.
template <int D>
struct MeanScore {
    const float* means;
    __device__ __forceinline__ float operator()(const float* qs, size_t row) const {
        const float4* m = reinterpret_cast<const float4*>(means + row * D);
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
        for (int e = 0; e < D / 4; ++e) {
            const float4 mv = __ldg(m + e);
            a0 = fmaf(qs[4 * e], mv.x, a0);
            a1 = fmaf(qs[4 * e + 1], mv.y, a1);
            a2 = fmaf(qs[4 * e + 2], mv.z, a2);
            a3 = fmaf(qs[4 * e + 3], mv.w, a3);
        }
        return (a0 + a1) + (a2 + a3);
    }
};

// Min/max gate (Quest): sum over channels of max(q_i kmin_i, q_i kmax_i).  q and the
// summaries are bf16 values, so every product is exact in fp32; only the sum rounds.
__device__ __forceinline__ float box_pair(float q0, float q1, uint32_t lo, uint32_t hi) {
    const float t0 = fmaxf(q0 * __uint_as_float(lo << 16), q0 * __uint_as_float(hi << 16));
    const float t1 = fmaxf(q1 * __uint_as_float(lo & 0xffff0000u), q1 * __uint_as_float(hi & 0xffff0000u));
    return t0 + t1;
}

template <int D>
struct MinMaxScore {
    const __nv_bfloat16* kmin;
    const __nv_bfloat16* kmax;
    __device__ __forceinline__ float operator()(const float* qs, size_t row) const {
        const uint4* lo = reinterpret_cast<const uint4*>(kmin + row * D);
        const uint4* hi = reinterpret_cast<const uint4*>(kmax + row * D);
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
        for (int e = 0; e < D / 8; ++e) {
            const uint4 l = __ldg(lo + e), h = __ldg(hi + e);
            const float* qe = qs + 8 * e;
            a0 += box_pair(qe[0], qe[1], l.x, h.x);
            a1 += box_pair(qe[2], qe[3], l.y, h.y);
            a2 += box_pair(qe[4], qe[5], l.z, h.z);
            a3 += box_pair(qe[6], qe[7], l.w, h.w);
        }
        return (a0 + a1) + (a2 + a3);
    }
};

// sel row of (sequence, head) w: slot 0 = own block c, slots 1..n_route = routed past blocks
// (best first), then -1; nsl[w] = 1 + n_route (0 for an empty sequence).
template <int D, int K, class Score>
__global__ void __launch_bounds__(kGateWarps * 32)
decode_gate_kernel(const __nv_bfloat16* __restrict__ q, Score score,
                   const int* __restrict__ cu, Problem P, int* __restrict__ sel,
                   int* __restrict__ nsl) {
    __shared__ float qs[kGateWarps][D];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int w = blockIdx.x * kGateWarps + warp;
    if (w >= P.batch * P.hq) return;  // whole warps leave
    const int seq = w / P.hq, h = w - seq * P.hq, g = h / P.group;
    const int L = __ldg(cu + seq + 1) - __ldg(cu + seq);
    int* srow = sel + (size_t)w * P.topk;
    if (L <= 0) {
        for (int i = lane; i < P.topk; i += 32) srow[i] = -1;
        if (lane == 0) nsl[w] = 0;
        return;
    }
    const int c = (L - 1) / P.chunk;
    const int n_route = min(P.topk - 1, c);
    if (n_route > 0) {
        for (int i = lane; i < D; i += 32) qs[warp][i] = __bfloat162float(q[(size_t)w * D + i]);
        __syncwarp();
        const int b0 = seq_block_base(cu, seq, P.chunk);
        // lane-local candidates j = lane, lane + 32, ... (increasing, so an equal score never
        // displaces an earlier block), kept best-first
        float val[K];
        int idx[K];
#pragma unroll
        for (int i = 0; i < K; ++i) {
            val[i] = -INFINITY;
            idx[i] = INT_MAX;
        }
        for (int j = lane; j < c; j += 32)
            insert_desc<K>(val, idx, score(qs[warp], (size_t)(b0 + j) * P.hkv + g), j, true);
        // n_route rounds of a warp argmax over the lists' heads, order (score desc, index asc)
        for (int r = 0; r < n_route; ++r) {
            float bv = val[0];
            int bi = idx[0];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
                if (ov > bv || (ov == bv && oi < bi)) {
                    bv = ov;
                    bi = oi;
                }
            }
            if (idx[0] == bi) {  // the owner of the winner drops its head
#pragma unroll
                for (int i = 0; i + 1 < K; ++i) {
                    val[i] = val[i + 1];
                    idx[i] = idx[i + 1];
                }
                val[K - 1] = -INFINITY;
                idx[K - 1] = INT_MAX;
            }
            if (lane == 0) srow[1 + r] = bi;
        }
    }
    if (lane == 0) {
        srow[0] = c;
        nsl[w] = 1 + n_route;
    }
    for (int i = 1 + n_route + lane; i < P.topk; i += 32) srow[i] = -1;
}

// One (sequence, head, slot, range): softmax attention of the new query over one key range of
// one selected block, written as a normalised fp32 partial (o, lse); an empty range writes
// o = 0, lse = -inf, which the merge weighs by zero.  Keys stream through shared memory in tiles
// of 64 rows (K and V, 16-byte loads; rows padded by 16 bytes so that the four threads that
// score one key, reading every fourth bf16 pair, hit distinct banks).  Scores are kept in
// log2 units (q pre-scaled by scale * log2 e); the running maximum and sum follow the
// online softmax.
template <int D>
__global__ void __launch_bounds__(kAttnThreads)
decode_attn_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                   const __nv_bfloat16* __restrict__ v, const int* __restrict__ cu, Problem P,
                   const int* __restrict__ sel, const int* __restrict__ nsl,
                   float* __restrict__ part_o, float* __restrict__ part_lse, int splits) {
    constexpr int kRowWords = D / 2 + 4;  // 32-bit words per padded smem row
    constexpr int kSub = kAttnThreads / D;  // threads per output dimension
    __shared__ float2 qs[D / 2];
    __shared__ __align__(16) uint32_t ks[kKeyTile * kRowWords];
    __shared__ __align__(16) uint32_t vs[kKeyTile * kRowWords];
    __shared__ float ps[kKeyTile];
    __shared__ float bcast[2];
    __shared__ float accs[kSub][D];

    const int slot = blockIdx.x / splits, rng = blockIdx.x - slot * splits;
    const int h = blockIdx.y, seq = blockIdx.z;
    const int w = seq * P.hq + h;
    if (slot >= __ldg(nsl + w)) return;  // uniform over the CTA
    const int j = __ldg(sel + (size_t)w * P.topk + slot);
    const int start = __ldg(cu + seq), L = __ldg(cu + seq + 1) - start;
    const int b0 = start + j * P.chunk, b1 = start + min((j + 1) * P.chunk, L);
    // this CTA's range: whole 64-key tiles of the block, cut into `splits` contiguous parts
    const int per = ((b1 - b0 + kKeyTile - 1) / kKeyTile + splits - 1) / splits * kKeyTile;
    const int k0 = b0 + rng * per, k1 = min(b1, k0 + per);
    const int g = h / P.group;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t pi = ((size_t)w * P.topk + slot) * splits + rng;
    if (k0 >= k1) {
        if (tid < D) part_o[pi * D + tid] = 0.f;
        if (tid == 0) part_lse[pi] = -INFINITY;
        return;
    }

    for (int i = tid; i < D / 2; i += kAttnThreads) {
        const __nv_bfloat162 b2 = reinterpret_cast<const __nv_bfloat162*>(q + (size_t)w * D)[i];
        const float2 f = __bfloat1622float2(b2);
        qs[i] = make_float2(f.x * P.scale_log2, f.y * P.scale_log2);
    }
    float m = -INFINITY, l = 0.f;  // running max (log2 units) and sum; kept by warp 0
    float acc = 0.f;               // output dimension tid % D over keys tid / D, tid / D + kSub ...
    const int dim = tid % D, sub = tid / D;
    const int key = tid >> 2, part = tid & 3;  // scoring: four threads per key

    for (int kt = k0; kt < k1; kt += kKeyTile) {
        const int nk = min(kKeyTile, k1 - kt);
        __syncthreads();  // the previous tile is consumed (and qs is written)
        for (int e = tid; e < nk * (D / 8); e += kAttnThreads) {
            const int r = e / (D / 8), cc = e - r * (D / 8);
            const size_t src = ((size_t)(kt + r) * P.hkv + g) * D + cc * 8;
            *reinterpret_cast<uint4*>(&ks[r * kRowWords + cc * 4]) = __ldg(reinterpret_cast<const uint4*>(k + src));
            *reinterpret_cast<uint4*>(&vs[r * kRowWords + cc * 4]) = __ldg(reinterpret_cast<const uint4*>(v + src));
        }
        __syncthreads();
        // scores: thread (key, part) sums bf16 pairs part, part + 4, ... of the key's row
        float sdot = 0.f;
        if (key < nk) {
#pragma unroll 8
            for (int p2 = part; p2 < D / 2; p2 += 4) {
                const uint32_t wv = ks[key * kRowWords + p2];
                const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv));
                const float2 qf = qs[p2];
                sdot = fmaf(qf.x, kf.x, fmaf(qf.y, kf.y, sdot));
            }
        }
        sdot += __shfl_xor_sync(0xffffffffu, sdot, 1);
        sdot += __shfl_xor_sync(0xffffffffu, sdot, 2);
        if (part == 0) ps[key] = (key < nk) ? sdot : -INFINITY;
        __syncthreads();
        if (warp == 0) {
            const float a = ps[lane], b = ps[lane + 32];
            float tmax = fmaxf(a, b);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
            const float mn = fmaxf(m, tmax);
            const float alpha = exp2f(m - mn);
            const float pa = exp2f(a - mn), pb = exp2f(b - mn);
            ps[lane] = pa;
            ps[lane + 32] = pb;
            float ts = pa + pb;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ts += __shfl_xor_sync(0xffffffffu, ts, off);
            l = l * alpha + ts;
            m = mn;
            if (lane == 0) bcast[0] = alpha;
        }
        __syncthreads();
        acc *= bcast[0];
        for (int kk = sub; kk < nk; kk += kSub) {
            const uint32_t wv = vs[kk * kRowWords + (dim >> 1)];
            const float2 vf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv));
            acc = fmaf(ps[kk], (dim & 1) ? vf.y : vf.x, acc);
        }
    }
    __syncthreads();  // every thread has read the last tile's rescale factor
    accs[sub][dim] = acc;
    if (tid == 0) {
        bcast[0] = l;
        bcast[1] = m;
    }
    __syncthreads();
    if (tid < D) {
        float o = 0.f;
#pragma unroll
        for (int s = 0; s < kSub; ++s) o += accs[s][tid];
        part_o[pi * D + tid] = o / bcast[0];
        if (tid == 0) part_lse[pi] = bcast[1] * 0.69314718055994531f + logf(bcast[0]);
    }
}

// out[seq, h] = sum_i e^(lse_i - m) o_i / sum_i e^(lse_i - m) over the row's slots, in fp32,
// rounded once to bf16; lse[h, seq] = m + log sum_i e^(lse_i - m).  An empty sequence has no
// query: zeros and -inf.
template <int D>
__global__ void __launch_bounds__(kGateWarps * 32)
decode_merge_kernel(const int* __restrict__ nsl, const float* __restrict__ part_o,
                    const float* __restrict__ part_lse, Problem P, __nv_bfloat16* __restrict__ out,
                    float* __restrict__ lse, int splits) {
    constexpr int V = D / 32;  // channels per lane
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int w = blockIdx.x * kGateWarps + warp;
    if (w >= P.batch * P.hq) return;
    const int seq = w / P.hq, h = w - seq * P.hq;
    const int ns = __ldg(nsl + w) * splits;  // partials of the row: its blocks' key ranges
    __nv_bfloat16* dst = out + (size_t)w * D + lane * V;
    if (ns == 0) {
#pragma unroll
        for (int e = 0; e < V; ++e) dst[e] = __float2bfloat16(0.f);
        if (lane == 0) lse[(size_t)h * P.batch + seq] = -INFINITY;
        return;
    }
    const size_t pbase = (size_t)w * P.topk * splits;
    // lane s holds partials s and s + 32 (at most 64 per row)
    const float la = (lane < ns) ? __ldg(part_lse + pbase + lane) : -INFINITY;
    const float lb = (lane + 32 < ns) ? __ldg(part_lse + pbase + lane + 32) : -INFINITY;
    float mx = fmaxf(la, lb);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float wa = (lane < ns) ? expf(la - mx) : 0.f;
    const float wb = (lane + 32 < ns) ? expf(lb - mx) : 0.f;
    float L = wa + wb;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
    for (int i = 0; i < ns; ++i) {
        const float wgt = (i < 32) ? __shfl_sync(0xffffffffu, wa, i & 31) : __shfl_sync(0xffffffffu, wb, i & 31);
        const float* src = part_o + (pbase + i) * D + lane * V;
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = fmaf(wgt, __ldg(src + e), acc[e]);
    }
    const float inv = 1.f / L;
#pragma unroll
    for (int e = 0; e < V; ++e) dst[e] = __float2bfloat16_rn(acc[e] * inv);
    if (lane == 0) lse[(size_t)h * P.batch + seq] = mx + logf(L);
}

template <int D, class Score>
void launch_decode_gate(const Problem& P, const __nv_bfloat16* q, Score score, const int* cu,
                        const DecodeWorkspace& ws, cudaStream_t st) {
    const int row_blocks = (P.batch * P.hq + kGateWarps - 1) / kGateWarps;
    const int route = P.topk - 1;  // list size must hold every routed block of one lane
    if (route <= 4)
        decode_gate_kernel<D, 4><<<row_blocks, kGateWarps * 32, 0, st>>>(q, score, cu, P, ws.sel, ws.nsl);
    else if (route <= 8)
        decode_gate_kernel<D, 8><<<row_blocks, kGateWarps * 32, 0, st>>>(q, score, cu, P, ws.sel, ws.nsl);
    else if (route <= 16)
        decode_gate_kernel<D, 16><<<row_blocks, kGateWarps * 32, 0, st>>>(q, score, cu, P, ws.sel, ws.nsl);
    else
        decode_gate_kernel<D, 32><<<row_blocks, kGateWarps * 32, 0, st>>>(q, score, cu, P, ws.sel, ws.nsl);
}

template <int D>
cudaError_t launch_decode_d(const Problem& P, const __nv_bfloat16* q, const __nv_bfloat16* k,
                            const __nv_bfloat16* v, const int* cu, const DecodeGate& gate,
                            const DecodeWorkspace& ws, __nv_bfloat16* out, float* lse,
                            cudaStream_t st) {
    const int rows = P.batch * P.hq;
    const int row_blocks = (rows + kGateWarps - 1) / kGateWarps;
    if (gate.means)
        launch_decode_gate<D>(P, q, MeanScore<D>{gate.means}, cu, ws, st);
    else
        launch_decode_gate<D>(P, q, MinMaxScore<D>{gate.kmin, gate.kmax}, cu, ws, st);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_attn_kernel<D><<<dim3(P.topk * ws.splits, P.hq, P.batch), kAttnThreads, 0, st>>>(
        q, k, v, cu, P, ws.sel, ws.nsl, ws.part_o, ws.part_lse, ws.splits);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_merge_kernel<D><<<row_blocks, kGateWarps * 32, 0, st>>>(ws.nsl, ws.part_o, ws.part_lse, P, out, lse,
                                                                   ws.splits);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const Problem& P, const __nv_bfloat16* q, const __nv_bfloat16* k,
                          const __nv_bfloat16* v, const int* cu_seqlens, const DecodeGate& gate,
                          const DecodeWorkspace& ws, __nv_bfloat16* out, float* lse,
                          cudaStream_t st) {
    if (P.d == 64) return launch_decode_d<64>(P, q, k, v, cu_seqlens, gate, ws, out, lse, st);
    return launch_decode_d<128>(P, q, k, v, cu_seqlens, gate, ws, out, lse, st);
}

}  // namespace moba
