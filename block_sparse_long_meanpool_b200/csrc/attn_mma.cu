// Step 5 of the forward, warp-level tensor-core version: attention of 128-row work items
// against one KV block, producing a partial (o, lse) per row and slot.
//
// The analysis page of the MoBA paper (§3.2): history blocks are attended without a causal
// mask (rule 1 of §2.3 already excluded every future block), the own block with a causal
// mask, and the partial softmax results are merged afterwards by their log-sum-exp.
//
// Work items come from the routing pass: a history tile is up to 128 routed rows (any query
// heads of one KV head) against one whole block; a current-block tile is 128 consecutive
// tokens of one query head against the causal prefix of their own block.  A persistent grid
// takes items from an atomic cursor, history tiles first and current-block tiles largest
// first.  Each CTA is 8 warps x 16 rows; keys stream through a 2-stage cp.async pipeline of
// 64-key chunks; QK^T and PV use mma.sync m16n8k16 bf16 with fp32 accumulation and an
// online softmax in the exp2 domain.
#include <climits>

#include "moba_internal.cuh"

namespace moba {

namespace {

constexpr int kThreads = 256;  // 8 warps x 16 rows = kTileM rows
constexpr int kN = 64;         // keys per pipeline stage

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    const int sz = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(sz));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;\n" ::); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Byte offset of 16-byte chunk ck of row r in a tile of D bf16 per row, XOR-swizzled so that
// 8 consecutive rows at the same chunk land in 8 different bank groups.
template <int D>
__device__ __forceinline__ uint32_t swz(int r, int ck) {
    return r * (D * 2) + ((ck ^ (r & 7)) << 4);
}

template <int D>
struct Smem {
    __nv_bfloat16 q[kTileM * D];
    __nv_bfloat16 k[2][kN * D];
    __nv_bfloat16 v[2][kN * D];
};

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
attn_mma_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                const __nv_bfloat16* __restrict__ v, Problem P, Workspace ws, int t0, int t1) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    Smem<D>& sm = *reinterpret_cast<Smem<D>*>(smem_raw);
    __shared__ long long s_qoff[kTileM];
    __shared__ int s_pidx[kTileM];
    __shared__ int s_tlim[kTileM];
    __shared__ int s_item;

    constexpr int CK = D / 8;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g4 = lane >> 2, t4 = lane & 3;
    const int n_items = ws.hdr->n_items;
    const uint32_t q_s = smem_u32(sm.q);

    for (;;) {
        if (tid == 0) s_item = (int)atomicAdd(&ws.hdr->work_counter, 1u);
        __syncthreads();
        const int it_idx = s_item;
        if (it_idx >= n_items) break;
        const WorkItem it = ws.items[it_idx];
        int g, key_start, key_end;
        if (it.kind == 0) {
            g = it.a / P.nb_cap;
            const int b = it.a - g * P.nb_cap;
            key_start = ws.blk_start[b];
            key_end = key_start + ws.blk_len[b];
            if (tid < kTileM) {
                if (tid < it.c) {
                    const int pidx = ws.entries[it.b + tid];
                    const int rid = pidx / P.topk;
                    const int t = t0 + rid / P.hq;
                    const int h = rid - (rid / P.hq) * P.hq;
                    s_qoff[tid] = ((long long)t * P.hq + h) * D;
                    s_pidx[tid] = pidx;
                } else {
                    s_qoff[tid] = -1;
                    s_pidx[tid] = -1;
                }
                s_tlim[tid] = INT_MAX;
            }
        } else {
            const int b = it.a, h = it.b, qt = it.c;
            g = h / P.group;
            key_start = ws.blk_start[b];
            const int len = ws.blk_len[b];
            key_end = key_start + min((qt + 1) * kTileM, len);
            if (tid < kTileM) {
                const int rr = qt * kTileM + tid;
                const int t = key_start + rr;
                const bool ok = rr < len && t >= t0 && t < t1;
                s_qoff[tid] = ok ? ((long long)t * P.hq + h) * D : -1;
                s_pidx[tid] = ok ? ((t - t0) * P.hq + h) * P.topk : -1;
                s_tlim[tid] = ok ? t : INT_MAX;
            }
        }
        __syncthreads();

        for (int e = tid; e < kTileM * CK; e += kThreads) {
            const int r = e / CK, ck = e - (e / CK) * CK;
            const long long off = s_qoff[r];
            cp_async16(q_s + swz<D>(r, ck), off >= 0 ? q + off + ck * 8 : q, off >= 0);
        }
        auto load_kv = [&](int chunk, int stage) {
            const int kb = key_start + chunk * kN;
            const uint32_t ks = smem_u32(sm.k[stage]), vs = smem_u32(sm.v[stage]);
            for (int e = tid; e < kN * CK; e += kThreads) {
                const int r = e / CK, ck = e - (e / CK) * CK;
                const int key = kb + r;
                const bool ok = key < key_end;
                const size_t off = ((size_t)(ok ? key : key_start) * P.hkv + g) * D + ck * 8;
                cp_async16(ks + swz<D>(r, ck), k + off, ok);
                cp_async16(vs + swz<D>(r, ck), v + off, ok);
            }
        };
        load_kv(0, 0);
        cp_async_commit();
        const int nchunks = (key_end - key_start + kN - 1) / kN;

        float o[D / 8][4];
#pragma unroll
        for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        const int row0 = warp * 16;
        const int tl0 = s_tlim[row0 + g4], tl1 = s_tlim[row0 + g4 + 8];

        for (int n = 0; n < nchunks; ++n) {
            if (n + 1 < nchunks) load_kv(n + 1, (n + 1) & 1);
            cp_async_commit();
            cp_async_wait1();
            __syncthreads();
            const uint32_t ks = smem_u32(sm.k[n & 1]), vs = smem_u32(sm.v[n & 1]);
            float s[kN / 8][4];
#pragma unroll
            for (int i = 0; i < kN / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                // Q fragment of this k-step, re-read from shared memory (keeps registers for O)
                uint32_t qf[4];
                {
                    const int mi = lane >> 3;
                    const int r = row0 + (mi & 1) * 8 + (lane & 7);
                    const int ck = kk * 2 + (mi >> 1);
                    ldsm_x4(q_s + swz<D>(r, ck), qf[0], qf[1], qf[2], qf[3]);
                }
#pragma unroll
                for (int np = 0; np < kN / 16; ++np) {
                    const int mi = lane >> 3;
                    const int key = np * 16 + (mi >> 1) * 8 + (lane & 7);
                    const int ck = kk * 2 + (mi & 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(ks + swz<D>(key, ck), b0, b1, b2, b3);
                    mma16816(s[2 * np], qf, b0, b1);
                    mma16816(s[2 * np + 1], qf, b2, b3);
                }
            }
            // scale into the exp2 domain, mask keys past the block / after the row
            const int kb = key_start + n * kN;
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < kN / 8; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = kb + nt * 8 + 2 * t4 + (e & 1);
                    const int tl = (e < 2) ? tl0 : tl1;
                    const bool ok = key < key_end && key <= tl;
                    const float x = ok ? s[nt][e] * P.scale_log2 : -INFINITY;
                    s[nt][e] = x;
                    if (e < 2) mx0 = fmaxf(mx0, x); else mx1 = fmaxf(mx1, x);
                }
            }
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
            const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
            const float b0f = (mn0 == -INFINITY) ? 0.f : mn0;
            const float b1f = (mn1 == -INFINITY) ? 0.f : mn1;
            const float al0 = exp2f(m0 - b0f), al1 = exp2f(m1 - b1f);
            m0 = mn0;
            m1 = mn1;
            float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
            for (int nt = 0; nt < kN / 8; ++nt) {
                s[nt][0] = exp2f(s[nt][0] - b0f);
                s[nt][1] = exp2f(s[nt][1] - b0f);
                s[nt][2] = exp2f(s[nt][2] - b1f);
                s[nt][3] = exp2f(s[nt][3] - b1f);
                rs0 += s[nt][0] + s[nt][1];
                rs1 += s[nt][2] + s[nt][3];
            }
            l0 = l0 * al0 + rs0;
            l1 = l1 * al1 + rs1;
#pragma unroll
            for (int i = 0; i < D / 8; ++i) {
                o[i][0] *= al0;
                o[i][1] *= al0;
                o[i][2] *= al1;
                o[i][3] *= al1;
            }
#pragma unroll
            for (int kk = 0; kk < kN / 16; ++kk) {
                uint32_t a[4];
                a[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
                a[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
                a[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
                a[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
                for (int np = 0; np < D / 16; ++np) {
                    const int mi = lane >> 3;
                    const int key = kk * 16 + (mi & 1) * 8 + (lane & 7);
                    const int ck = np * 2 + (mi >> 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(vs + swz<D>(key, ck), b0, b1, b2, b3);
                    mma16816(o[2 * np], a, b0, b1);
                    mma16816(o[2 * np + 1], a, b2, b3);
                }
            }
            __syncthreads();
        }

        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
        const int p0 = s_pidx[row0 + g4], p1 = s_pidx[row0 + g4 + 8];
        const float ln2 = 0.69314718055994531f;
        if (p0 >= 0) {
            const float inv = 1.f / l0;
            float* dst = ws.part_o + (size_t)p0 * D + 2 * t4;
#pragma unroll
            for (int i = 0; i < D / 8; ++i)
                *reinterpret_cast<float2*>(dst + i * 8) = make_float2(o[i][0] * inv, o[i][1] * inv);
            if (t4 == 0) ws.part_lse[p0] = m0 * ln2 + logf(l0);
        }
        if (p1 >= 0) {
            const float inv = 1.f / l1;
            float* dst = ws.part_o + (size_t)p1 * D + 2 * t4;
#pragma unroll
            for (int i = 0; i < D / 8; ++i)
                *reinterpret_cast<float2*>(dst + i * 8) = make_float2(o[i][2] * inv, o[i][3] * inv);
            if (t4 == 0) ws.part_lse[p1] = m1 * ln2 + logf(l1);
        }
    }
}

template <int D>
cudaError_t launch_attn_d(const Problem& P, const __nv_bfloat16* q, const __nv_bfloat16* k,
                          const __nv_bfloat16* v, const Workspace& ws, int t0, int t1, int num_sms,
                          cudaStream_t st) {
    const int smem = (int)sizeof(Smem<D>);
    cudaError_t e = cudaFuncSetAttribute(attn_mma_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_mma_kernel<D><<<num_sms * 2, kThreads, smem, st>>>(q, k, v, P, ws, t0, t1);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const Problem& P, const __nv_bfloat16* q, const __nv_bfloat16* k,
                             const __nv_bfloat16* v, const Workspace& ws, int t0, int t1,
                             int num_sms, cudaStream_t st) {
    if (P.d == 64) return launch_attn_d<64>(P, q, k, v, ws, t0, t1, num_sms, st);
    return launch_attn_d<128>(P, q, k, v, ws, t0, t1, num_sms, st);
}

}  // namespace moba
