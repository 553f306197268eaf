// attention.cuh — grouped-query attention of block (or prefix) queries over the KV arena.
//
// One CTA serves one sequence, one KV head and 64 packed query rows: packed row r is query
// head kvh*G + (r % G) at position pos0 + r / G, so the G query heads sharing a KV head
// share every K/V tile load.  K/V tiles of 64 keys are staged in shared memory with
// cp.async (double-buffered, zero-filled past the last key, XOR-swizzled 16-byte chunks);
// QK^T and PV run on mma.sync (bf16 in, f32 accumulate) with an online softmax in the
// exp2 domain.  With n_splits > 1 the keys are split across CTAs (flash-decoding); the CTA
// that finishes a query tile last merges the partial (max, sum, O) triples in split order.
#pragma once
#include "common.cuh"

namespace attn {

struct Params {
    const bf16 *q;        // packed: q[((j * nkv + kvh) * G * rows_per_seq + position * G + g) * HD + d]
    int q_ld;
    const bf16 *kc, *vc;  // this slot's K/V: + b * seq_stride + kvh * head_stride + pos * HD
    long long seq_stride, head_stride;
    RowMap map;
    int G, nq, kv_len, causal;
    int n_splits, keys_per_split;  // keys_per_split a multiple of 64
    bf16 *out;                     // out[m * out_ld + h * HD + d] (n_splits == 1)
    int out_ld;
    float *ws_o, *ws_ml;           // partials (n_splits > 1): [split][m][h][HD] and [split][m][h][2]
    int *counters;                 // per (sequence, kv head, query tile): splits done (left at zero)
    int m_rows;                    // rows of the whole launch (for partial indexing)
    float scale_log2;              // log2(e) / sqrt(HD)
};

__device__ __forceinline__ void cp_async16(void *dst, const void *src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// element offset of 16-byte chunk `ch` of row `r` in a swizzled [rows][HD] bf16 tile
template <int HD>
__device__ __forceinline__ int swz(int r, int ch) {
    return r * HD + ((ch ^ (r & 7)) << 3);
}

template <int HD>
__global__ void __launch_bounds__(128) attn_kernel(Params p) {
    constexpr int CPR = HD / 8;  // 16-byte chunks per row
    constexpr int ND = HD / 8;   // 8-wide d tiles of the output
    extern __shared__ __align__(128) uint8_t sm[];
    bf16 *sQ = reinterpret_cast<bf16 *>(sm);
    bf16 *sK = sQ + 64 * HD;
    bf16 *sV = sK + 2 * 64 * HD;

    pdl_enter();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g8 = lane >> 2, t4 = lane & 3;
    const int j = blockIdx.z;
    const int kvh = blockIdx.y / p.n_splits, split = blockIdx.y % p.n_splits;
    const int b = p.map.seq_of[j];
    const int Tq = p.map.rows_per_seq;
    const int stride_packed = p.G * Tq;  // packed q rows per (sequence slot, kv head)
    // rows of this sequence slot (fewer than Tq when the rows are compacted) and their positions
    const int seq_rows = p.map.seq_cnt ? p.map.seq_cnt[j] : Tq;
    const int off = p.map.seq_off ? p.map.seq_off[j] : j * Tq;
    const int rows_packed = p.G * seq_rows;
    const int r0 = blockIdx.x * 64;
    if (r0 >= rows_packed) return;  // uniform: no query rows in this tile
    auto pos_of = [&](int u) { return p.map.pos0 + (p.map.row_t ? p.map.row_t[off + u] : u); };

    // key range of this CTA
    int kstart = split * p.keys_per_split;
    int kend = min(p.kv_len, kstart + p.keys_per_split);
    if (p.causal) {
        const int last = min(r0 + 63, rows_packed - 1);
        kend = min(kend, pos_of(last / p.G) + 1);
    }

    // Q tile
    for (int c = tid; c < 64 * CPR; c += 128) {
        const int r = c / CPR, ch = c % CPR, rp = r0 + r;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (rp < rows_packed)
            val = *reinterpret_cast<const uint4 *>(p.q + (((long long)j * (p.nq / p.G) + kvh) * stride_packed + rp) * HD +
                                                   ch * 8);
        *reinterpret_cast<uint4 *>(sQ + swz<HD>(r, ch)) = val;
    }

    const bf16 *kbase = p.kc + (long long)b * p.seq_stride + (long long)kvh * p.head_stride;
    const bf16 *vbase = p.vc + (long long)b * p.seq_stride + (long long)kvh * p.head_stride;
    auto load_tile = [&](int buf, int k0) {
        for (int c = tid; c < 64 * CPR; c += 128) {
            const int r = c / CPR, ch = c % CPR, key = k0 + r;
            const bool ok = key < kend;
            const long long off = (long long)(ok ? key : 0) * HD + ch * 8;
            cp_async16(sK + buf * 64 * HD + swz<HD>(r, ch), kbase + off, ok ? 16 : 0);
            cp_async16(sV + buf * 64 * HD + swz<HD>(r, ch), vbase + off, ok ? 16 : 0);
        }
        cp_async_commit();
    };

    const int n_tiles = kend > kstart ? (kend - kstart + 63) / 64 : 0;
    if (n_tiles > 0) load_tile(0, kstart);
    __syncthreads();  // Q tile visible

    // this thread's two rows (g8 and g8 + 8 of the warp's 16) and their positions
    int qpos[2];
    bool rvalid[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int rp = r0 + warp * 16 + g8 + i * 8;
        rvalid[i] = rp < rows_packed;
        qpos[i] = rvalid[i] ? pos_of(rp / p.G) : p.map.pos0;
    }

    uint32_t qf[HD / 16][4];
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
        const int r = warp * 16 + (lane & 15), ch = kk * 2 + (lane >> 4);
        ldsm_x4(smem_u32(sQ + swz<HD>(r, ch)), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
    }

    float o[ND][4];
#pragma unroll
    for (int i = 0; i < ND; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_run[2] = {-1e30f, -1e30f}, l_run[2] = {0.f, 0.f};

    for (int it = 0; it < n_tiles; ++it) {
        const int buf = it & 1;
        const int k0 = kstart + it * 64;
        if (it + 1 < n_tiles) {
            load_tile(buf ^ 1, k0 + 64);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const bf16 *tK = sK + buf * 64 * HD;
        const bf16 *tV = sV + buf * 64 * HD;

        float s[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
                const int ch = kk * 2 + ((lane >> 3) & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(smem_u32(tK + swz<HD>(key, ch)), b0, b1, b2, b3);
                mma_bf16_16816(s[2 * np], qf[kk], b0, b1);
                mma_bf16_16816(s[2 * np + 1], qf[kk], b2, b3);
            }
        }
        // scale, mask, online softmax
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int ri = e >> 1;
                const int key = k0 + nt * 8 + 2 * t4 + (e & 1);
                const bool ok = key < kend && (!p.causal || key <= qpos[ri]);
                const float v = ok ? s[nt][e] * p.scale_log2 : -INFINITY;
                s[nt][e] = v;
                mx[ri] = fmaxf(mx[ri], v);
            }
        }
#pragma unroll
        for (int ri = 0; ri < 2; ++ri) {
            mx[ri] = fmaxf(mx[ri], __shfl_xor_sync(0xffffffffu, mx[ri], 1));
            mx[ri] = fmaxf(mx[ri], __shfl_xor_sync(0xffffffffu, mx[ri], 2));
        }
        float corr[2];
#pragma unroll
        for (int ri = 0; ri < 2; ++ri) {
            const float m_new = fmaxf(m_run[ri], mx[ri]);
            corr[ri] = exp2f(m_run[ri] - m_new);
            m_run[ri] = m_new;
            l_run[ri] *= corr[ri];
        }
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float pv = exp2f(s[nt][e] - m_run[e >> 1]);
                s[nt][e] = pv;
                l_run[e >> 1] += pv;
            }
        }
#pragma unroll
        for (int dt = 0; dt < ND; ++dt) {
            o[dt][0] *= corr[0];
            o[dt][1] *= corr[0];
            o[dt][2] *= corr[1];
            o[dt][3] *= corr[1];
        }
        // O += P V
#pragma unroll
        for (int kk2 = 0; kk2 < 4; ++kk2) {
            uint32_t a[4];
            a[0] = pack_bf16(s[2 * kk2][0], s[2 * kk2][1]);
            a[1] = pack_bf16(s[2 * kk2][2], s[2 * kk2][3]);
            a[2] = pack_bf16(s[2 * kk2 + 1][0], s[2 * kk2 + 1][1]);
            a[3] = pack_bf16(s[2 * kk2 + 1][2], s[2 * kk2 + 1][3]);
#pragma unroll
            for (int dp = 0; dp < ND / 2; ++dp) {
                const int key = kk2 * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                const int ch = dp * 2 + (lane >> 4);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(smem_u32(tV + swz<HD>(key, ch)), b0, b1, b2, b3);
                mma_bf16_16816(o[2 * dp], a, b0, b1);
                mma_bf16_16816(o[2 * dp + 1], a, b2, b3);
            }
        }
        __syncthreads();  // buffer `buf` is refilled two iterations later
    }

    // finish: quad-reduce the row sums, write normalised output or the split partials
#pragma unroll
    for (int ri = 0; ri < 2; ++ri) {
        l_run[ri] += __shfl_xor_sync(0xffffffffu, l_run[ri], 1);
        l_run[ri] += __shfl_xor_sync(0xffffffffu, l_run[ri], 2);
    }
#pragma unroll
    for (int ri = 0; ri < 2; ++ri) {
        if (!rvalid[ri]) continue;
        const int rp = r0 + warp * 16 + g8 + ri * 8;
        const int t = rp / p.G, h = kvh * p.G + rp % p.G;
        const int m = off + t;
        if (p.n_splits == 1) {
            const float inv = l_run[ri] > 0.f ? 1.f / l_run[ri] : 0.f;
            bf16 *dst = p.out + (long long)m * p.out_ld + h * HD;
#pragma unroll
            for (int dt = 0; dt < ND; ++dt) {
                const int d = dt * 8 + 2 * t4;
                *reinterpret_cast<__nv_bfloat162 *>(dst + d) =
                    __floats2bfloat162_rn(o[dt][2 * ri] * inv, o[dt][2 * ri + 1] * inv);
            }
        } else {
            const long long row = ((long long)split * p.m_rows + m) * p.nq + h;
            float *dst = p.ws_o + row * HD;
#pragma unroll
            for (int dt = 0; dt < ND; ++dt) {
                const int d = dt * 8 + 2 * t4;
                *reinterpret_cast<float2 *>(dst + d) = make_float2(o[dt][2 * ri], o[dt][2 * ri + 1]);
            }
            if (t4 == 0) {
                p.ws_ml[row * 2 + 0] = m_run[ri];
                p.ws_ml[row * 2 + 1] = l_run[ri];
            }
        }
    }
    if (p.n_splits == 1) return;

    // The CTA that finishes a (sequence, kv head, query tile) last merges the split partials in
    // split order: O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s (deterministic).
    __shared__ int last;
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        int *cnt = p.counters + ((long long)j * gridDim.y / p.n_splits + kvh) * gridDim.x + blockIdx.x;
        const int prev = atomicAdd(cnt, 1);
        last = prev == p.n_splits - 1;
        if (last) *cnt = 0;
    }
    __syncthreads();
    if (!last) return;
    __threadfence();
    const int rows_here = min(64, rows_packed - r0);
    for (int idx = tid; idx < rows_here * (HD / 4); idx += 128) {
        const int rl = idx / (HD / 4), d = (idx % (HD / 4)) * 4;
        const int rp = r0 + rl;
        const int t = rp / p.G, h = kvh * p.G + rp % p.G;
        const int m = off + t;
        float M = -INFINITY;
        for (int s = 0; s < p.n_splits; ++s)
            M = fmaxf(M, __ldcg(p.ws_ml + (((long long)s * p.m_rows + m) * p.nq + h) * 2));
        float L = 0.f, a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        for (int s = 0; s < p.n_splits; ++s) {
            const long long row = ((long long)s * p.m_rows + m) * p.nq + h;
            const float w = exp2f(__ldcg(p.ws_ml + row * 2) - M);
            L += w * __ldcg(p.ws_ml + row * 2 + 1);
            const float4 o4 = __ldcg(reinterpret_cast<const float4 *>(p.ws_o + row * HD + d));
            a0 += w * o4.x;
            a1 += w * o4.y;
            a2 += w * o4.z;
            a3 += w * o4.w;
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        bf16 *dst = p.out + (long long)m * p.out_ld + h * HD + d;
        *reinterpret_cast<__nv_bfloat162 *>(dst) = __floats2bfloat162_rn(a0 * inv, a1 * inv);
        *reinterpret_cast<__nv_bfloat162 *>(dst + 2) = __floats2bfloat162_rn(a2 * inv, a3 * inv);
    }
}

}  // namespace attn
