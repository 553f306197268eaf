// kernels.cuh — the non-GEMM kernels of the ALoDLM step: embedding gather, RMSNorm,
// q/k norm + RoPE + KV-arena write, depth fallback copy, readout norm + ExitGate, the
// fixed-order LM-head combine (entropy, argmax, cumulative halting), the commit/merge
// kernel and the loop planner that compacts rows between loops.
#pragma once
#include "common.cuh"

namespace k {

// ---------------------------------------------------------------------------------
// set-up
// ---------------------------------------------------------------------------------

// dst[r, :] = bf16(src[src_row(r), :]) with src_row from an optional row map
__global__ void pack_rows_kernel(const void *src, int src_is_f32, long long src_ld, const int *row_map, int n_rows,
                                 int n_cols, bf16 *dst, long long dst_ld) {
    const int r = blockIdx.x;
    if (r >= n_rows) return;
    const long long sr = row_map ? row_map[r] : r;
    for (int c = threadIdx.x; c < n_cols; c += blockDim.x) {
        bf16 v;
        if (src_is_f32)
            v = __float2bfloat16_rn(static_cast<const float *>(src)[sr * src_ld + c]);
        else
            v = static_cast<const bf16 *>(src)[sr * src_ld + c];
        dst[(long long)r * dst_ld + c] = v;
    }
}

// Gate/up interleave for the fused SwiGLU epilogue: groups of 32 rows hold 16 gate rows then
// the 16 up rows of the same 16 features.
__global__ void pack_gate_up_kernel(const void *gate, const void *up, int src_is_f32, int I, int H, bf16 *dst) {
    const int r = blockIdx.x;
    const int grp = r >> 5, wi = r & 31;
    const void *src = wi < 16 ? gate : up;
    const long long sr = grp * 16 + (wi & 15);
    for (int c = threadIdx.x; c < H; c += blockDim.x) {
        bf16 v;
        if (src_is_f32)
            v = __float2bfloat16_rn(static_cast<const float *>(src)[sr * H + c]);
        else
            v = static_cast<const bf16 *>(src)[sr * H + c];
        dst[(long long)r * H + c] = v;
    }
}

// Tiled weight layout: tile (rt, kt) = rows [rt*RT, rt*RT+RT) x columns [kt*64, kt*64+64) of the
// row-major source, stored contiguously (RT x 64, row-major) at tile index rt*KT + kt; columns
// past `cols` are zero.  One block per tile.
__global__ void tile_matrix_kernel(const bf16 *src, int rows, int cols, int RT, int KT, bf16 *dst) {
    const int rt = blockIdx.x / KT, kt = blockIdx.x % KT;
    bf16 *d = dst + (long long)blockIdx.x * RT * 64;
    for (int idx = threadIdx.x; idx < RT * 64; idx += blockDim.x) {
        const int r = idx >> 6, c = idx & 63;
        const int row = rt * RT + r, col = kt * 64 + c;
        d[idx] = (row < rows && col < cols) ? src[(long long)row * cols + col] : __float2bfloat16_rn(0.f);
    }
}

// rope[pos][j] = (cos, sin)(pos * base^(-2j/hd)), evaluated in double precision
__global__ void rope_table_kernel(float2 *rope, int n_pos, int half, double base) {
    const long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (idx >= (long long)n_pos * half) return;
    const int pos = (int)(idx / half), jj = (int)(idx % half);
    const double inv = pow(base, -2.0 * jj / (2.0 * half));
    double s, c;
    sincos((double)pos * inv, &s, &c);
    rope[idx] = make_float2((float)c, (float)s);
}

// ---------------------------------------------------------------------------------
// per-layer kernels
// ---------------------------------------------------------------------------------

// h[m, :] = Emb[ids[b, t], :] (bf16 -> f32)
__global__ void embed_kernel(const int *ids, int ids_ld, RowMap map, const bf16 *emb, int vocab, int H, float *h,
                             int *err) {
    pdl_enter();
    const int m = blockIdx.x;
    const int jj = m / map.rows_per_seq, t = m % map.rows_per_seq;
    const int b = map.seq_of[jj];
    int id = ids[(long long)b * ids_ld + t];
    if (id < 0 || id >= vocab) {
        if (threadIdx.x == 0) atomicOr(err, DEVERR_BOUNDS);
        id = 0;
    }
    const bf16 *src = emb + (long long)id * H;
    float *dst = h + (long long)m * H;
    for (int c = threadIdx.x * 2; c < H; c += blockDim.x * 2) {
        const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(src + c));
        *reinterpret_cast<float2 *>(dst + c) = v;
    }
}

// y[m, :] = bf16(x[m, :] / sqrt(mean(x^2) + eps) * g)
__global__ void rmsnorm_kernel(const float *x, const float *g, bf16 *y, int H, float eps) {
    pdl_enter();
    __shared__ float red[32];
    const long long m = blockIdx.x;
    const float4 *xr = reinterpret_cast<const float4 *>(x + m * H);
    float ss = 0.f;
    for (int c = threadIdx.x; c < H / 4; c += blockDim.x) {
        const float4 v = xr[c];
        ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    ss = block_sum(ss, red);
    const float r = rsqrtf(ss / H + eps);
    const float4 *gr = reinterpret_cast<const float4 *>(g);
    __nv_bfloat162 *yr = reinterpret_cast<__nv_bfloat162 *>(y + m * H);
    for (int c = threadIdx.x; c < H / 4; c += blockDim.x) {
        const float4 v = xr[c], w = gr[c];
        yr[2 * c] = __floats2bfloat162_rn(v.x * r * w.x, v.y * r * w.y);
        yr[2 * c + 1] = __floats2bfloat162_rn(v.z * r * w.z, v.w * r * w.w);
    }
}

// The same with one warp per row (rows per block = blockDim / 32), for many rows: every lane
// keeps eight float4 loads in flight, the sum of squares is a fixed per-lane order and a fixed
// butterfly, and the second pass re-reads the row (from L1).  H a multiple of 128.
__global__ void rmsnorm_warp_kernel(const float *x, const float *g, bf16 *y, int M, int H, float eps) {
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const long long m = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (m >= M) return;
    const float4 *xr = reinterpret_cast<const float4 *>(x + m * H);
    const int n4 = H / 4;
    float ss[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int c0 = 0; c0 < n4; c0 += 32 * 8) {
        float4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int c = c0 + i * 32 + lane;
            v[i] = c < n4 ? xr[c] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) ss[i] += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
    }
    const float tot = warp_sum(((ss[0] + ss[1]) + (ss[2] + ss[3])) + ((ss[4] + ss[5]) + (ss[6] + ss[7])));
    const float r = rsqrtf(tot / H + eps);
    const float4 *gr = reinterpret_cast<const float4 *>(g);
    __nv_bfloat162 *yr = reinterpret_cast<__nv_bfloat162 *>(y + m * H);
    for (int c = lane; c < n4; c += 32) {
        const float4 v = xr[c], w = gr[c];
        yr[2 * c] = __floats2bfloat162_rn(v.x * r * w.x, v.y * r * w.y);
        yr[2 * c + 1] = __floats2bfloat162_rn(v.z * r * w.z, v.w * r * w.w);
    }
}

// One warp per row with the whole row in registers (H a multiple of 128, at most 128 * MAXV):
// every lane issues all of its float4 loads before the first use, so a row costs one memory
// round trip instead of one per batch, and the second pass needs no re-read.  The sum of
// squares is a fixed per-lane order and a fixed butterfly.
template <int MAXV>
__global__ void __launch_bounds__(128) rmsnorm_row_regs_kernel(const float *x, const float *g, bf16 *y, int M, int H,
                                                                float eps) {
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const long long m = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (m >= M) return;
    const float4 *xr = reinterpret_cast<const float4 *>(x + m * H);
    const int nv = H / 128;  // float4 per lane
    float4 v[MAXV];
#pragma unroll
    for (int i = 0; i < MAXV; ++i) v[i] = i < nv ? xr[i * 32 + lane] : make_float4(0.f, 0.f, 0.f, 0.f);
    float ss[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < MAXV; ++i) ss[i & 3] += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
    const float r = rsqrtf(warp_sum((ss[0] + ss[1]) + (ss[2] + ss[3])) / H + eps);
    const float4 *gr = reinterpret_cast<const float4 *>(g);
    uint2 *yr = reinterpret_cast<uint2 *>(y + m * H);
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
        if (i < nv) {
            const float4 w = gr[i * 32 + lane];
            const __nv_bfloat162 lo = __floats2bfloat162_rn(v[i].x * r * w.x, v[i].y * r * w.y);
            const __nv_bfloat162 hi = __floats2bfloat162_rn(v[i].z * r * w.z, v[i].w * r * w.w);
            uint2 pk;
            memcpy(&pk.x, &lo, 4);
            memcpy(&pk.y, &hi, 4);
            yr[i * 32 + lane] = pk;
        }
    }
}

// Per row m and head: optional per-head RMSNorm of q and k, rotate-half RoPE at the row's
// position, then q -> q_out (bf16, packed: [slot j][kv head][position * G + head-in-group][hd],
// so the G query heads of a KV head are consecutive rows) and k, v -> the KV arena slot (bf16).
__global__ void qkv_post_kernel(const float *qkv, int nq, int nkv, int hd, const float *qn, const float *kn,
                                int qk_norm, float eps, const float2 *rope, RowMap map, bf16 *q_out, bf16 *kc,
                                bf16 *vc, long long seq_stride, long long head_stride) {
    pdl_enter();
    const int m = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    int jj, u, t;
    row_of(map, m, jj, u, t);
    const int b = map.seq_of[jj];
    const int pos = map.pos0 + t;
    const int E = hd >> 5;  // 2 or 4 elements per lane, lane l holds d = l*E .. l*E+E-1
    const int half = hd >> 1;
    const int n_heads = nq + 2 * nkv;
    const float *row = qkv + (long long)m * n_heads * hd;
    // blockIdx.y selects a group of nw heads: one warp per (row, head)
    for (int hh = blockIdx.y * nw + warp; hh < min(n_heads, (int)(blockIdx.y + 1) * nw); hh += nw) {
        float x[4] = {0.f, 0.f, 0.f, 0.f};
        if (E == 4) {
            const float4 t4 = *reinterpret_cast<const float4 *>(row + hh * hd + lane * 4);
            x[0] = t4.x;
            x[1] = t4.y;
            x[2] = t4.z;
            x[3] = t4.w;
        } else {
            const float2 t2 = *reinterpret_cast<const float2 *>(row + hh * hd + lane * 2);
            x[0] = t2.x;
            x[1] = t2.y;
        }
        if (hh < nq + nkv) {
            const float *w = hh < nq ? qn : kn;
            if (qk_norm) {
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (e < E) ss += x[e] * x[e];
                ss = warp_sum(ss);
                const float r = rsqrtf(ss / hd + eps);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (e < E) x[e] = x[e] * r * w[lane * E + e];
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (e < E) {
                    const float other = __shfl_xor_sync(0xffffffffu, x[e], 16);
                    const int d = lane * E + e;
                    const float2 cs = rope[(long long)pos * half + (d % half)];
                    x[e] = (d < half) ? (x[e] * cs.x - other * cs.y) : (x[e] * cs.x + other * cs.y);
                }
            }
        }
        bf16 *dst;
        if (hh < nq) {
            // packed query order: per (sequence slot, kv head), row = position * G + head-in-group
            const int G = nq / nkv;
            const int RP = G * map.rows_per_seq;
            dst = q_out + (((long long)jj * nkv + hh / G) * RP + (long long)u * G + hh % G) * hd;
        } else if (hh < nq + nkv) {
            dst = kc + (long long)b * seq_stride + (long long)(hh - nq) * head_stride + (long long)pos * hd;
        } else {
            dst = vc + (long long)b * seq_stride + (long long)(hh - nq - nkv) * head_stride + (long long)pos * hd;
        }
        if (E == 4) {
            __nv_bfloat162 b2[2] = {__floats2bfloat162_rn(x[0], x[1]), __floats2bfloat162_rn(x[2], x[3])};
            *reinterpret_cast<uint2 *>(dst + lane * 4) = *reinterpret_cast<const uint2 *>(b2);
        } else {
            *reinterpret_cast<__nv_bfloat162 *>(dst + lane * 2) = __floats2bfloat162_rn(x[0], x[1]);
        }
    }
}

// The same for head_dim 128 with one block per row and each warp taking `hpw` (<= 8) heads of
// it: every head's load and the row's RoPE table entries are issued before any arithmetic, so
// a warp waits for one memory round trip instead of one per head.  At 64 registers four blocks
// share an SM (80 left three).
__global__ void __launch_bounds__(256, 4)
    qkv_post128_kernel(const float *qkv, int nq, int nkv, int hpw, const float *qn, const float *kn, int qk_norm,
                       float eps, const float2 *rope, RowMap map, bf16 *q_out, bf16 *kc, bf16 *vc,
                       long long seq_stride, long long head_stride) {
    pdl_enter();
    constexpr int HD = 128, MAXH = 8;
    const int m = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int jj, u, t;
    row_of(map, m, jj, u, t);
    const int pos = map.pos0 + t;
    const int n_heads = nq + 2 * nkv;
    const int h0 = warp * hpw, h1 = min(n_heads, h0 + hpw);
    if (h0 >= h1) return;
    const float *row = qkv + (long long)m * n_heads * HD;
    float4 x[MAXH];
#pragma unroll
    for (int i = 0; i < MAXH; ++i)
        if (h0 + i < h1) x[i] = *reinterpret_cast<const float4 *>(row + (h0 + i) * HD + lane * 4);
    float2 cs[4];
    rope_lane128(rope, pos, lane, cs);
    const float4 wq = qk_norm ? *reinterpret_cast<const float4 *>(qn + lane * 4) : make_float4(1.f, 1.f, 1.f, 1.f);
    const float4 wk = qk_norm ? *reinterpret_cast<const float4 *>(kn + lane * 4) : make_float4(1.f, 1.f, 1.f, 1.f);
    const int b = map.seq_of[jj];
    const int G = nq / nkv, RP = G * map.rows_per_seq;
#pragma unroll
    for (int i = 0; i < MAXH; ++i) {
        const int hh = h0 + i;
        if (hh >= h1) break;  // uniform across the warp
        const float4 v = head_post128(x[i], hh < nq + nkv, qk_norm, hh < nq ? wq : wk, eps, cs, lane);
        bf16 *dst;
        if (hh < nq)
            dst = q_out + (((long long)jj * nkv + hh / G) * RP + (long long)u * G + hh % G) * HD;
        else if (hh < nq + nkv)
            dst = kc + (long long)b * seq_stride + (long long)(hh - nq) * head_stride + (long long)pos * HD;
        else
            dst = vc + (long long)b * seq_stride + (long long)(hh - nq - nkv) * head_stride + (long long)pos * HD;
        store_bf16x4(dst + lane * 4, v);
    }
}

// Prefill depth fallback: for prefix positions whose exit depth is below the current depth,
// the KV at this depth is the KV of the previous depth (which by induction is the KV of
// their exit depth).  Positions pos0 .. pos0+n-1 of sequence b0 + blockIdx.x, whose exit
// depths are exit_depth[(b0 + blockIdx.x) * n + t]; one block per (sequence, kv head),
// threads over positions.
__global__ void kv_fallback_kernel(const int *exit_depth, int n, int pos0, int b0, int depth, const bf16 *src_k,
                                   const bf16 *src_v, bf16 *dst_k, bf16 *dst_v, long long seq_stride,
                                   long long head_stride, int hd) {
    pdl_enter();
    const int b = b0 + blockIdx.x, kvh = blockIdx.y;
    const long long base = (long long)b * seq_stride + (long long)kvh * head_stride;
    const int chunks = hd / 8;
    for (long long idx = threadIdx.x; idx < (long long)n * chunks; idx += blockDim.x) {
        const int t = (int)(idx / chunks), ch = (int)(idx % chunks);
        if (exit_depth[(long long)b * n + t] >= depth) continue;
        const long long off = base + (long long)(pos0 + t) * hd + ch * 8;
        *reinterpret_cast<uint4 *>(dst_k + off) = *reinterpret_cast<const uint4 *>(src_k + off);
        *reinterpret_cast<uint4 *>(dst_v + off) = *reinterpret_cast<const uint4 *>(src_v + off);
    }
}

// Error-path probe: one thread waits, bounded, on an mbarrier that nothing ever arrives on, so
// the wait expires and the device error word records a timeout -- the path every bounded wait
// of the library takes, exercised without a GPU fault (no trap, no endless loop).
__global__ void wait_expiry_kernel(int *err) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbarrier_init();
        mbar_wait(&bar, 0, err);
    }
}

// h_exit[m] = h[m] for prefix rows whose exit depth equals `depth`
__global__ void capture_exit_kernel(const int *exit_depth, int P, int b0, int depth, const float *h, float *h_exit,
                                    int H) {
    pdl_enter();
    const int m = blockIdx.x;
    const int b = b0 + m / P, pos = m % P;
    if (exit_depth[(long long)b * P + pos] != depth) return;
    const float4 *src = reinterpret_cast<const float4 *>(h + (long long)m * H);
    float4 *dst = reinterpret_cast<float4 *>(h_exit + (long long)m * H);
    for (int c = threadIdx.x; c < H / 4; c += blockDim.x) dst[c] = src[c];
}

// Depth-on-demand prefill.  Rows of depth d are compacted to the positions whose exit depth
// reaches d: row m of depth d is original row orig[m] = row_seq[m] * n + row_t[m] of the group.
// h_exit[orig] = h[m] for the rows whose exit depth equals d
__global__ void scatter_exit_kernel(const int *exit_depth, int n, int b0, int depth, const int *row_seq,
                                    const int *row_t, const float *h, float *h_exit, int H) {
    pdl_enter();
    const int m = blockIdx.x;
    const int jj = row_seq[m], t = row_t[m];
    if (exit_depth[(long long)(b0 + jj) * n + t] != depth) return;
    const float4 *src = reinterpret_cast<const float4 *>(h + (long long)m * H);
    float4 *dst = reinterpret_cast<float4 *>(h_exit + ((long long)jj * n + t) * H);
    for (int c = threadIdx.x; c < H / 4; c += blockDim.x) dst[c] = src[c];
}

// dst[m] = src[idx[m]] (rows of H floats)
__global__ void gather_idx_rows_kernel(const float *src, float *dst, const int *idx, int H) {
    pdl_enter();
    const int m = blockIdx.x;
    const float4 *s = reinterpret_cast<const float4 *>(src + (long long)idx[m] * H);
    float4 *d = reinterpret_cast<float4 *>(dst + (long long)m * H);
    for (int c = threadIdx.x; c < H / 4; c += blockDim.x) d[c] = s[c];
}

// Positions [0, n_pos) of sequences 0..nb-1, every KV head: slot dst = slot src (K and V).
// Fills a Core depth that no position had reached yet from the deepest one built.
__global__ void copy_positions_kernel(const bf16 *src_k, const bf16 *src_v, bf16 *dst_k, bf16 *dst_v, int n_pos,
                                      long long seq_stride, long long head_stride, int hd) {
    pdl_enter();
    const int b = blockIdx.x, kvh = blockIdx.y;
    const long long base = (long long)b * seq_stride + (long long)kvh * head_stride;
    const long long n = (long long)n_pos * hd / 8;
    for (long long i = threadIdx.x; i < n; i += blockDim.x) {
        *reinterpret_cast<uint4 *>(dst_k + base + i * 8) = *reinterpret_cast<const uint4 *>(src_k + base + i * 8);
        *reinterpret_cast<uint4 *>(dst_v + base + i * 8) = *reinterpret_cast<const uint4 *>(src_v + base + i * 8);
    }
}

// ---------------------------------------------------------------------------------
// readout
// ---------------------------------------------------------------------------------

// For every active row m: r = RMSNorm_f(hc[m]) (f32).  Rows in U (ridx[m] >= 0) get their
// bf16 copy for the LM head and lambda = sigmoid(w . r + b); with a debug buffer every row's
// r is also stored at [b, i].
__global__ void final_norm_kernel(const float *hc, const float *g, const float *exit_w, float exit_b, int H, float eps,
                                  RowMap map, const int *ridx, bf16 *rb, float *lam_rr, float *dbg_r) {
    pdl_enter();
    __shared__ float red[32];
    const int m = blockIdx.x;
    const int rr = ridx[m];
    if (rr < 0 && dbg_r == nullptr) return;
    const int N = map.rows_per_seq;
    const int b = map.seq_of[m / N], i = m % N;
    const float *x = hc + (long long)m * H;
    float ss = 0.f;
    for (int c = threadIdx.x; c < H; c += blockDim.x) ss += x[c] * x[c];
    ss = block_sum(ss, red);
    const float rs = rsqrtf(ss / H + eps);
    float dot = 0.f;
    for (int c = threadIdx.x; c < H; c += blockDim.x) {
        const float r = x[c] * rs * g[c];
        dot = fmaf(r, exit_w[c], dot);
        if (rr >= 0) rb[(long long)rr * H + c] = __float2bfloat16_rn(r);
        if (dbg_r) dbg_r[((long long)b * N + i) * H + c] = r;
    }
    dot = block_sum(dot, red);
    if (rr >= 0 && threadIdx.x == 0) lam_rr[rr] = 1.f / (1.f + expf(-(dot + exit_b)));
}

struct Stat {
    float m, s, t;
    int idx;
};
__device__ __forceinline__ Stat merge_stat(Stat a, Stat b) {
    // prefer the larger max; on equal max the lower vocabulary id
    const bool take_b = (b.m > a.m) || (b.m == a.m && b.idx < a.idx);
    const float M = fmaxf(a.m, b.m);
    const float ea = expf(a.m - M), eb = expf(b.m - M);
    Stat r;
    r.m = M;
    r.s = a.s * ea + b.s * eb;
    r.t = ea * (a.t + a.s * (a.m - M)) + eb * (b.t + b.s * (b.m - M));
    r.idx = take_b ? b.idx : a.idx;
    return r;
}

// One warp per readout row: merge the per-vocab-tile (max, sum e^(z-max), sum e^(z-max)(z-max),
// argmax) in a fixed order -> entropy H = log S - T/S (nats) and argmax; then the cumulative
// halt a <- a + (1 - a) lambda and the traces.
// With sampling on, the committed token is instead the id of the largest z_v + g_v over the
// per-tile (score, id) partials (larger score first, the lower id on equal scores).
__global__ void readout_combine_kernel(const float4 *part, const double2 *spart, const SampleParams *samp, int n_vt,
                                       const int *R_dev, const int *rr_b, const int *rr_i, const float *lam_rr, int N,
                                       int Kstep, int s, float *a_state, float *cur_H, int *cur_y, float *tr_H,
                                       float *tr_lam, float *tr_a) {
    pdl_enter();
    const int rr = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (rr >= *R_dev) return;
    const float4 *p = part + (long long)rr * n_vt;
    Stat acc = {-INFINITY, 0.f, 0.f, 0x7fffffff};
    bool have = false;
    for (int v = lane; v < n_vt; v += 32) {
        const float4 x = p[v];
        Stat st = {x.x, x.y, x.z, __float_as_int(x.w)};
        acc = have ? merge_stat(acc, st) : st;
        have = true;
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        Stat other;
        other.m = __shfl_xor_sync(0xffffffffu, acc.m, o);
        other.s = __shfl_xor_sync(0xffffffffu, acc.s, o);
        other.t = __shfl_xor_sync(0xffffffffu, acc.t, o);
        other.idx = __shfl_xor_sync(0xffffffffu, acc.idx, o);
        const bool other_have = __shfl_xor_sync(0xffffffffu, (int)have, o) != 0;
        // order the pair by lane so both lanes compute the same value
        if (other_have) {
            if (!have)
                acc = other;
            else
                acc = ((lane & o) == 0) ? merge_stat(acc, other) : merge_stat(other, acc);
        }
        have = have || other_have;
    }
    int token = acc.idx;
    if (samp->enabled) {
        const double2 *sp = spart + (long long)rr * n_vt;
        double best = -INFINITY;
        int bid = 0x7fffffff;
        for (int v = lane; v < n_vt; v += 32) {
            const double2 x = sp[v];
            const int id = (int)x.y;
            if (x.x > best || (x.x == best && id < bid)) {
                best = x.x;
                bid = id;
            }
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bid, o);
            if (ob > best || (ob == best && oi < bid)) {
                best = ob;
                bid = oi;
            }
        }
        token = bid;
    }
    if (lane == 0) {
        const int b = rr_b[rr], i = rr_i[rr];
        const float H = logf(acc.s) - acc.t / acc.s;
        const float lam = lam_rr[rr];
        const long long bi = (long long)b * N + i;
        const float a = a_state[bi] + (1.f - a_state[bi]) * lam;
        a_state[bi] = a;
        cur_H[bi] = H;
        cur_y[bi] = token;
        const long long tr = ((long long)b * Kstep + (s - 1)) * N + i;
        tr_H[tr] = H;
        tr_lam[tr] = lam;
        tr_a[tr] = a;
    }
}

// ---------------------------------------------------------------------------------
// step control
// ---------------------------------------------------------------------------------

struct StepState {
    int *tokens, *exit_depth;  // caller outputs [B, N]
    float *tr_H, *tr_lam, *tr_a;
    int *loops_run, *active_rows, *readout_rows;
    unsigned char *U;          // [B, N] still unresolved
    float *a;                  // [B, N] cumulative halt
    float *cur_H;              // [B, N] this loop's entropy
    int *cur_y;                // [B, N] this loop's argmax
    int *cont;                 // [B] 1 while the sequence keeps looping
    int *n_commit;             // [B] commits in this step
};

__global__ void step_init_kernel(const int *block_ids, int B, int N, int Kstep, int mask_id, StepState st,
                                 SampleParams sp, SampleParams *samp) {
    pdl_enter();
    if (blockIdx.x == 0 && threadIdx.x == 0) *samp = sp;
    const long long total = (long long)B * N;
    const float qnan = __int_as_float(0x7fc00000);
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int id = block_ids[idx];
        st.tokens[idx] = id;
        st.exit_depth[idx] = 0;
        st.U[idx] = (id == mask_id) ? 1 : 0;
        st.a[idx] = 0.f;
        const int b = (int)(idx / N), i = (int)(idx % N);
        for (int s = 0; s < Kstep; ++s) {
            const long long tr = ((long long)b * Kstep + s) * N + i;
            st.tr_H[tr] = qnan;
            st.tr_lam[tr] = qnan;
            st.tr_a[tr] = qnan;
        }
        if (i == 0) {
            st.cont[b] = 1;
            st.n_commit[b] = 0;
            st.loops_run[b] = 0;
        }
        if (idx == 0)
            for (int s = 0; s < Kstep; ++s) {
                st.active_rows[s] = 0;
                st.readout_rows[s] = 0;
            }
    }
}

// *left = 1 if any of ids[0, total) is the mask id (*left cleared by the caller)
__global__ void any_mask_kernel(const int *ids, long long total, int mask_id, int *left) {
    pdl_enter();
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x)
        if (ids[idx] == mask_id) *left = 1;
}

// Block decoding, after denoising step t (1-based) of in_ids -> tokens / exit_depth: record the
// step and depth of this step's commits, count the step for sequences that had masks at its
// start, and raise *left if any [MASK] remains.
__global__ void decode_update_kernel(const int *in_ids, const int *tokens, const int *exit_depth, int t, int B,
                                     int N, int mask_id, int *commit_step, int *commit_depth, int *steps_run,
                                     int *left) {
    pdl_enter();
    const long long total = (long long)B * N;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int d = exit_depth[idx];
        if (d > 0) {
            commit_step[idx] = t;
            commit_depth[idx] = d;
        }
        if (in_ids[idx] == mask_id) steps_run[idx / N] = t;  // same value from every writer
        if (tokens[idx] == mask_id) *left = 1;
    }
}

// One block per looping sequence (slot j): commit per rule, halting decision, forced
// commit, and the Eq. 3 merge of committed rows into the loop state h.
__global__ void commit_kernel(RowMap map, int s, int Kstep, int rule, float tau, float lam, const bf16 *emb, int H,
                              float *h, StepState st) {
    pdl_enter();
    __shared__ float red[32];
    __shared__ int red_i[32];
    const int jj = blockIdx.x;
    const int N = map.rows_per_seq;
    const int b = map.seq_of[jj];
    const long long base = (long long)b * N;
    int n_new = 0, n_left = 0;
    float a_left = 0.f;
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
        if (!st.U[base + i]) continue;
        const float Hh = st.cur_H[base + i], a = st.a[base + i];
        const bool c = (Hh <= tau) || (rule == 1 && (a >= lam || s == Kstep));
        if (c) {
            st.tokens[base + i] = st.cur_y[base + i];
            st.exit_depth[base + i] = s;
            st.U[base + i] = 0;
            ++n_new;
        } else {
            ++n_left;
            a_left += a;
        }
    }
    const float f_new = block_sum((float)n_new, red);
    const float f_left = block_sum((float)n_left, red);
    const float sum_a = block_sum(a_left, red);
    const int total_new = (int)f_new, total_left = (int)f_left;
    const int committed = st.n_commit[b] + total_new;
    bool stop = (total_left == 0) || (s == Kstep);
    if (rule == 0 && total_left > 0 && sum_a / (float)total_left >= lam) stop = true;
    int forced = 0;
    if (stop && rule == 0 && committed == 0 && total_left > 0) {
        // lowest entropy of this loop among the unresolved, lowest index on ties
        float bestH = INFINITY;
        int besti = 0x7fffffff;
        for (int i = threadIdx.x; i < N; i += blockDim.x) {
            if (!st.U[base + i]) continue;
            const float Hh = st.cur_H[base + i];
            if (Hh < bestH || (Hh == bestH && i < besti)) {
                bestH = Hh;
                besti = i;
            }
        }
        for (int o = 16; o > 0; o >>= 1) {
            const float oh = __shfl_xor_sync(0xffffffffu, bestH, o);
            const int oi = __shfl_xor_sync(0xffffffffu, besti, o);
            if (oh < bestH || (oh == bestH && oi < besti)) {
                bestH = oh;
                besti = oi;
            }
        }
        const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
        __syncthreads();
        if (l == 0) {
            red[w] = bestH;
            red_i[w] = besti;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            for (int ww = 1; ww < (int)(blockDim.x >> 5); ++ww)
                if (red[ww] < red[0] || (red[ww] == red[0] && red_i[ww] < red_i[0])) {
                    red[0] = red[ww];
                    red_i[0] = red_i[ww];
                }
            const int i = red_i[0];
            st.tokens[base + i] = st.cur_y[base + i];
            st.exit_depth[base + i] = s;
            st.U[base + i] = 0;
        }
        forced = 1;
    }
    if (threadIdx.x == 0) {
        st.n_commit[b] = committed + forced;
        if (stop) {
            st.loops_run[b] = s;
            st.cont[b] = 0;
        }
    }
    if (!stop) {
        // Eq. 3: committed rows re-enter as Emb(y); unresolved and given rows keep h~.
        // One warp per row, rows spread over the warps.
        const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
        for (int i = w; i < N; i += nw) {
            if (st.exit_depth[base + i] == 0) continue;
            const bf16 *src = emb + (long long)st.tokens[base + i] * H;
            float *dst = h + ((long long)jj * N + i) * H;
            for (int c = l * 8; c < H; c += 32 * 8) {
                const uint4 raw = *reinterpret_cast<const uint4 *>(src + c);
                const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
                const float2 f0 = __bfloat1622float2(p2[0]), f1 = __bfloat1622float2(p2[1]);
                const float2 f2 = __bfloat1622float2(p2[2]), f3 = __bfloat1622float2(p2[3]);
                *reinterpret_cast<float4 *>(dst + c) = make_float4(f0.x, f0.y, f1.x, f1.y);
                *reinterpret_cast<float4 *>(dst + c + 4) = make_float4(f2.x, f2.y, f3.x, f3.y);
            }
        }
    }
}

// Single block: order-preserving compaction of the looping sequences, the readout row
// list of the next loop (U rows only) and the counters read by the host.
// counts[0] = looping sequences, counts[1] = readout rows, counts[2] = device error word.
__global__ void plan_kernel(int n_cur, const int *seq_cur, int N, const int *cont, const unsigned char *U,
                            int *seq_next, int *old_slot, int *ridx, int *rr_b, int *rr_i, int *counts, int s_next,
                            int Kstep, int *active_rows, int *readout_rows, const int *err) {
    pdl_enter();
    __shared__ int n_next;
    __shared__ int scan[1024];
    __shared__ int carry;
    if (threadIdx.x == 0) {
        int n = 0;
        for (int jj = 0; jj < n_cur; ++jj) {
            const int b = seq_cur[jj];
            if (cont[b]) {
                seq_next[n] = b;
                old_slot[n] = jj;
                ++n;
            }
        }
        n_next = n;
        carry = 0;
    }
    __syncthreads();
    const int rows = n_next * N;
    for (int c0 = 0; c0 < rows; c0 += blockDim.x) {
        const int m = c0 + threadIdx.x;
        int flag = 0, b = 0, i = 0;
        if (m < rows) {
            b = seq_next[m / N];
            i = m % N;
            flag = U[(long long)b * N + i] ? 1 : 0;
        }
        scan[threadIdx.x] = flag;
        __syncthreads();
        for (int off = 1; off < (int)blockDim.x; off <<= 1) {
            const int v = (threadIdx.x >= (unsigned)off) ? scan[threadIdx.x - off] : 0;
            __syncthreads();
            scan[threadIdx.x] += v;
            __syncthreads();
        }
        if (m < rows) {
            const int pos = carry + scan[threadIdx.x] - flag;
            ridx[m] = flag ? pos : -1;
            if (flag) {
                rr_b[pos] = b;
                rr_i[pos] = i;
            }
        }
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry += scan[threadIdx.x];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        counts[0] = n_next;
        counts[1] = carry;
        counts[2] = *err;
        if (s_next <= Kstep && n_next > 0) {
            active_rows[s_next - 1] = n_next * N;
            readout_rows[s_next - 1] = carry;
        }
    }
}

// dst rows of the next loop's compact layout from the current layout
__global__ void gather_rows_kernel(const float *src, float *dst, const int *old_slot, int N, int H) {
    pdl_enter();
    const int m = blockIdx.x;
    const int jn = m / N, i = m % N;
    const float4 *s = reinterpret_cast<const float4 *>(src + ((long long)old_slot[jn] * N + i) * H);
    float4 *d = reinterpret_cast<float4 *>(dst + (long long)m * H);
    for (int c = threadIdx.x; c < H / 4; c += blockDim.x) d[c] = s[c];
}

// debug copy of compact rows to [b, i] order
__global__ void dump_rows_kernel(const float *src, RowMap map, int H, float *dst) {
    pdl_enter();
    const int m = blockIdx.x;
    const int N = map.rows_per_seq;
    const int b = map.seq_of[m / N], i = m % N;
    const float4 *s = reinterpret_cast<const float4 *>(src + (long long)m * H);
    float4 *d = reinterpret_cast<float4 *>(dst + ((long long)b * N + i) * H);
    for (int c = threadIdx.x; c < H / 4; c += blockDim.x) d[c] = s[c];
}

}  // namespace k
