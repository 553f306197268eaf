// attention_tc.cuh — block attention of a denoising step on the fifth-generation tensor core.
//
// One CTA serves 128 packed query rows of one (sequence, KV head): packed row r is query head
// kvh*G + r % G at block position r / G (q is stored in that packed order), so the G query
// heads of a KV head share every K/V tile.  head_dim 64 or 128 (a template argument: one or two
// 64-wide, 128-byte-swizzled halves per head vector).  A denoising step's block attends
// every prefix key and every block key (no mask inside [0, kv_len)); causal rows (a prefill or
// an append, possibly compacted to the positions that run a Core depth) attend keys up to their
// own position: the CTA's key range ends at its last row's position, and the key tiles that
// cross the tile's first row's position mask each row at its own.
//
//   warp 0      TMA: Q once; K and V tiles of 128 keys (64-wide halves, 128-byte swizzle)
//               into a 2-stage ring, straight from the depth-aware KV arena
//   warp 1      tcgen05.mma: S_i = Q K_i^T into a double-buffered TMEM tile (M=128, N=128),
//               then O += P_i V_i into the TMEM accumulator (V read MN-major)
//   warps 2-5   softmax, one thread per query row: tcgen05.ld its S row, exp2 with a running
//               reference max that only moves when the row max passes it by more than 8
//               (rescaling O in TMEM then), P_i as bf16 into a double-buffered shared-memory
//               tile in the MMA's 128-byte-swizzled K-major layout (the exponentials of tile i
//               overlap PV_{i-1}); at the end O / l to global memory
//
// With n_splits > 1 the keys are split across the S CTAs of a cluster.  CTA r owns 128/S
// query rows of the tile: once every CTA of the cluster is done with its K/V ring, each CTA
// stores its partial (O row, reference max, l) of every row straight into the owner's ring
// (remote stores), one cluster barrier, and each owner merges the S partials in rank order.
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"

namespace attn_tc {

namespace cg = cooperative_groups;

constexpr int HD = 128;        // head_dim of the two-tile kernel (attention_pq.cuh)
constexpr int BQ = 128;        // query rows per CTA
constexpr int BKV = 128;       // keys per tile
constexpr int KV_STAGES = 2;
constexpr uint32_t HALF = BQ * 64 * 2;  // one [128 rows][64] bf16 region = 16 KB
constexpr uint32_t Q_BYTES = 2 * HALF;
constexpr uint32_t KV_BYTES = 2 * HALF;  // one K (or V) tile
constexpr uint32_t P_BYTES = 2 * HALF;
constexpr uint32_t TMEM_COLS = 512;      // S0 [0,128) S1 [128,256) O [256,384)
constexpr uint32_t O_COL = 256;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units
// shared memory at head_dim D: Q, the K and V rings, P double-buffered, barriers
template <int D>
constexpr size_t smem_bytes() {
    return 1024 + (D / 64) * HALF + 2 * KV_STAGES * (D / 64) * HALF + 2 * P_BYTES + 256;
}
constexpr size_t SMEM = smem_bytes<HD>();

struct Params {
    int RP;            // packed query rows per (sequence, kv head) = G * rows_per_seq
    int G, nkv, nq, Tq;
    int kv_len;        // keys [0, kv_len) of the slot
    int slot, max_batch, pos_stride;
    const int *seq_of;
    int n_splits, keys_per_split;  // keys_per_split a multiple of BKV
    bf16 *out;
    int out_ld;
    int m_rows;
    float scale_log2;
    int *err;
    // keys [0, static_keys) are not written by the kernels this launch depends on (the cached
    // prefix during a step): their first K/V stages are requested before griddepcontrol.wait.
    // 0: every key waits.
    int static_keys;
    // 1: the last key split runs to kv_len even past keys_per_split (a remainder shorter than
    // a key tile rides on the last rank instead of costing every rank a second tile)
    int last_to_end;
    // 1: row u of sequence slot j sits at position pos0 + (row_t ? row_t[row_off + u] : u) and
    // sees keys [0, that position] (n_splits must be 1).  Row tables (compacted rows, null
    // otherwise, causal or not): slot j owns output rows [seq_off[j], seq_off[j] + seq_cnt[j]),
    // in position order; without them its rows are j * Tq + u, u < Tq.
    int causal, pos0;
    const int *row_t, *seq_off, *seq_cnt;
};

// K-major operand, 128-byte swizzle (8-row atoms of 128 B, 1024 B apart)
__device__ __forceinline__ uint64_t sdesc_k(uint32_t saddr) { return umma_sdesc_sw128(saddr); }

// MN-major operand, 128-byte swizzle: 64 MN elements per 128-byte row, one row per K index,
// 8-row atoms 1024 B apart (stride byte offset), the next 64 MN elements `lbo` bytes on
__device__ __forceinline__ uint64_t sdesc_mn(uint32_t saddr, uint32_t lbo) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
        "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
        "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
        "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
        "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    uint32_t u;
    memcpy(&u, &v, 4);
    return u;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int D>
__global__ void __launch_bounds__(192, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, Params p) {
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    constexpr int NH = D / 64;              // 64-wide halves of a head vector
    constexpr uint32_t QB = NH * HALF;      // the Q tile
    constexpr uint32_t KVB = NH * HALF;     // one K (or V) tile
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;
    uint8_t *sK = sQ + QB;                       // [stage] K tiles
    uint8_t *sV = sK + KV_STAGES * KVB;          // [stage] V tiles
    uint8_t *sP = sV + KV_STAGES * KVB;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sP + 2 * P_BYTES);
    uint64_t *q_full = bars;
    uint64_t *k_full = bars + 1;                      // [2]
    uint64_t *v_full = bars + 3;                      // [2]
    uint64_t *kv_empty = bars + 5;                    // [2]
    uint64_t *s_full = bars + 7;                      // [2]
    uint64_t *p_full = bars + 9;
    uint64_t *pv_done = bars + 10;                    // [2], PV_i completes pv_done[i & 1]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 12);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // causal: the last query tiles (the longest key ranges) are scheduled first
    const int qtile = p.causal ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x;
    const int kvh = blockIdx.y / p.n_splits, split = blockIdx.y % p.n_splits;
    const int j = blockIdx.z;
    // this slot's query rows (fewer than Tq when compacted; the row tables were copied in before
    // the layer's first kernel started, so they are read before griddepcontrol.wait)
    const int seq_rows = p.seq_cnt ? p.seq_cnt[j] : p.Tq;
    const int row_off = p.seq_off ? p.seq_off[j] : j * p.Tq;
    const int rows_packed = p.G * seq_rows;
    auto pos_of = [&](int u) { return p.pos0 + (p.row_t ? p.row_t[row_off + u] : u); };
    const int kstart = split * p.keys_per_split;
    // the last rank may also take a ragged remainder past its range (last_to_end)
    int kend = (p.last_to_end && split == p.n_splits - 1) ? p.kv_len : min(p.kv_len, kstart + p.keys_per_split);
    int mask_from = kend;  // the first key that some row of the tile does not see
    if (qtile * BQ >= rows_packed) {
        kend = kstart;  // no query rows in this tile
    } else if (p.causal) {
        // rows are in position order: the last row sees the most keys, the first the fewest
        kend = min(kend, pos_of(min(qtile * BQ + BQ - 1, rows_packed - 1) / p.G) + 1);
        mask_from = min(kend, pos_of(qtile * BQ / p.G) + 1);
    }
    const int n_tiles = kend > kstart ? (kend - kstart + BKV - 1) / BKV : 0;

    int pre = 0;  // K/V stages requested before the wait (thread 0, the producer)
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(k_full + s, 1);
            mbar_init(v_full + s, 1);
            mbar_init(kv_empty + s, 1);
            mbar_init(s_full + s, 1);
        }
        mbar_init(p_full, 128);
        mbar_init(pv_done, 1);
        mbar_init(pv_done + 1, 1);
        fence_mbarrier_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        if (n_tiles > 0 && kstart + BKV <= p.static_keys) {
            const int b0 = p.seq_of[j];
            const int kvrow0 = (int)((((long long)p.slot * p.max_batch + b0) * p.nkv + kvh) * p.pos_stride);
            for (; pre < min(n_tiles, KV_STAGES) && kstart + (pre + 1) * BKV <= p.static_keys; ++pre) {
                const int row = kvrow0 + kstart + pre * BKV;
                mbar_arrive_expect_tx(k_full + pre, KVB);
                for (int hh = 0; hh < NH; ++hh) tma_load_2d(sK + pre * KVB + hh * HALF, &tmK, k_full + pre, 64 * hh, row);
                mbar_arrive_expect_tx(v_full + pre, KVB);
                for (int hh = 0; hh < NH; ++hh) tma_load_2d(sV + pre * KVB + hh * HALF, &tmV, v_full + pre, 64 * hh, row);
            }
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_enter();
    const int b = p.seq_of[j];
    float m_ref = -INFINITY, l = 0.f;  // softmax thread: running reference max and sum
    bool have_partial = false;         // split partial ready in TMEM

    if (warp == 0) {
        if (lane == 0 && n_tiles > 0) {
            const int qrow = (j * p.nkv + kvh) * p.RP + qtile * BQ;
            mbar_arrive_expect_tx(q_full, QB);
            for (int hh = 0; hh < NH; ++hh) tma_load_2d(sQ + hh * HALF, &tmQ, q_full, 64 * hh, qrow);
            const int kvrow0 = (int)((((long long)p.slot * p.max_batch + b) * p.nkv + kvh) * p.pos_stride);
            int issued = pre;
            for (int i = pre; i < n_tiles; ++i) {
                const int s = i & 1;
                if (!mbar_wait(kv_empty + s, ((uint32_t)(i >> 1) & 1u) ^ 1u, p.err)) break;
                issued = i + 1;
                const int row = kvrow0 + kstart + i * BKV;
                mbar_arrive_expect_tx(k_full + s, KVB);
                for (int hh = 0; hh < NH; ++hh) tma_load_2d(sK + s * KVB + hh * HALF, &tmK, k_full + s, 64 * hh, row);
                mbar_arrive_expect_tx(v_full + s, KVB);
                for (int hh = 0; hh < NH; ++hh) tma_load_2d(sV + s * KVB + hh * HALF, &tmV, v_full + s, 64 * hh, row);
            }
            // no copy into shared memory may still be in flight when the CTA exits
            mbar_wait(q_full, 0, p.err);
            for (int i = max(0, issued - KV_STAGES); i < issued; ++i) {
                mbar_wait(k_full + (i & 1), ((uint32_t)(i >> 1)) & 1u, p.err);
                mbar_wait(v_full + (i & 1), ((uint32_t)(i >> 1)) & 1u, p.err);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && n_tiles > 0) {
            constexpr uint32_t idesc_s = umma_idesc_bf16(BQ, BKV);
            constexpr uint32_t idesc_o = umma_idesc_bf16(BQ, D) | (1u << 16);  // B (V) MN-major
            const uint32_t q_addr = smem_u32(sQ), p_addr = smem_u32(sP);
            auto issue_s = [&](int i) {
                const int s = i & 1;
                const uint32_t k_addr = smem_u32(sK + s * KVB);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
                    umma_f16(tmem + s * BKV, sdesc_k(q_addr + off), sdesc_k(k_addr + off), idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(s_full + s);
            };
            bool ok = mbar_wait(q_full, 0, p.err) && mbar_wait(k_full, 0, p.err);
            if (ok) {
                tc_fence_after();
                issue_s(0);
            }
            for (int i = 0; i < n_tiles && ok; ++i) {
                const int s = i & 1;
                if (i + 1 < n_tiles) {
                    if (!mbar_wait(k_full + ((i + 1) & 1), ((uint32_t)((i + 1) >> 1)) & 1u, p.err)) break;
                    tc_fence_after();
                    issue_s(i + 1);
                }
                if (!mbar_wait(p_full, (uint32_t)i & 1u, p.err)) break;
                if (!mbar_wait(v_full + s, ((uint32_t)(i >> 1)) & 1u, p.err)) break;
                tc_fence_after();
                const uint32_t v_addr = smem_u32(sV + s * KVB);
                const uint32_t pb_addr = p_addr + (i & 1) * P_BYTES;
#pragma unroll
                for (int kk = 0; kk < BKV / 16; ++kk) {
                    const uint32_t a_off = (kk >> 2) * HALF + (kk & 3) * 32;  // P: keys contiguous
                    const uint32_t b_off = kk * 16 * 128;                      // V: 16 key rows of 128 B
                    umma_f16(tmem + O_COL, sdesc_k(pb_addr + a_off), sdesc_mn(v_addr + b_off, HALF), idesc_o,
                             (i > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(pv_done + (i & 1));
                umma_commit(kv_empty + s);
            }
        }
    } else {
        // ---------------- softmax warps: thread t owns query row t ----------------
        const int q = warp & 3;
        const int t = q * 32 + lane;  // TMEM lane = row of the tile
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        // keys [0, row_end) of this row; every row sees key 0, so the first tile of an
        // unsplit range sets a finite reference max
        const int rp_t = qtile * BQ + t;
        const int row_end = (p.causal && rp_t < rows_packed) ? min(kend, pos_of(rp_t / p.G) + 1) : kend;
        bool ok = n_tiles > 0;
        for (int i = 0; i < n_tiles && ok; ++i) {
            const int s = i & 1;
            if (!mbar_wait(s_full + s, ((uint32_t)(i >> 1)) & 1u, p.err)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float sv[BKV];
            {
                uint32_t r[BKV];
#pragma unroll
                for (int c0 = 0; c0 < BKV; c0 += 16) tmem_ld16_async(tmem + lane_base + s * BKV + c0, &r[c0]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < BKV; ++c) {
                    reg_after_wait(r[c]);
                    sv[c] = __uint_as_float(r[c]);
                }
            }
            const int key0 = kstart + i * BKV;
            if (key0 + BKV > mask_from) {  // ragged last tile or causal diagonal (uniform across the CTA)
#pragma unroll
                for (int c = 0; c < BKV; ++c)
                    if (key0 + c >= row_end) sv[c] = -INFINITY;
            }
            // row max of the raw scores (the scale is positive), as eight independent chains
            float mx[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) mx[c] = sv[c];
#pragma unroll
            for (int c = 8; c < BKV; ++c) mx[c & 7] = fmaxf(mx[c & 7], sv[c]);
            const float mt =
                fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) *
                p.scale_log2;
            // the reference max moves only when this tile's max passes it by more than 2^8
            const bool resc = mt > m_ref + RESCALE_THRESHOLD;
            const float f = (resc && i > 0) ? exp2f(m_ref - mt) : 1.f;
            if (resc) m_ref = mt;
            // p = 2^(s * scale - m_ref), summed as eight independent chains; 32-key chunks that
            // lie wholly past the range (a ragged last tile) are zero without exponentials
            const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;  // a row with no key yet: p = 0
            float sm[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) sm[c] = 0.f;
#pragma unroll
            for (int c0 = 0; c0 < BKV; c0 += 32) {
                if (key0 + c0 < kend) {  // uniform across the CTA
#pragma unroll
                    for (int c = c0; c < c0 + 32; ++c) {
                        sv[c] = ex2_approx(fmaf(sv[c], p.scale_log2, neg_m));
                        sm[c & 7] += sv[c];
                    }
                } else {
#pragma unroll
                    for (int c = c0; c < c0 + 32; ++c) sv[c] = 0.f;
                }
            }
            const float lt = ((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7]));
            l = l * f + lt;
            // P buffer i & 1 was last read by PV_{i-2}; a rescale of O needs PV_{i-1} complete
            if (i >= 2 && !mbar_wait(pv_done + (i & 1), ((uint32_t)((i - 2) >> 1)) & 1u, p.err)) {
                ok = false;
                break;
            }
            if (resc && i > 0) {
                if (!mbar_wait(pv_done + ((i - 1) & 1), ((uint32_t)((i - 1) >> 1)) & 1u, p.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 16) {
                    float v[16];
                    tmem_ld16(tmem + lane_base + O_COL + c0, v);
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] *= f;
                    tmem_st16(tmem + lane_base + O_COL + c0, v);
                }
            }
            // P row in the K-major 128-byte-swizzled layout: keys 0-63 in the first region,
            // 64-127 in the second; 16-byte chunk c of row t at (t/8)*1024 + (t%8)*128 + ((c ^ t%8)*16)
            uint8_t *pbuf = sP + (i & 1) * P_BYTES;
#pragma unroll
            for (int c = 0; c < BKV / 8; ++c) {
                uint4 pk;
                pk.x = pack2_bf16(sv[c * 8 + 0], sv[c * 8 + 1]);
                pk.y = pack2_bf16(sv[c * 8 + 2], sv[c * 8 + 3]);
                pk.z = pack2_bf16(sv[c * 8 + 4], sv[c * 8 + 5]);
                pk.w = pack2_bf16(sv[c * 8 + 6], sv[c * 8 + 7]);
                const int region = c >> 3, ch = c & 7;
                uint8_t *dst = pbuf + region * HALF + (t >> 3) * 1024 + (t & 7) * 128 + ((ch ^ (t & 7)) << 4);
                *reinterpret_cast<uint4 *>(dst) = pk;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(p_full);
        }
        // ---------------- output ----------------
        if (ok && n_tiles > 0 &&
            mbar_wait(pv_done + ((n_tiles - 1) & 1), ((uint32_t)((n_tiles - 1) >> 1)) & 1u, p.err)) {
            tc_fence_after();
            const int rp = qtile * BQ + t;
            const bool valid = rp < rows_packed;
            const int tt = rp / p.G, h = kvh * p.G + rp % p.G;
            const int m = row_off + tt;
            if (p.n_splits == 1) {
                const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 16) {
                    float v[16];
                    tmem_ld16(tmem + lane_base + O_COL + c0, v);
                    if (valid) {
                        uint4 w0, w1;
                        w0.x = pack2_bf16(v[0] * inv, v[1] * inv);
                        w0.y = pack2_bf16(v[2] * inv, v[3] * inv);
                        w0.z = pack2_bf16(v[4] * inv, v[5] * inv);
                        w0.w = pack2_bf16(v[6] * inv, v[7] * inv);
                        w1.x = pack2_bf16(v[8] * inv, v[9] * inv);
                        w1.y = pack2_bf16(v[10] * inv, v[11] * inv);
                        w1.z = pack2_bf16(v[12] * inv, v[13] * inv);
                        w1.w = pack2_bf16(v[14] * inv, v[15] * inv);
                        bf16 *dst = p.out + (long long)m * p.out_ld + h * D + c0;
                        *reinterpret_cast<uint4 *>(dst) = w0;
                        *reinterpret_cast<uint4 *>(dst + 8) = w1;
                    }
                }
            } else {
                have_partial = true;  // pushed to the row's owner below
            }
        }
        tc_fence_before();
    }
    if (p.n_splits > 1) {
        // The splits of this (sequence, kv head, query tile) form one cluster (rank = split).
        // Phase 0: every CTA is done with its K/V ring and P tiles (a softmax thread gets here
        // after the last PV product completed, or with no keys at all), which become receive
        // buffers: [source rank][owned row][D + 4] f32 partial O rows in the K/V ring (66 KB at D = 128) and
        // (reference max, l) pairs in the P tiles.
        const int S = p.n_splits, rs = BQ / S;
        float *recv_o = reinterpret_cast<float *>(sK);
        float *recv_ml = reinterpret_cast<float *>(sP);
        constexpr int LDO = D + 4;
        cluster_arrive_relaxed();
        cluster_wait_acquire();
        if (warp >= 2) {
            const int t = (warp & 3) * 32 + lane;
            const uint32_t owner = (uint32_t)(t / rs);
            const int slot = split * rs + t % rs;
            const uint32_t dst_ml = cluster_map(smem_u32(recv_ml + 2 * slot), owner);
            st_cluster_v2(dst_ml, have_partial ? m_ref : -1e30f, have_partial ? l : 0.f);
            if (have_partial) {
                const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
                const uint32_t dst = cluster_map(smem_u32(recv_o + (size_t)slot * LDO), owner);
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld16_async(tmem + lane_base + O_COL + c0, &r[0]);
                    tmem_ld16_async(tmem + lane_base + O_COL + c0 + 16, &r[16]);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) reg_after_wait(r[e]);
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        st_cluster_v4(dst + (uint32_t)(c0 + e) * 4u, __uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                                      __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
                }
            }
        }
        cluster_arrive_release();
        cluster_wait_acquire();  // every partial of the rows owned here has landed
        // merge, in rank order: O = sum_r 2^(m_r - M) O_r / sum_r 2^(m_r - M) l_r over the ranks
        // that saw keys (l_r > 0); thread = (owned row, 8 columns)
        constexpr int CH = D / 8;
        for (int e = threadIdx.x; e < rs * CH; e += blockDim.x) {
            const int lr = e / CH, c8 = (e % CH) * 8;
            const int rp = qtile * BQ + split * rs + lr;
            if (rp >= rows_packed) continue;
            float M = -INFINITY;
            for (int rr = 0; rr < S; ++rr) {
                const float *ml = recv_ml + 2 * (rr * rs + lr);
                if (ml[1] > 0.f) M = fmaxf(M, ml[0]);
            }
            float L = 0.f, acc[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = 0.f;
            for (int rr = 0; rr < S; ++rr) {
                const float *ml = recv_ml + 2 * (rr * rs + lr);
                if (!(ml[1] > 0.f)) continue;
                const float w = exp2f(ml[0] - M);
                L += w * ml[1];
                const float4 *o = reinterpret_cast<const float4 *>(recv_o + (size_t)(rr * rs + lr) * LDO + c8);
                const float4 a0 = o[0], a1 = o[1];
                acc[0] += w * a0.x;
                acc[1] += w * a0.y;
                acc[2] += w * a0.z;
                acc[3] += w * a0.w;
                acc[4] += w * a1.x;
                acc[5] += w * a1.y;
                acc[6] += w * a1.z;
                acc[7] += w * a1.w;
            }
            const float inv = L > 0.f ? 1.f / L : 0.f;
            const int tt = rp / p.G, h = kvh * p.G + rp % p.G;
            uint4 pk;
            pk.x = pack2_bf16(acc[0] * inv, acc[1] * inv);
            pk.y = pack2_bf16(acc[2] * inv, acc[3] * inv);
            pk.z = pack2_bf16(acc[4] * inv, acc[5] * inv);
            pk.w = pack2_bf16(acc[6] * inv, acc[7] * inv);
            *reinterpret_cast<uint4 *>(p.out + (long long)(row_off + tt) * p.out_ld + h * D + c8) = pk;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace attn_tc
