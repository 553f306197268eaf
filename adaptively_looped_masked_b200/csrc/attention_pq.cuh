// attention_pq.cuh — block attention of a denoising step with two query tiles per CTA.
//
// Same computation as attn_tc_kernel (packed GQA query rows of one (sequence, KV head), every
// prefix and block key, head_dim 128, softmax in the exp2 domain with a reference max that
// moves only when passed by 2^8), for (sequence, KV head) pairs with at least two 128-row
// query tiles: one CTA serves two tiles, so each K/V tile is loaded once for both, and two
// softmax warpgroups work on them in turn -- while one computes its exponentials the tensor
// core runs the other's products, and each SM scheduler has two softmax warps to issue from.
//
//   warp 0      TMA: both Q tiles once; K tiles (2-stage ring) and V tiles (1 stage)
//   warp 1      tcgen05.mma: S_w = Q_w K_i^T into TMEM tile w (M=128, N=128) as soon as
//               warpgroup w has read S_w of the previous key tile; O_w += P_w V_i once P_w is
//               written (V MN-major), O_w in TMEM
//   warps 2-5   softmax of query tile 2u (thread = row), warps 6-9 of tile 2u+1: read S_w,
//               release it, exponentials, rescale O_w when the reference max moves (after
//               PV_w of the previous tile), P_w as bf16 in the 128-byte-swizzled K-major layout
// No key split: the host uses this kernel only where the CTAs already cover the SMs.
#pragma once
#include "attention_tc.cuh"
#include "common.cuh"

namespace attn_pq {

using attn_tc::BKV;
using attn_tc::BQ;
using attn_tc::HALF;
using attn_tc::HD;
using attn_tc::KV_BYTES;
using attn_tc::P_BYTES;
using attn_tc::Q_BYTES;
using attn_tc::RESCALE_THRESHOLD;

constexpr int K_STAGES = 2;
constexpr uint32_t TMEM_COLS = 512;  // S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512)
constexpr uint32_t O_COL = 256;
constexpr int THREADS = 320;
constexpr size_t SMEM = 1024 + 2 * Q_BYTES + K_STAGES * KV_BYTES + KV_BYTES + 2 * P_BYTES + 256;

__global__ void __launch_bounds__(THREADS, 1)
    attn_pq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, attn_tc::Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;                       // [2] query tiles
    uint8_t *sK = sQ + 2 * Q_BYTES;           // [K_STAGES] K tiles
    uint8_t *sV = sK + K_STAGES * KV_BYTES;   // one V tile
    uint8_t *sP = sV + KV_BYTES;              // [2] P tiles, one per query tile
    uint64_t *bars = reinterpret_cast<uint64_t *>(sP + 2 * P_BYTES);
    uint64_t *q_full = bars;
    uint64_t *k_full = bars + 1;   // [2]
    uint64_t *k_empty = bars + 3;  // [2]
    uint64_t *v_full = bars + 5;
    uint64_t *v_empty = bars + 6;
    uint64_t *s_full = bars + 7;   // [2] per query tile
    uint64_t *s_free = bars + 9;   // [2]
    uint64_t *p_full = bars + 11;  // [2]
    uint64_t *pv_done = bars + 13; // [2]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 15);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kvh = blockIdx.y, j = blockIdx.z;
    const int qt0 = 2 * blockIdx.x;                                 // first query tile of this CTA
    const int n_str = (p.RP > (qt0 + 1) * BQ) ? 2 : 1;              // query tiles present
    const int n_tiles = (p.kv_len + BKV - 1) / BKV;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(k_full + s, 1);
            mbar_init(k_empty + s, 1);
            mbar_init(s_full + s, 1);
            mbar_init(s_free + s, 4);
            mbar_init(p_full + s, 128);
            mbar_init(pv_done + s, 1);
        }
        mbar_init(v_full, 1);
        mbar_init(v_empty, 1);
        fence_mbarrier_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
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
    if (warp == 0) {
        if (lane == 0 && n_tiles > 0) {
            const int qrow = (j * p.nkv + kvh) * p.RP + qt0 * BQ;
            mbar_arrive_expect_tx(q_full, n_str * Q_BYTES);
            for (int w = 0; w < n_str; ++w) {
                tma_load_2d(sQ + w * Q_BYTES, &tmQ, q_full, 0, qrow + w * BQ);
                tma_load_2d(sQ + w * Q_BYTES + HALF, &tmQ, q_full, 64, qrow + w * BQ);
            }
            const int kvrow0 = (int)((((long long)p.slot * p.max_batch + b) * p.nkv + kvh) * p.pos_stride);
            int k_issued = 0, v_issued = 0;
            for (int i = 0; i < n_tiles; ++i) {
                const int s = i & 1;
                const int row = kvrow0 + i * BKV;
                if (!mbar_wait(k_empty + s, ((uint32_t)(i >> 1) & 1u) ^ 1u, p.err)) break;
                mbar_arrive_expect_tx(k_full + s, KV_BYTES);
                tma_load_2d(sK + s * KV_BYTES, &tmK, k_full + s, 0, row);
                tma_load_2d(sK + s * KV_BYTES + HALF, &tmK, k_full + s, 64, row);
                k_issued = i + 1;
                if (!mbar_wait(v_empty, ((uint32_t)i & 1u) ^ 1u, p.err)) break;
                mbar_arrive_expect_tx(v_full, KV_BYTES);
                tma_load_2d(sV, &tmV, v_full, 0, row);
                tma_load_2d(sV + HALF, &tmV, v_full, 64, row);
                v_issued = i + 1;
            }
            // no copy into shared memory may still be in flight when the CTA exits
            mbar_wait(q_full, 0, p.err);
            for (int i = max(0, k_issued - K_STAGES); i < k_issued; ++i)
                mbar_wait(k_full + (i & 1), ((uint32_t)(i >> 1)) & 1u, p.err);
            if (v_issued > 0) mbar_wait(v_full, (uint32_t)(v_issued - 1) & 1u, p.err);
        }
    } else if (warp == 1) {
        if (lane == 0 && n_tiles > 0) {
            constexpr uint32_t idesc_s = umma_idesc_bf16(BQ, BKV);
            constexpr uint32_t idesc_o = umma_idesc_bf16(BQ, HD) | (1u << 16);  // B (V) MN-major
            const uint32_t q_addr = smem_u32(sQ), p_addr = smem_u32(sP), v_addr = smem_u32(sV);
            auto issue_s = [&](int w, int i) {
                const uint32_t k_addr = smem_u32(sK + (i & 1) * KV_BYTES);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
                    umma_f16(tmem + w * BKV, attn_tc::sdesc_k(q_addr + w * Q_BYTES + off), attn_tc::sdesc_k(k_addr + off),
                             idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(s_full + w);
            };
            bool ok = mbar_wait(q_full, 0, p.err) && mbar_wait(k_full, 0, p.err);
            if (ok) {
                tc_fence_after();
                for (int w = 0; w < n_str; ++w) issue_s(w, 0);
                umma_commit(k_empty);
            }
            for (int i = 0; i < n_tiles && ok; ++i) {
                if (i + 1 < n_tiles) {
                    // S of the next key tile as soon as each warpgroup has read its current S
                    if (!mbar_wait(k_full + ((i + 1) & 1), ((uint32_t)((i + 1) >> 1)) & 1u, p.err)) break;
                    for (int w = 0; w < n_str && ok; ++w) {
                        if (!mbar_wait(s_free + w, (uint32_t)i & 1u, p.err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_s(w, i + 1);
                    }
                    if (!ok) break;
                    umma_commit(k_empty + ((i + 1) & 1));
                }
                if (!mbar_wait(v_full, (uint32_t)i & 1u, p.err)) break;
                for (int w = 0; w < n_str && ok; ++w) {
                    if (!mbar_wait(p_full + w, (uint32_t)i & 1u, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t pb_addr = p_addr + w * P_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BKV / 16; ++kk) {
                        const uint32_t a_off = (kk >> 2) * HALF + (kk & 3) * 32;  // P: keys contiguous
                        const uint32_t b_off = kk * 16 * 128;                      // V: 16 key rows of 128 B
                        umma_f16(tmem + O_COL + w * HD, attn_tc::sdesc_k(pb_addr + a_off),
                                 attn_tc::sdesc_mn(v_addr + b_off, HALF), idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(pv_done + w);
                }
                if (!ok) break;
                umma_commit(v_empty);
            }
        }
    } else {
        // ---------------- softmax warpgroups: warps 2-5 query tile qt0, warps 6-9 qt0 + 1 ----------------
        const int w = (warp - 2) >> 2;
        const int q = warp & 3;       // TMEM lane quarter this warp may access
        const int t = q * 32 + lane;  // row of the tile = TMEM lane
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const uint32_t s_col = w * BKV, o_col = O_COL + w * HD;
        float m_ref = -INFINITY, l = 0.f;
        bool ok = n_tiles > 0 && w < n_str;
        for (int i = 0; i < n_tiles && ok; ++i) {
            if (!mbar_wait(s_full + w, (uint32_t)i & 1u, p.err)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float sv[BKV];
            {
                uint32_t r[BKV];
#pragma unroll
                for (int c0 = 0; c0 < BKV; c0 += 16) tmem_ld16_async(tmem + lane_base + s_col + c0, &r[c0]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < BKV; ++c) {
                    reg_after_wait(r[c]);
                    sv[c] = __uint_as_float(r[c]);
                }
            }
            // this warp is done with S_w: the next key tile's product may overwrite it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_free + w);
            const int key0 = i * BKV;
            if (key0 + BKV > p.kv_len) {  // ragged last tile (uniform across the CTA)
#pragma unroll
                for (int c = 0; c < BKV; ++c)
                    if (key0 + c >= p.kv_len) sv[c] = -INFINITY;
            }
            float mx[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) mx[c] = sv[c];
#pragma unroll
            for (int c = 8; c < BKV; ++c) mx[c & 7] = fmaxf(mx[c & 7], sv[c]);
            const float mt =
                fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) *
                p.scale_log2;
            const bool resc = mt > m_ref + RESCALE_THRESHOLD;
            const float f = (resc && i > 0) ? exp2f(m_ref - mt) : 1.f;
            if (resc) m_ref = mt;
            const float neg_m = -m_ref;
            float sm[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) sm[c] = 0.f;
#pragma unroll
            for (int c = 0; c < BKV; ++c) {
                sv[c] = ex2_approx(fmaf(sv[c], p.scale_log2, neg_m));
                sm[c & 7] += sv[c];
            }
            const float lt = ((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7]));
            l = l * f + lt;
            // P_w was last read by PV_w of the previous key tile, which a rescale of O_w also needs done
            if (i >= 1 && !mbar_wait(pv_done + w, (uint32_t)(i - 1) & 1u, p.err)) {
                ok = false;
                break;
            }
            if (resc && i > 0) {
                tc_fence_after();
#pragma unroll 1
                for (int c0 = 0; c0 < HD; c0 += 16) {
                    float v[16];
                    tmem_ld16(tmem + lane_base + o_col + c0, v);
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] *= f;
                    attn_tc::tmem_st16(tmem + lane_base + o_col + c0, v);
                }
            }
            // P row in the K-major 128-byte-swizzled layout (as attn_tc_kernel writes it)
            uint8_t *pbuf = sP + w * P_BYTES;
#pragma unroll
            for (int c = 0; c < BKV / 8; ++c) {
                uint4 pk;
                pk.x = attn_tc::pack2_bf16(sv[c * 8 + 0], sv[c * 8 + 1]);
                pk.y = attn_tc::pack2_bf16(sv[c * 8 + 2], sv[c * 8 + 3]);
                pk.z = attn_tc::pack2_bf16(sv[c * 8 + 4], sv[c * 8 + 5]);
                pk.w = attn_tc::pack2_bf16(sv[c * 8 + 6], sv[c * 8 + 7]);
                const int region = c >> 3, ch = c & 7;
                uint8_t *dst = pbuf + region * HALF + (t >> 3) * 1024 + (t & 7) * 128 + ((ch ^ (t & 7)) << 4);
                *reinterpret_cast<uint4 *>(dst) = pk;
            }
            attn_tc::fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(p_full + w);
        }
        // ---------------- output: O_w / l ----------------
        if (ok && mbar_wait(pv_done + w, (uint32_t)(n_tiles - 1) & 1u, p.err)) {
            tc_fence_after();
            const int rp = (qt0 + w) * BQ + t;
            const bool valid = rp < p.RP;
            const int tt = rp / p.G, h = kvh * p.G + rp % p.G;
            const int m = j * p.Tq + tt;
            const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
            for (int c0 = 0; c0 < HD; c0 += 16) {
                float v[16];
                tmem_ld16(tmem + lane_base + o_col + c0, v);
                if (valid) {
                    uint4 w0, w1;
                    w0.x = attn_tc::pack2_bf16(v[0] * inv, v[1] * inv);
                    w0.y = attn_tc::pack2_bf16(v[2] * inv, v[3] * inv);
                    w0.z = attn_tc::pack2_bf16(v[4] * inv, v[5] * inv);
                    w0.w = attn_tc::pack2_bf16(v[6] * inv, v[7] * inv);
                    w1.x = attn_tc::pack2_bf16(v[8] * inv, v[9] * inv);
                    w1.y = attn_tc::pack2_bf16(v[10] * inv, v[11] * inv);
                    w1.z = attn_tc::pack2_bf16(v[12] * inv, v[13] * inv);
                    w1.w = attn_tc::pack2_bf16(v[14] * inv, v[15] * inv);
                    bf16 *dst = p.out + (long long)m * p.out_ld + h * HD + c0;
                    *reinterpret_cast<uint4 *>(dst) = w0;
                    *reinterpret_cast<uint4 *>(dst + 8) = w1;
                }
            }
        }
        tc_fence_before();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace attn_pq
