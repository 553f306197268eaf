// gemm_tc.cuh — bf16 GEMM on the fifth-generation tensor core (tcgen05 + TMEM + TMA).
//
// D[a, b] = sum_k A[a, k] * B[b, k], both operands K-major bf16 in global memory, f32
// accumulation in tensor memory.  One CTA computes one 128 x BN tile (128 rows of A = the
// MMA's M side, BN rows of B = its N side) over a range of K.  With split-K the S splits of a
// tile form one thread-block cluster: each CTA owns 128/S rows of the tile, every CTA stores
// its partial of those rows straight into the owner's shared memory (remote stores, no
// round-trip latency), one cluster barrier, and each owner adds the S partials in rank order
// (deterministic) and applies the epilogue.  Roles:
//   warp 0      one thread issues TMA loads of A and B k-tiles (64 wide, 128-byte swizzle)
//               into a ring of STAGES shared-memory slots,
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (M=128, N=BN, K=16) per
//               16-wide k step and releases each slot with tcgen05.commit,
//   warps 2-5   epilogue: tcgen05.ld the accumulator (thread = one A row, registers =
//               its BN columns) and apply the fused epilogue.
//
// For the decoder's linear layers A is the weight (output features on TMEM lanes) and B
// the activation rows (swap-AB): a 32-row step still fills the 128-row MMA, and the
// epilogue writes consecutive features from consecutive lanes (coalesced).  For the LM-head
// readout A is the readout rows and B the vocabulary, so each thread owns one row's logits
// and reduces them without shuffles; the logits never leave the SM.
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace gemm {

constexpr int BM = 128;
constexpr int BK = 64;

enum Epi { EPI_F32 = 0, EPI_ADD = 1, EPI_SWIGLU = 2, EPI_READOUT = 3 };

struct EpiParams {
    float *out;           // EPI_F32 / EPI_ADD: out[b_row * ldo + a_row]
    int ldo;
    bf16 *act;            // EPI_SWIGLU: act[b_row * ld_act + feature]
    int ld_act;
    float4 *partials;     // EPI_READOUT: partials[a_row * n_btiles + b_tile] = (max, sum e, sum e*d, argmax)
    int n_btiles;
    // EPI_READOUT with sampling (samp->enabled): spartials[a_row * n_btiles + b_tile] = (max of
    // z_v + g_v, its id v) with g_v the Gumbel noise of readout row a_row = position
    // rr_b[a_row] * N + rr_i[a_row] at loop `loop`
    double2 *spartials;
    const SampleParams *samp;
    const int *rr_b, *rr_i;
    int N, loop;
    // RMSNorm folded into the linear layers around it (y = x / rms(x) * g feeds a projection
    // W: y W^T = (1 / rms(x)) * ((x * g) W^T), the scale being one number per activation row).
    // Residual-add epilogue (EPI_ADD) with xg set: besides x it writes xg[b * ldo + f] =
    // bf16(x[b, f] * g_next[f]) -- the next projection's operand -- and partial sums of x[b, f]^2
    // over groups of features, ss[b * ss_ld + f / G]: G = 32 (per-tile kernel), 16 (split-K
    // owners), 128 (staged epilogue of the persistent and pair kernels).
    bf16 *xg;
    const float *g_next;
    float *ss;
    int ss_ld;
    // Projection after a folded RMSNorm (EPI_F32 / EPI_SWIGLU) with ss_in set: every output of
    // activation row b is scaled by 1 / sqrt(sum_{i < ss_n} ss_in[b * ss_ld + i] / norm_h + eps)
    // before the epilogue (SwiGLU: gate and up both).
    const float *ss_in;
    int ss_n;
    float norm_h, norm_eps;
};

// 1 / rms of activation rows b0 .. b0 + n - 1 (n a power of two, 32 .. 256) from their partial
// sums of squares, into rb[0, n), by the 128 epilogue threads (tid = 0 .. 127).  Every thread's
// loads are issued before its additions, so the whole computation costs about one L2 round
// trip: with n < 128 each row is shared by 128 / n consecutive threads, each summing a
// contiguous share of the partials in index order, then combined by a fixed butterfly; with
// n >= 128 each thread sums whole rows.  Deterministic.
__device__ __forceinline__ float sum_partials(const float *p, int cnt) {
    float acc = 0.f;
    int k = 0;
    for (; k + 16 <= cnt; k += 16) {
        float v[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = p[k + e];
#pragma unroll
        for (int e = 0; e < 16; ++e) acc += v[e];
    }
    for (; k < cnt; ++k) acc += p[k];
    return acc;
}
__device__ __forceinline__ void fold_scales(const EpiParams &ep, int b0, int n, int rowsB, float *rb, int tid) {
    if (n >= 128) {
        for (int i = tid; i < n; i += 128) {
            const int b = b0 + i;
            const float sq = b < rowsB ? sum_partials(ep.ss_in + (long long)b * ep.ss_ld, ep.ss_n) : 0.f;
            rb[i] = rsqrtf(sq / ep.norm_h + ep.norm_eps);
        }
    } else {
        const int tpr = 128 / n, i = tid / tpr, part = tid % tpr;  // tpr in {1, 2, 4}
        const int b = b0 + i;
        const int chunk = (ep.ss_n + tpr - 1) / tpr, k0 = min(ep.ss_n, part * chunk);
        const int cnt = min(ep.ss_n, k0 + chunk) - k0;
        float sq = b < rowsB ? sum_partials(ep.ss_in + (long long)b * ep.ss_ld + k0, cnt) : 0.f;
        for (int o = 1; o < tpr; o <<= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (part == 0) rb[i] = rsqrtf(sq / ep.norm_h + ep.norm_eps);
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    uint32_t u;
    memcpy(&u, &v, 4);
    return u;
}

// sum over the 16 lanes of an aligned half-warp
__device__ __forceinline__ float half_warp_sum(float v) {
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Write (EPI_F32) or add to (EPI_ADD) 16 consecutive rows of one output column: p points at
// row 0, rows `ld` floats apart, only the first `n_rows` exist.  For the residual add every
// old value is loaded before any store, so the 16 loads are in flight together.
template <int EPI>
__device__ __forceinline__ void store_chunk(const float (&v)[16], float *__restrict__ p, int ld, int n_rows) {
    if constexpr (EPI == EPI_ADD) {
        float old[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) old[j] = (j < n_rows) ? p[(long long)j * ld] : 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < n_rows) p[(long long)j * ld] = old[j] + v[j];
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < n_rows) p[(long long)j * ld] = v[j];
    }
}

// EPI_ADD over NC consecutive output columns (rows of p, `ld` floats apart; the first n_rows
// exist): every old value is loaded before any store, so all NC loads are in flight together.
template <int NC>
__device__ __forceinline__ void add_cols(const float (&v)[NC], float *__restrict__ p, int ld, int n_rows) {
    float old[NC];
#pragma unroll
    for (int j = 0; j < NC; ++j) old[j] = (j < n_rows) ? p[(long long)j * ld] : 0.f;
#pragma unroll
    for (int j = 0; j < NC; ++j)
        if (j < n_rows) p[(long long)j * ld] = old[j] + v[j];
}

// Operand layouts in global memory.  Plain: row-major [rows, K] (TMA box at x = k, y = row).
// Tiled (the library's own weights): every [tile_rows x 64] tile of the matrix stored
// contiguously, tiles ordered (row tile, k tile), k padded with zeros to a multiple of 64 --
// one TMA box then streams one contiguous run of HBM instead of tile_rows 128-byte pieces.
// `tiled` bit 0: operand A tiled with 128-row tiles; bit 1: operand B tiled with BN-row tiles.
__device__ __forceinline__ void tma_operand(void *dst, const CUtensorMap *map, uint64_t *bar, bool tiled, int tile,
                                            int tile_rows, int kt, int k_tiles) {
    if (tiled)
        tma_load_2d(dst, map, bar, 0, (tile * k_tiles + kt) * tile_rows);
    else
        tma_load_2d(dst, map, bar, kt * BK, tile * tile_rows);
}

// NC accumulator columns starting at column c0, summed over NACC accumulators BN columns
// apart (in accumulator order).  All loads are issued before one wait.
template <int NACC, int BN, int NC>
__device__ __forceinline__ void acc_ld(uint32_t taddr, int c0, float (&v)[NC]) {
    uint32_t r[NACC][NC];
#pragma unroll
    for (int a = 0; a < NACC; ++a)
#pragma unroll
        for (int c = 0; c < NC; c += 16) tmem_ld16_async(taddr + a * BN + c0 + c, &r[a][c]);
    tmem_wait_ld();
#pragma unroll
    for (int a = 0; a < NACC; ++a)
#pragma unroll
        for (int j = 0; j < NC; ++j) reg_after_wait(r[a][j]);
#pragma unroll
    for (int j = 0; j < NC; ++j) {
        float x = __uint_as_float(r[0][j]);
#pragma unroll
        for (int a = 1; a < NACC; ++a) x += __uint_as_float(r[a][j]);
        v[j] = x;
    }
}
template <int NACC, int BN>
__device__ __forceinline__ void acc_ld16(uint32_t taddr, int c0, float (&v)[16]) {
    acc_ld<NACC, BN, 16>(taddr, c0, v);
}

// Compile-time tuning of the few-row tiles: ring depth of the 32-wide tiles (4 keeps two CTAs
// per SM, which the 192-tile gate/up launch at 32 rows needs) and TMEM accumulators per tile
// for BN <= 64 (1: the MMAs of a stage chain on one accumulator; more measured no faster).
#ifndef ALODLM_STAGES_SMALL
#define ALODLM_STAGES_SMALL 4
#endif
#ifndef ALODLM_NACC_SMALL
#define ALODLM_NACC_SMALL 1
#endif

template <int BN>
struct Cfg {
    // 64-wide tiles take three stages so that two CTAs with their split-K receive buffer still
    // share an SM (four made it 131 KB: one CTA per SM, and the planner's 256-CTA split-K grids
    // ran in two waves)
    static constexpr int STAGES = (BN <= 32) ? ALODLM_STAGES_SMALL : (BN == 64 ? 3 : (BN == 128 ? 5 : 4));
    static constexpr uint32_t A_BYTES = BM * BK * 2;
    static constexpr uint32_t B_BYTES = BN * BK * 2;
    static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
    // With NACC > 1 the 16-wide k steps of a stage rotate over NACC independent TMEM
    // accumulators (shorter dependency chains for the small few-row MMAs), summed in a fixed
    // order by the epilogue; the default is one.
    static constexpr int NACC = (BN <= 64) ? ALODLM_NACC_SMALL : 1;
    // epilogue columns per TMEM round trip: a narrow tile's whole row at once
    static constexpr int EC = (BN <= 64) ? BN : 16;
    static constexpr uint32_t TMEM_COLS = BN * NACC;  // power of two >= 32
    // behind the ring: 256 bytes of barriers, then 1 KB of per-activation-row scales (folded
    // RMSNorm), then the kernel's own extra buffer
    static constexpr uint32_t RB_OFF = STAGES * STAGE_BYTES + 256;
    static constexpr uint32_t EXTRA_OFF = RB_OFF + 1024;
    static constexpr size_t SMEM = 1024 /*align slack*/ + (size_t)EXTRA_OFF;
    // split-K receive buffer: [split][owned row][BN + 4] f32.  Narrow tiles get a buffer of their own behind the barriers (a partial can then be
    // pushed while the owner is still streaming); wide tiles reuse the stage ring once every CTA
    // of the cluster is done with its own.
    static constexpr bool RECV_SEPARATE = BN <= 64;
    static constexpr int RECV_LD = BN + 4;  // floats per received row (16-byte aligned rows)
    static constexpr size_t RECV_BYTES = (size_t)BM * RECV_LD * 4;
    static constexpr size_t SMEM_SPLIT = SMEM + (RECV_SEPARATE ? RECV_BYTES : 0);
    // persistent kernel: behind the barriers, a [64 columns][128 rows] f32 staging tile through
    // which the epilogue turns its per-row registers into row-contiguous vector stores
    static constexpr size_t STG_BYTES = 64 * BM * 4;
    static constexpr size_t SMEM_PERSIST = SMEM + STG_BYTES;
    static_assert(RECV_SEPARATE || RECV_BYTES <= (size_t)STAGES * STAGE_BYTES, "split-K partials must fit the ring");
};

// Two CTAs per SM (the split-K planner counts on it for tiles up to 64 wide): registers are
// capped at 170 per thread (the 64-wide residual-add instance otherwise took 196, leaving one
// CTA per SM and its 256-CTA grids in two waves).
template <int BN, int EPI>
__global__ void __launch_bounds__(192, 2)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int rowsA,
                   int rowsB, const int *rowsA_dyn, int k_tiles, int kt_per_split, int a_fastest, int tiled,
                   EpiParams ep, int *err) {
    static_assert(EPI != EPI_READOUT, "the LM-head readout runs in the persistent kernel");
    using C = Cfg<BN>;
    constexpr int STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * C::STAGE_BYTES);
    uint64_t *empty = full + STAGES;
    uint64_t *accum = empty + STAGES;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accum + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int a_tile = a_fastest ? blockIdx.x : blockIdx.y;
    const int b_tile = a_fastest ? blockIdx.y : blockIdx.x;
    if (rowsA_dyn) {  // row count known only on the device (grid sized for the maximum)
        pdl_wait();
        const int live = *rowsA_dyn;
        if (a_tile * BM >= live) return;
        rowsA = min(rowsA, live);
    }
    const int split = blockIdx.z;
    const int kt0 = split * kt_per_split;
    const int nkt = min(k_tiles, kt0 + kt_per_split) - kt0;  // >= 1 by construction on the host

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        mbar_init(accum, 1);
        fence_mbarrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        // The A operand of the linear layers is a weight, which no kernel writes: its first
        // stages are requested right away (before the TMEM allocation and, under programmatic
        // dependent launch, before the predecessor kernel has finished), so the pipeline fills
        // while the rest starts up.  The readout's A operand is produced by the predecessor
        // (rowsA_dyn set): then everything waits.
        if (!rowsA_dyn) {
            const int pre = min(nkt, STAGES);
            for (int it = 0; it < pre; ++it) {
                mbar_arrive_expect_tx(full + it, C::STAGE_BYTES);
                tma_operand(smem + it * C::STAGE_BYTES, &tmA, full + it, tiled & 1, a_tile, BM, kt0 + it, k_tiles);
            }
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_trigger();
    constexpr bool SPLIT_EPI = EPI == EPI_F32 || EPI == EPI_ADD || EPI == EPI_SWIGLU;
    const bool split_k = SPLIT_EPI && gridDim.z > 1;
    float *recv = reinterpret_cast<float *>(C::RECV_SEPARATE ? smem + C::EXTRA_OFF : smem);
    float *rbuf = reinterpret_cast<float *>(smem + C::RB_OFF);  // 1 / rms per column (folded RMSNorm)
    // phase 0 of the cluster barrier: "every CTA of the cluster has started" (separate receive
    // buffer) or "every CTA is done with its stage ring" (receive buffer in the ring, arrived below)
    if (split_k && C::RECV_SEPARATE) cluster_arrive_relaxed();
    bool ep_ready = false;

    if (warp == 0) {
        if (lane == 0) {
            const int pre = rowsA_dyn ? 0 : min(nkt, STAGES);  // A stages already requested above
            pdl_wait();
            for (int it = 0; it < pre; ++it)
                tma_operand(smem + it * C::STAGE_BYTES + C::A_BYTES, &tmB, full + it, tiled & 2, b_tile, BN, kt0 + it,
                            k_tiles);
            int issued = pre;
            for (int it = pre; it < nkt; ++it) {
                const int s = it % STAGES;
                const uint32_t use = (uint32_t)(it / STAGES);
                if (!mbar_wait(empty + s, (use & 1u) ^ 1u, err)) break;
                mbar_arrive_expect_tx(full + s, C::STAGE_BYTES);
                uint8_t *sa = smem + s * C::STAGE_BYTES;
                const int kx = (kt0 + it) * BK;
                tma_operand(sa, &tmA, full + s, tiled & 1, a_tile, BM, kt0 + it, k_tiles);
                tma_operand(sa + C::A_BYTES, &tmB, full + s, tiled & 2, b_tile, BN, kt0 + it, k_tiles);
                (void)kx;
                issued = it + 1;
            }
            // make sure no copy into shared memory is still in flight when the CTA exits
            for (int it = max(0, issued - STAGES); it < issued; ++it)
                mbar_wait(full + (it % STAGES), (uint32_t)(it / STAGES) & 1u, err);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16(BM, BN);
            for (int it = 0; it < nkt; ++it) {
                const int s = it % STAGES;
                if (!mbar_wait(full + s, (uint32_t)(it / STAGES) & 1u, err)) break;
                tc_fence_after();
                const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
                const uint64_t da = umma_sdesc_sw128(sa);
                const uint64_t db = umma_sdesc_sw128(sa + C::A_BYTES);
#pragma unroll
                for (int k = 0; k < BK / 16; ++k)  // 16 bf16 = 32 bytes = 2 descriptor units per k step
                    umma_f16(tmem_base + (k % C::NACC) * BN, da + 2 * k, db + 2 * k, idesc,
                             (it > 0 || k >= C::NACC) ? 1u : 0u);
                umma_commit(empty + s);
            }
            umma_commit(accum);
        }
    } else {
        // ---------------- epilogue (warps 2..5) ----------------
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        pdl_wait();
        if constexpr (EPI == EPI_F32 || EPI == EPI_SWIGLU) {
            if (ep.ss_in) {  // the folded RMSNorm's row scales, while the MMAs run
                fold_scales(ep, b_tile * BN, BN, rowsB, rbuf, q * 32 + lane);
                epilogue_bar();
            }
        }
        const bool ready = mbar_wait(accum, 0, err);
        ep_ready = ready;
        tc_fence_after();
        const int a_row = a_tile * BM + q * 32 + lane;
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16);
        const int b0 = b_tile * BN;
        if (ready) {
            if constexpr (EPI == EPI_F32 || EPI == EPI_ADD || EPI == EPI_SWIGLU) {
                // final epilogue of one 16-column chunk (warp-uniform: SwiGLU and the folded
                // RMSNorm's sums of squares shuffle lanes)
                auto apply = [&](int c0, const float (&v_in)[16]) {
                    float v[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[j] = v_in[j];
                    if constexpr (EPI != EPI_ADD) {
                        if (ep.ss_in) {
#pragma unroll
                            for (int j = 0; j < 16; ++j) v[j] *= rbuf[c0 + j];
                        }
                    }
                    if constexpr (EPI == EPI_SWIGLU) {
                        // weight rows interleaved in groups of 32: 16 gate rows then the 16 up rows
                        // of the same features, so lane l < 16 holds gate and lane l + 16 holds up
                        const int feat = (a_row >> 5) * 16 + (lane & 15);
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float up = __shfl_xor_sync(0xffffffffu, v[j], 16);
                            const int br = b0 + c0 + j;
                            if (lane < 16 && a_row < rowsA && br < rowsB)
                                ep.act[(long long)br * ep.ld_act + feat] = __float2bfloat16_rn(silu_f(v[j]) * up);
                        }
                    } else if (EPI == EPI_ADD && ep.xg) {
                        // residual add feeding a folded RMSNorm: x, bf16(x * g), and per column the
                        // sum of x^2 over this warp's 32 features
                        const bool fv = a_row < rowsA;
                        const int nr = rowsB - (b0 + c0);
                        float *p = ep.out + (long long)(b0 + c0) * ep.ldo + a_row;
                        bf16 *px = ep.xg + (long long)(b0 + c0) * ep.ldo + a_row;
                        const float gf = fv ? ep.g_next[a_row] : 0.f;
                        float nv[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) nv[j] = (fv && j < nr) ? p[(long long)j * ep.ldo] : 0.f;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            nv[j] += v[j];
                            if (fv && j < nr) {
                                p[(long long)j * ep.ldo] = nv[j];
                                px[(long long)j * ep.ldo] = __float2bfloat16_rn(nv[j] * gf);
                            }
                        }
                        const int f0 = a_tile * BM + q * 32;  // first feature of this warp
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float sq = warp_sum((fv && j < nr) ? nv[j] * nv[j] : 0.f);
                            if (lane == 0 && j < nr && f0 < rowsA)
                                ep.ss[(long long)(b0 + c0 + j) * ep.ss_ld + f0 / 32] = sq;
                        }
                    } else if (a_row < rowsA) {
                        store_chunk<EPI>(v, ep.out + (long long)(b0 + c0) * ep.ldo + a_row, ep.ldo, rowsB - (b0 + c0));
                    }
                };
                if (gridDim.z == 1) {
                    for (int c0 = 0; c0 < BN; c0 += C::EC) {
                        if (b0 + c0 >= rowsB) break;  // warp-uniform
                        float v[C::EC];
                        acc_ld<C::NACC, BN, C::EC>(taddr, c0, v);
#pragma unroll
                        for (int sc = 0; sc < C::EC; sc += 16) {
                            if (b0 + c0 + sc >= rowsB) break;
                            apply(c0 + sc, *reinterpret_cast<const float(*)[16]>(&v[sc]));
                        }
                    }
                }  // split-K: pushed to the owners below
            }
        }
    }
    if constexpr (SPLIT_EPI) {
        if (split_k) {
            const int S = gridDim.z, r = split;  // cluster rank = split (S a power of two)
            const int rs = BM / S;                // tile rows owned by each rank
            const int lg_rs = __ffs(rs) - 1;
            constexpr int LD = C::RECV_LD;
            // With the receive buffer in the ring: an epilogue thread gets here only once the
            // accumulator is complete (every MMA has read its stage), so this arrival means
            // "this CTA no longer uses its ring".
            if (!C::RECV_SEPARATE) cluster_arrive_relaxed();
            cluster_wait_acquire();
            if (warp >= 2 && ep_ready) {
                // push this split's partial rows to their owners: row -> (owner, owned-row index)
                const int q = warp & 3, tr = q * 32 + lane;
                int owner, lr;
                if constexpr (EPI == EPI_SWIGLU) {
                    // owners split by feature so that a feature's gate and up rows (16 apart in
                    // each 32-row group) meet at one owner: features [o*fs, (o+1)*fs), gate rows
                    // first, then the up rows
                    const int fs = 64 / S, f = (tr >> 5) * 16 + (tr & 15);
                    owner = f / fs;
                    lr = (f - owner * fs) + ((tr & 16) ? fs : 0);
                } else {
                    owner = tr / rs;
                    lr = tr - owner * rs;
                }
                const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16);
                const uint32_t dst = cluster_map(smem_u32(recv + (size_t)(r * rs + lr) * LD), (uint32_t)owner);
                for (int c0 = 0; c0 < BN; c0 += C::EC) {
                    float v[C::EC];
                    acc_ld<C::NACC, BN, C::EC>(taddr, c0, v);
#pragma unroll
                    for (int j = 0; j < C::EC; j += 4)
                        st_cluster_v4(dst + (uint32_t)(c0 + j) * 4u, v[j], v[j + 1], v[j + 2], v[j + 3]);
                }
            }
            cluster_arrive_release();
            cluster_wait_acquire();  // every partial of the rows owned here has landed
            constexpr int NT = 192;
            if constexpr (EPI == EPI_SWIGLU) {
                const int fs = 64 / S, lg_fs = lg_rs - 1;
                for (int e = threadIdx.x; e < fs * BN; e += NT) {
                    const int fl = e & (fs - 1), col = e >> lg_fs;
                    float g = 0.f, u = 0.f;
                    for (int rr = 0; rr < S; ++rr) {
                        g += recv[(rr * rs + fl) * LD + col];
                        u += recv[(rr * rs + fs + fl) * LD + col];
                    }
                    if (ep.ss_in) {
                        g *= rbuf[col];
                        u *= rbuf[col];
                    }
                    const int ft = r * fs + fl, grow = (ft >> 4) * 32 + (ft & 15);
                    const int br = b_tile * BN + col;
                    if (a_tile * BM + grow < rowsA && br < rowsB)
                        ep.act[(long long)br * ep.ld_act + a_tile * 64 + ft] = __float2bfloat16_rn(silu_f(g) * u);
                }
            } else {
                // consecutive threads take consecutive rows of one output column (coalesced);
                // eight elements per thread at a time so that the residual loads overlap.  rs * BN
                // and NT are multiples of 32, so each warp's lanes enter every round together, and
                // an aligned half-warp holds 16 consecutive features of one column.
                const int total = rs * BN;
                for (int base = threadIdx.x; base < total; base += 8 * NT) {
                    float acc[8], old[8];
                    long long off[8];
                    bool ok[8];
                    int ars[8], brs[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int e = base + i * NT;
                        const int lrow = e & (rs - 1), col = e >> lg_rs;
                        const int ar = a_tile * BM + r * rs + lrow, br = b_tile * BN + col;
                        ars[i] = ar;
                        brs[i] = br;
                        ok[i] = e < total && ar < rowsA && br < rowsB;
                        off[i] = (long long)br * ep.ldo + ar;
                        float a = 0.f;
                        if (e < total)
                            for (int rr = 0; rr < S; ++rr) a += recv[(rr * rs + lrow) * LD + col];
                        if (EPI == EPI_F32 && ep.ss_in && e < total) a *= rbuf[col];
                        acc[i] = a;
                        old[i] = 0.f;
                    }
                    if constexpr (EPI == EPI_ADD) {
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            if (ok[i]) old[i] = ep.out[off[i]];
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        if (ok[i]) ep.out[off[i]] = old[i] + acc[i];
                    if constexpr (EPI == EPI_ADD) {
                        if (ep.xg) {  // folded RMSNorm: bf16(x * g) and sums of x^2 over 16 features
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const float nv = old[i] + acc[i];
                                if (ok[i]) ep.xg[off[i]] = __float2bfloat16_rn(nv * ep.g_next[ars[i]]);
                                const float sq = half_warp_sum(ok[i] ? nv * nv : 0.f);
                                if ((lane & 15) == 0 && base + i * NT < total && ars[i] < rowsA && brs[i] < rowsB)
                                    ep.ss[(long long)brs[i] * ep.ss_ld + ars[i] / 16] = sq;
                            }
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace gemm

namespace gemm {

// ---------------------------------------------------------------------------------
// Stream-K variant for few activation rows (one BN-row tile covers them all): a grid of at
// most one CTA per SM walks a contiguous, equal share of the (weight tile, k-tile) units, so
// every SM streams the same number of weight bytes.  The accumulator is double-buffered in
// TMEM (the epilogue of one tile overlaps the MMAs of the next).  A tile whose k range is
// split across CTAs is finished by the CTA that completes last: it sums the partials in
// segment order (deterministic, independent of arrival order) and applies the epilogue.
// ---------------------------------------------------------------------------------
#ifndef ALODLM_SK_STAGES
#define ALODLM_SK_STAGES 8
#endif
#ifndef ALODLM_SK_EVICT_FIRST
#define ALODLM_SK_EVICT_FIRST 1
#endif

template <int BN>
struct SkCfg {
    static constexpr int STAGES = ALODLM_SK_STAGES;
    static constexpr uint32_t A_BYTES = BM * BK * 2;
    static constexpr uint32_t B_BYTES = BN * BK * 2;
    static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr uint32_t TMEM_COLS = 2 * BN;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + 256;
};

template <int EPI, int BN>
__device__ __forceinline__ void sk_epilogue(const float (&acc)[BN], int a_row, int lane, int rowsA, int rowsB,
                                            const EpiParams &ep) {
    if constexpr (EPI == EPI_SWIGLU) {
        const int feat = (a_row >> 5) * 16 + (lane & 15);
#pragma unroll
        for (int j = 0; j < BN; ++j) {
            const float up = __shfl_xor_sync(0xffffffffu, acc[j], 16);
            if (lane < 16 && a_row < rowsA && j < rowsB)
                ep.act[(long long)j * ep.ld_act + feat] = __float2bfloat16_rn(silu_f(acc[j]) * up);
        }
    } else {
        if (a_row < rowsA) {
#pragma unroll
            for (int c0 = 0; c0 < BN; c0 += 16) {
                float v[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = acc[c0 + j];
                store_chunk<EPI>(v, ep.out + (long long)c0 * ep.ldo + a_row, ep.ldo, rowsB - c0);
            }
        }
    }
}

template <int BN, int EPI>
__global__ void __launch_bounds__(192, 1)
    gemm_sk_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int rowsA,
                   int rowsB, int k_tiles, int n_tiles, int upc, EpiParams ep, float *ws, int max_seg, int *counters,
                   int *err) {
    using C = SkCfg<BN>;
    constexpr int STAGES = C::STAGES;
    const long long total = (long long)n_tiles * k_tiles;
    const long long u0 = (long long)blockIdx.x * upc;
    const long long u1 = min(total, u0 + upc);
    if (u0 >= u1) return;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * C::STAGE_BYTES);
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;  // [2] accumulator buffer ready
    uint64_t *tempty = tfull + 2;      // [2] accumulator buffer drained
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
    int *last_flag = reinterpret_cast<int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull + b, 1);
            mbar_init(tempty + b, 4);
        }
        fence_mbarrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_w = l2_policy_evict_first();
            int issued = 0;
            for (long long u = u0; u < u1; ++u) {
                const int it = (int)(u - u0);
                const int s = it % STAGES;
                if (!mbar_wait(empty + s, ((uint32_t)(it / STAGES) & 1u) ^ 1u, err)) break;
                const int tile = (int)(u / k_tiles), kt = (int)(u % k_tiles);
                mbar_arrive_expect_tx(full + s, C::STAGE_BYTES);
                uint8_t *sa = smem + s * C::STAGE_BYTES;
                if (ALODLM_SK_EVICT_FIRST)
                    tma_load_2d_hint(sa, &tmA, full + s, kt * BK, tile * BM, pol_w);
                else
                    tma_load_2d(sa, &tmA, full + s, kt * BK, tile * BM);
                tma_load_2d(sa + C::A_BYTES, &tmB, full + s, kt * BK, 0);
                issued = it + 1;
            }
            for (int it = max(0, issued - STAGES); it < issued; ++it)
                mbar_wait(full + (it % STAGES), (uint32_t)(it / STAGES) & 1u, err);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16(BM, BN);
            int seg = 0;
            bool ok = true;
            for (long long u = u0; u < u1 && ok; ++u) {
                const int it = (int)(u - u0);
                const int s = it % STAGES;
                const int kt = (int)(u % k_tiles);
                const bool first = (u == u0) || kt == 0;
                const int buf = seg & 1;
                if (first && !mbar_wait(tempty + buf, ((uint32_t)(seg >> 1) & 1u) ^ 1u, err)) break;
                if (!mbar_wait(full + s, (uint32_t)(it / STAGES) & 1u, err)) break;
                tc_fence_after();
                const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
                const uint64_t da = umma_sdesc_sw128(sa);
                const uint64_t db = umma_sdesc_sw128(sa + C::A_BYTES);
#pragma unroll
                for (int k = 0; k < BK / 16; ++k)
                    umma_f16(tmem_base + buf * BN, da + 2 * k, db + 2 * k, idesc, (first && k == 0) ? 0u : 1u);
                umma_commit(empty + s);
                if (u + 1 == u1 || kt == k_tiles - 1) {
                    umma_commit(tfull + buf);
                    ++seg;
                }
            }
            (void)ok;
        }
    } else {
        const int q = warp & 3;
        const int ep_tid = threadIdx.x - 64;  // 0..127
        int seg = 0;
        long long u = u0;
        while (u < u1) {
            const int tile = (int)(u / k_tiles);
            const int kt_begin = (int)(u % k_tiles);
            const long long tile_end = (long long)(tile + 1) * k_tiles;
            const long long seg_end = min(u1, tile_end);
            const int buf = seg & 1;
            const bool ready = mbar_wait(tfull + buf, (uint32_t)(seg >> 1) & 1u, err);
            tc_fence_after();
            float acc[BN];
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + buf * BN;
#pragma unroll
            for (int c0 = 0; c0 < BN; c0 += 16) {
                float v[16];
                tmem_ld16(taddr + c0, v);
#pragma unroll
                for (int j = 0; j < 16; ++j) acc[c0 + j] = v[j];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty + buf);
            if (!ready) break;
            const int a_row = tile * BM + q * 32 + lane;
            if (kt_begin == 0 && seg_end == tile_end) {
                sk_epilogue<EPI, BN>(acc, a_row, lane, rowsA, rowsB, ep);
            } else {
                const int c_first = (int)(((long long)tile * k_tiles) / upc);
                const int c_last = (int)((tile_end - 1) / upc);
                const int nseg = c_last - c_first + 1;
                const int myseg = (int)blockIdx.x - c_first;
                float *mine = ws + (((long long)tile * max_seg + myseg) * BM + q * 32 + lane) * BN;
#pragma unroll
                for (int j = 0; j < BN; j += 4)
                    *reinterpret_cast<float4 *>(mine + j) = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
                __threadfence();
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (ep_tid == 0) {
                    const int prev = atomicAdd(counters + tile, 1);
                    *last_flag = (prev == nseg - 1);
                    if (prev == nseg - 1) counters[tile] = 0;  // every segment has arrived: re-arm
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (*last_flag) {
                    __threadfence();
                    float sum[BN];
#pragma unroll
                    for (int j = 0; j < BN; ++j) sum[j] = 0.f;
                    for (int sg = 0; sg < nseg; ++sg) {
                        const float *p = ws + (((long long)tile * max_seg + sg) * BM + q * 32 + lane) * BN;
#pragma unroll
                        for (int j = 0; j < BN; j += 4) {
                            const float4 v = __ldcg(reinterpret_cast<const float4 *>(p + j));
                            sum[j] += v.x;
                            sum[j + 1] += v.y;
                            sum[j + 2] += v.z;
                            sum[j + 3] += v.w;
                        }
                    }
                    sk_epilogue<EPI, BN>(sum, a_row, lane, rowsA, rowsB, ep);
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");  // last_flag is reused by the next segment
            }
            ++seg;
            u = seg_end;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace gemm

namespace gemm {

// ---------------------------------------------------------------------------------
// Persistent variant for many tiles: a grid of at most one CTA per SM walks the output tiles
// (consecutive CTAs share the weight tile, so it is read from HBM once), with the TMEM
// accumulator double-buffered so that the epilogue of one tile overlaps the MMAs of the next
// and the TMA ring streams across tile boundaries without a pipeline refill.
// ---------------------------------------------------------------------------------
template <int EPI, int BN>
__device__ __forceinline__ void linear_chunk(int c0, const float (&v)[16], int a_row, int lane, int b0, int rowsA,
                                             int rowsB, const EpiParams &ep) {
    if constexpr (EPI == EPI_SWIGLU) {
        const int feat = (a_row >> 5) * 16 + (lane & 15);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float up = __shfl_xor_sync(0xffffffffu, v[j], 16);
            const int br = b0 + c0 + j;
            if (lane < 16 && a_row < rowsA && br < rowsB)
                ep.act[(long long)br * ep.ld_act + feat] = __float2bfloat16_rn(silu_f(v[j]) * up);
        }
    } else if (a_row < rowsA) {
        store_chunk<EPI>(v, ep.out + (long long)(b0 + c0) * ep.ldo + a_row, ep.ldo, rowsB - (b0 + c0));
    }
}

template <int BN>
__device__ __forceinline__ void readout_tile(uint32_t taddr, int a_row, int b0, int b_tile, int rowsA, int rowsB,
                                             const EpiParams &ep) {
    float best = -INFINITY;
    int best_idx = b0;
    for (int c0 = 0; c0 < BN; c0 += 16) {
        if (b0 + c0 >= rowsB) break;
        float v[16];
        tmem_ld16(taddr + c0, v);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int vid = b0 + c0 + j;
            if (vid < rowsB && v[j] > best) {  // strict: lowest id wins ties
                best = v[j];
                best_idx = vid;
            }
        }
    }
    float se = 0.f, sed = 0.f;
    const float LOG2E = 1.4426950408889634f;
    for (int c0 = 0; c0 < BN; c0 += 16) {
        if (b0 + c0 >= rowsB) break;
        float v[16];
        tmem_ld16(taddr + c0, v);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            if (b0 + c0 + j < rowsB) {
                const float d = v[j] - best;
                const float e = exp2f(d * LOG2E);
                se += e;
                sed = fmaf(e, d, sed);
            }
        }
    }
    if (a_row < rowsA)
        ep.partials[(long long)a_row * ep.n_btiles + b_tile] = make_float4(best, se, sed, __int_as_float(best_idx));
    if (ep.samp != nullptr && ep.samp->enabled) {  // uniform: every lane takes part in the TMEM loads
        // Gumbel-max: the largest z_v + g_v of the tile and its id, in double precision
        const long long pos = a_row < rowsA ? (long long)ep.rr_b[a_row] * ep.N + ep.rr_i[a_row] : 0;
        const uint64_t k0 = ep.samp->seed, k1 = ep.samp->step;
        double sbest = -INFINITY;
        int sidx = b0;
        for (int c0 = 0; c0 < BN; c0 += 16) {
            if (b0 + c0 >= rowsB) break;
            float v[16];
            tmem_ld16(taddr + c0, v);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint64_t x[4] = {(uint64_t)((b0 + c0) / 4 + q), (uint64_t)pos, (uint64_t)ep.loop, 0ull};
                philox4x64_10(x, k0, k1);
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const int vid = b0 + c0 + 4 * q + w;
                    if (vid < rowsB) {
                        const double sc = (double)v[4 * q + w] + gumbel_from_bits(x[w]);
                        if (sc > sbest) {  // strict: lowest id wins ties
                            sbest = sc;
                            sidx = vid;
                        }
                    }
                }
            }
        }
        if (a_row < rowsA) ep.spartials[(long long)a_row * ep.n_btiles + b_tile] = make_double2(sbest, (double)sidx);
    }
}

// Epilogue of 64 accumulator columns [c0, c0 + 64) of a 128-row tile, by the 128 epilogue
// threads (thread = tile row `row`, v = its 64 values).  The values go through the staging tile
// stg[col][row] so that each warp then writes whole output rows: for the f32 / residual-add
// epilogues 128 consecutive features of one activation row as one 512-byte float4 store per
// warp, for SwiGLU the tile's 64 features (gate rows (f/16)*32 + f%16, up rows 16 further) of
// one activation row as bf16 pairs.  Falls back to per-element stores where a row is ragged or
// not 16-byte aligned.  Every epilogue thread must call it (named barriers).
template <int EPI>
__device__ __forceinline__ void staged_cols(float *stg, const float (&v)[64], int row, int a, int b_first,
                                            int rowsA, int rowsB, const EpiParams &ep) {
    constexpr int LD = BM;  // floats per staged column
#pragma unroll
    for (int j = 0; j < 64; ++j) stg[j * LD + row] = v[j];
    epilogue_bar();
    const int w = (threadIdx.x >> 5) & 3, lane = threadIdx.x & 31;
    if constexpr (EPI == EPI_SWIGLU) {
        const int f = 2 * lane;                       // features f, f + 1 of the tile
        const int g = (f >> 4) * 32 + (f & 15);       // their gate rows (adjacent)
        const bool fits = a * BM + g + 17 < rowsA + 1 && (ep.ld_act % 2) == 0;
#pragma unroll 4
        for (int j = w; j < 64; j += 4) {
            const int br = b_first + j;
            if (br >= rowsB) break;
            const float2 gt = *reinterpret_cast<const float2 *>(stg + j * LD + g);
            const float2 up = *reinterpret_cast<const float2 *>(stg + j * LD + g + 16);
            bf16 *dst = ep.act + (long long)br * ep.ld_act + a * 64 + f;
            if (fits) {
                *reinterpret_cast<__nv_bfloat162 *>(dst) = __floats2bfloat162_rn(silu_f(gt.x) * up.x, silu_f(gt.y) * up.y);
            } else {
                if (a * BM + g < rowsA) dst[0] = __float2bfloat16_rn(silu_f(gt.x) * up.x);
                if (a * BM + g + 1 < rowsA) dst[1] = __float2bfloat16_rn(silu_f(gt.y) * up.y);
            }
        }
    } else {
        const int r0 = 4 * lane;                      // tile rows r0 .. r0 + 3
        const bool vec = a * BM + BM <= rowsA && (ep.ldo % 4) == 0;
        constexpr int PER = 16;                       // output rows per warp per call
        float4 val[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) val[i] = *reinterpret_cast<const float4 *>(stg + (w + 4 * i) * LD + r0);
        if (EPI == EPI_ADD && ep.xg) {
            // residual add feeding a folded RMSNorm: x, bf16(x * g), and per output row the sum
            // of x^2 over the tile's 128 features (one warp covers them)
            float gg[4];
            bool fin[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                fin[e] = a * BM + r0 + e < rowsA;
                gg[e] = fin[e] ? ep.g_next[a * BM + r0 + e] : 0.f;
            }
            float4 old[PER];
#pragma unroll
            for (int i = 0; i < PER; ++i) {  // every old value in flight before any store
                const int br = b_first + w + 4 * i;
                const float *src = ep.out + (long long)br * ep.ldo + a * BM + r0;
                if (br >= rowsB) {
                    old[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                } else if (vec) {
                    old[i] = *reinterpret_cast<const float4 *>(src);
                } else {
                    old[i].x = fin[0] ? src[0] : 0.f;
                    old[i].y = fin[1] ? src[1] : 0.f;
                    old[i].z = fin[2] ? src[2] : 0.f;
                    old[i].w = fin[3] ? src[3] : 0.f;
                }
            }
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int br = b_first + w + 4 * i;
                if (br >= rowsB) break;  // uniform across the warp
                float *dst = ep.out + (long long)br * ep.ldo + a * BM + r0;
                bf16 *dx = ep.xg + (long long)br * ep.ldo + a * BM + r0;
                float nv[4] = {old[i].x + val[i].x, old[i].y + val[i].y, old[i].z + val[i].z, old[i].w + val[i].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) nv[e] = fin[e] ? nv[e] : 0.f;
                if (vec) {
                    *reinterpret_cast<float4 *>(dst) = make_float4(nv[0], nv[1], nv[2], nv[3]);
                    uint2 pk;
                    pk.x = pack_bf16x2(nv[0] * gg[0], nv[1] * gg[1]);
                    pk.y = pack_bf16x2(nv[2] * gg[2], nv[3] * gg[3]);
                    *reinterpret_cast<uint2 *>(dx) = pk;
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (fin[e]) {
                            dst[e] = nv[e];
                            dx[e] = __float2bfloat16_rn(nv[e] * gg[e]);
                        }
                }
                const float sq = warp_sum(nv[0] * nv[0] + nv[1] * nv[1] + nv[2] * nv[2] + nv[3] * nv[3]);
                if (lane == 0) ep.ss[(long long)br * ep.ss_ld + a] = sq;
            }
        } else if (vec) {
            float4 old[PER];
            if constexpr (EPI == EPI_ADD) {
#pragma unroll
                for (int i = 0; i < PER; ++i) {
                    const int br = b_first + w + 4 * i;
                    old[i] = br < rowsB ? *reinterpret_cast<const float4 *>(ep.out + (long long)br * ep.ldo + a * BM + r0)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int br = b_first + w + 4 * i;
                if (br >= rowsB) continue;
                float4 x = val[i];
                if constexpr (EPI == EPI_ADD) {
                    x.x += old[i].x;
                    x.y += old[i].y;
                    x.z += old[i].z;
                    x.w += old[i].w;
                }
                *reinterpret_cast<float4 *>(ep.out + (long long)br * ep.ldo + a * BM + r0) = x;
            }
        } else {
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int br = b_first + w + 4 * i;
                if (br >= rowsB) continue;
                float *dst = ep.out + (long long)br * ep.ldo + a * BM + r0;
                const float xs[4] = {val[i].x, val[i].y, val[i].z, val[i].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (a * BM + r0 + e < rowsA) {
                        if constexpr (EPI == EPI_ADD)
                            dst[e] += xs[e];
                        else
                            dst[e] = xs[e];
                    }
                }
            }
        }
    }
    epilogue_bar();  // the staging tile is free again
}

// Persistent kernel: at most one CTA per SM walks whole output tiles blockIdx.x,
// blockIdx.x + gridDim.x, ... with a double-buffered TMEM accumulator, so the epilogue of one
// tile overlaps the MMAs of the next and the TMA ring streams across tile boundaries.  No CTA
// waits on another CTA: every wait is on this CTA's own mbarriers.
template <int BN, int EPI>
__global__ void __launch_bounds__(192, 1)
    gemm_persist_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int rowsA,
                        int rowsB, const int *rowsA_dyn, int k_tiles, int a_fastest, int tiled, EpiParams ep,
                        int *err) {
    using C = Cfg<BN>;
    constexpr int STAGES = C::STAGES;
    constexpr uint32_t TCOLS = 2 * BN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * C::STAGE_BYTES);
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
    float *stg = reinterpret_cast<float *>(smem + C::EXTRA_OFF);  // epilogue staging
    float *rbuf = reinterpret_cast<float *>(smem + C::RB_OFF);     // 1 / rms per column (folded RMSNorm)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull + b, 1);
            mbar_init(tempty + b, 4);
        }
        fence_mbarrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TCOLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_trigger();
    if (rowsA_dyn) {  // row count known only on the device
        pdl_wait();
        rowsA = min(rowsA, *rowsA_dyn);
    }
    const int n_a = (rowsA + BM - 1) / BM, n_b = (rowsB + BN - 1) / BN;
    const int total = n_a * n_b;
    auto tile_of = [&](int t, int &a, int &b) {
        if (a_fastest) {
            a = t % n_a;
            b = t / n_a;
        } else {
            b = t % n_b;
            a = t / n_b;
        }
    };

    if (warp == 0) {
        if (lane == 0) {
            int t = blockIdx.x, a = 0, b = 0;
            // weights (operand A of the linear layers) do not depend on earlier kernels: the
            // first stages of the first tile are requested before waiting for them
            int pre = 0;
            if (t < total) {
                tile_of(t, a, b);
                pre = rowsA_dyn ? 0 : min(k_tiles, STAGES);
                for (int i = 0; i < pre; ++i) {
                    mbar_arrive_expect_tx(full + i, C::STAGE_BYTES);
                    tma_operand(smem + i * C::STAGE_BYTES, &tmA, full + i, tiled & 1, a, BM, i, k_tiles);
                }
            }
            pdl_wait();
            for (int i = 0; i < pre; ++i)
                tma_operand(smem + i * C::STAGE_BYTES + C::A_BYTES, &tmB, full + i, tiled & 2, b, BN, i, k_tiles);
            int g = 0, issued = pre;
            bool ok = true;
            for (; t < total && ok; t += gridDim.x) {
                tile_of(t, a, b);
                for (int kt = 0; kt < k_tiles; ++kt, ++g) {
                    if (g < pre) continue;
                    const int s = g % STAGES;
                    if (!mbar_wait(empty + s, ((uint32_t)(g / STAGES) & 1u) ^ 1u, err)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(full + s, C::STAGE_BYTES);
                    uint8_t *sa = smem + s * C::STAGE_BYTES;
                    tma_operand(sa, &tmA, full + s, tiled & 1, a, BM, kt, k_tiles);
                    tma_operand(sa + C::A_BYTES, &tmB, full + s, tiled & 2, b, BN, kt, k_tiles);
                    issued = g + 1;
                }
            }
            for (int i = max(0, issued - STAGES); i < issued; ++i)
                mbar_wait(full + (i % STAGES), (uint32_t)(i / STAGES) & 1u, err);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16(BM, BN);
            int g = 0, li = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++li) {
                const int buf = li & 1;
                if (!mbar_wait(tempty + buf, ((uint32_t)(li >> 1) & 1u) ^ 1u, err)) break;
                tc_fence_after();
                for (int kt = 0; kt < k_tiles; ++kt, ++g) {
                    const int s = g % STAGES;
                    if (!mbar_wait(full + s, (uint32_t)(g / STAGES) & 1u, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
                    const uint64_t da = umma_sdesc_sw128(sa);
                    const uint64_t db = umma_sdesc_sw128(sa + C::A_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma_f16(tmem_base + buf * BN, da + 2 * k, db + 2 * k, idesc, (kt > 0 || k > 0) ? 1u : 0u);
                    umma_commit(empty + s);
                }
                umma_commit(tfull + buf);
            }
        }
    } else {
        const int q = warp & 3;
        const int row = q * 32 + lane;  // row of the tile = TMEM lane
        pdl_wait();
        int li = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++li) {
            int a, b;
            tile_of(t, a, b);
            const int buf = li & 1;
            if constexpr (EPI == EPI_F32 || EPI == EPI_SWIGLU) {
                if (ep.ss_in) fold_scales(ep, b * BN, BN, rowsB, rbuf, row);  // ordered by the barrier below
            }
            // one verdict for all epilogue threads (they take named barriers below)
            const bool ready = epilogue_all(mbar_wait(tfull + buf, (uint32_t)(li >> 1) & 1u, err));
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + buf * BN;
            const int a_row = a * BM + row;
            const int b0 = b * BN;
            if (ready) {
                if constexpr (EPI == EPI_READOUT) {
                    readout_tile<BN>(taddr, a_row, b0, b, rowsA, rowsB, ep);
                } else {
                    // rounds of 64 columns: one TMEM wait, then row-contiguous stores
                    for (int c0 = 0; c0 < BN; c0 += 64) {
                        if (b0 + c0 >= rowsB) break;  // uniform across the epilogue warps
                        float v[64];
                        acc_ld<1, BN, 64>(taddr, c0, v);
                        if constexpr (EPI == EPI_F32 || EPI == EPI_SWIGLU) {
                            if (ep.ss_in) {
#pragma unroll
                                for (int j = 0; j < 64; ++j) v[j] *= rbuf[c0 + j];
                            }
                        }
                        staged_cols<EPI>(stg, v, row, a, b0 + c0, rowsA, rowsB, ep);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty + buf);
            if (!ready) break;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TCOLS);
    }
}

}  // namespace gemm

namespace gemm {

// ---------------------------------------------------------------------------------
// Persistent GEMM on CTA pairs (cta_group::2) for linear layers over many activation rows.
// A cluster of two CTAs computes 256 x 256 output tiles: 256 weight rows (each CTA loads its
// own 128, in the tiled weight layout) x 256 activation rows (each CTA loads its own 128), so
// per k-tile an SM streams 32 KB for 128 x 256 x 64 multiply-adds, two thirds of what a
// 128 x 256 tile on one SM needs.  The even CTA's MMA thread issues M = 256, N = 256 MMAs over
// both CTAs' shared memory; each CTA receives its 128 accumulator rows in its own tensor memory
// (double-buffered) and runs the usual staged epilogue on them.  Both CTAs' loads complete on
// the even CTA's stage barrier (which expects the bytes of both); the MMA releases each stage,
// and announces each finished accumulator, to both CTAs with one commit per CTA; both CTAs'
// epilogues report a drained accumulator to the even CTA.  No load is multicast.
// ---------------------------------------------------------------------------------
struct PairCfg {
    static constexpr int TN = 256;                        // activation rows per pair tile
    static constexpr int HALF = 128;                      // ... loaded by each CTA
    static constexpr int STAGES = 6;
    static constexpr uint32_t A_BYTES = BM * BK * 2;      // this CTA's 128 weight rows x 64
    static constexpr uint32_t B_BYTES = HALF * BK * 2;    // this CTA's 128 activation rows x 64
    static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr uint32_t TMEM_COLS = 2 * TN;         // two 128 x 256 f32 accumulators
    static constexpr size_t STG_BYTES = 64 * BM * 4;
    static constexpr uint32_t RB_OFF = STAGES * STAGE_BYTES + 256;  // 1 KB of per-row scales
    static constexpr uint32_t EXTRA_OFF = RB_OFF + 1024;             // staging tile
    static constexpr size_t SMEM = 1024 + (size_t)EXTRA_OFF + STG_BYTES;
};

__device__ __forceinline__ void tma_operand_pair(void *dst, const CUtensorMap *map, uint32_t bar, bool tiled, int tile,
                                                 int tile_rows, int kt, int k_tiles) {
    if (tiled)
        tma_load_2d_pair(dst, map, bar, 0, (tile * k_tiles + kt) * tile_rows);
    else
        tma_load_2d_pair(dst, map, bar, kt * BK, tile * tile_rows);
}

template <int EPI>
__global__ void __launch_bounds__(192, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int rowsA,
                     int rowsB, int k_tiles, int tiled_a, EpiParams ep, int *err) {
    static_assert(EPI == EPI_F32 || EPI == EPI_ADD || EPI == EPI_SWIGLU, "linear-layer epilogues only");
    using C = PairCfg;
    constexpr int STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * C::STAGE_BYTES);  // used in the even CTA
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + 2;    // used in the even CTA: 4 epilogue warps of each CTA arrive
    uint64_t *mma_done = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    float *stg = reinterpret_cast<float *>(smem + C::EXTRA_OFF);
    float *rbuf = reinterpret_cast<float *>(smem + C::RB_OFF);  // 1 / rms per column (folded RMSNorm)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank() & 1u;  // 0: the CTA whose thread issues the pair's MMAs
    const int pair = (int)(blockIdx.x >> 1), n_pairs = (int)(gridDim.x >> 1);
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull + b, 1);
            mbar_init(tempty + b, 8);
        }
        mbar_init(mma_done, 1);
        fence_mbarrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_arrive_release();
    cluster_wait_acquire();  // both CTAs' barriers are initialised before any cross-CTA signal
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_trigger();
    const int n_a = (rowsA + 2 * BM - 1) / (2 * BM), n_b = (rowsB + C::TN - 1) / C::TN;
    const int total = n_a * n_b;
    // shared::cluster addresses: the even CTA's stage and drain barriers, and each CTA's own
    const uint32_t full_lead = cluster_map(smem_u32(full), 0u);
    const uint32_t tempty_lead = cluster_map(smem_u32(tempty), 0u);

    if (warp == 0) {
        if (lane == 0) {
            int t = pair, issued = 0, g = 0, pre = 0;
            bool ok = true;
            // the weights do not depend on earlier kernels: the first stages of the first tile are
            // requested before waiting for them
            if (t < total) {
                const int a = t / n_b;
                pre = min(k_tiles, STAGES);
                for (int i = 0; i < pre; ++i) {
                    if (rank == 0) mbar_arrive_expect_tx(full + i, 2 * C::STAGE_BYTES);
                    tma_operand_pair(smem + i * C::STAGE_BYTES, &tmA, full_lead + 8u * i, tiled_a & 1, 2 * a + rank, BM,
                                     i, k_tiles);
                }
            }
            pdl_wait();
            if (t < total) {
                const int b = t % n_b;
                for (int i = 0; i < pre; ++i)
                    tma_load_2d_pair(smem + i * C::STAGE_BYTES + C::A_BYTES, &tmB, full_lead + 8u * i, i * BK,
                                     b * C::TN + (int)rank * C::HALF);
            }
            issued = pre;
            for (; t < total && ok; t += n_pairs) {
                const int a = t / n_b, b = t % n_b;
                for (int kt = 0; kt < k_tiles; ++kt, ++g) {
                    if (g < pre) continue;
                    const int s = g % STAGES;
                    if (!mbar_wait(empty + s, ((uint32_t)(g / STAGES) & 1u) ^ 1u, err)) {
                        ok = false;
                        break;
                    }
                    if (rank == 0) mbar_arrive_expect_tx(full + s, 2 * C::STAGE_BYTES);
                    uint8_t *sa = smem + s * C::STAGE_BYTES;
                    tma_operand_pair(sa, &tmA, full_lead + 8u * s, tiled_a & 1, 2 * a + rank, BM, kt, k_tiles);
                    tma_load_2d_pair(sa + C::A_BYTES, &tmB, full_lead + 8u * s, kt * BK, b * C::TN + (int)rank * C::HALF);
                    issued = g + 1;
                }
            }
            // no copy into this CTA's shared memory may still be in flight when it exits: a stage
            // is released (to both CTAs) only after the MMAs that read it, i.e. after it landed
            for (int i = max(0, issued - STAGES); i < issued; ++i)
                mbar_wait(empty + (i % STAGES), (uint32_t)(i / STAGES) & 1u, err);
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16(2 * BM, C::TN);
            const uint32_t empty_self = cluster_map(smem_u32(empty), 0u), empty_peer = cluster_map(smem_u32(empty), 1u);
            const uint32_t tfull_self = cluster_map(smem_u32(tfull), 0u), tfull_peer = cluster_map(smem_u32(tfull), 1u);
            int g = 0, li = 0;
            bool ok = true;
            for (int t = pair; t < total && ok; t += n_pairs, ++li) {
                const int buf = li & 1;
                if (!mbar_wait(tempty + buf, ((uint32_t)(li >> 1) & 1u) ^ 1u, err)) break;
                tc_fence_after();
                for (int kt = 0; kt < k_tiles; ++kt, ++g) {
                    const int s = g % STAGES;
                    if (!mbar_wait(full + s, (uint32_t)(g / STAGES) & 1u, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
                    const uint64_t da = umma_sdesc_sw128(sa);
                    const uint64_t db = umma_sdesc_sw128(sa + C::A_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma_f16_pair(tmem_base + buf * C::TN, da + 2 * k, db + 2 * k, idesc, (kt > 0 || k > 0) ? 1u : 0u);
                    umma_commit_pair(empty_self + 8u * s);
                    umma_commit_pair(empty_peer + 8u * s);
                }
                if (!ok) break;
                umma_commit_pair(tfull_self + 8u * buf);
                umma_commit_pair(tfull_peer + 8u * buf);
            }
            // every MMA issued above has completed before tensor memory is released
            umma_commit_pair(smem_u32(mma_done));
            mbar_wait(mma_done, 0, err);
        }
    } else {
        const int q = warp & 3;
        const int row = q * 32 + lane;  // row of this CTA's 128-row half = TMEM lane
        pdl_wait();
        int li = 0;
        for (int t = pair; t < total; t += n_pairs, ++li) {
            const int a = t / n_b, b = t % n_b;
            const int buf = li & 1;
            if constexpr (EPI == EPI_F32 || EPI == EPI_SWIGLU) {
                if (ep.ss_in) fold_scales(ep, b * C::TN, C::TN, rowsB, rbuf, row);  // ordered by the barrier below
            }
            const bool ready = epilogue_all(mbar_wait(tfull + buf, (uint32_t)(li >> 1) & 1u, err));
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + buf * C::TN;
            const int a128 = 2 * a + (int)rank;  // this CTA's 128 weight rows
            if (ready) {
                for (int c0 = 0; c0 < C::TN; c0 += 64) {
                    if (b * C::TN + c0 >= rowsB) break;  // uniform across the epilogue warps
                    float v[64];
                    acc_ld<1, C::TN, 64>(taddr, c0, v);
                    if constexpr (EPI == EPI_F32 || EPI == EPI_SWIGLU) {
                        if (ep.ss_in) {
#pragma unroll
                            for (int j = 0; j < 64; ++j) v[j] *= rbuf[c0 + j];
                        }
                    }
                    staged_cols<EPI>(stg, v, row, a128, b * C::TN + c0, rowsA, rowsB, ep);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty_lead + 8u * buf);
            if (!ready) break;
        }
    }
    tc_fence_before();
    cluster_arrive_release();
    cluster_wait_acquire();  // the pair is done with each other's barriers and tensor memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace gemm
