// common.cuh — device helpers shared by the ALoDLM kernels (sm_100a only).
//
// PTX wrappers for mbarriers, TMA (cp.async.bulk.tensor, no multicast), and the fifth-
// generation tensor core (tcgen05.alloc/mma/commit/ld), plus bounded waits: every spin on
// an mbarrier gives up after a wall-clock limit, raises the device error word and lets
// the kernel unwind instead of hanging the GPU.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a only"
#endif

typedef __nv_bfloat16 bf16;

// device error word bits (host maps them to ALODLM_ETIMEOUT / ALODLM_EDEVICE)
#define DEVERR_TIMEOUT 1
#define DEVERR_BOUNDS 2

// wall-clock limit of one bounded wait (ns); far above any legitimate wait in this library
#define WAIT_LIMIT_NS 2000000000ull

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Thread-block cluster barrier in two halves (every thread of every CTA of the cluster
// arrives, then waits; the next arrive needs a wait in between).  Not .aligned: the threads
// of a warp may reach it on different paths.
__device__ __forceinline__ void cluster_arrive_relaxed() { asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory"); }
__device__ __forceinline__ void cluster_arrive_release() { asm volatile("barrier.cluster.arrive.release;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait_acquire() { asm volatile("barrier.cluster.wait.acquire;" ::: "memory"); }
// shared::cluster address of `local` (a shared-memory address of this CTA) in CTA `rank`
__device__ __forceinline__ uint32_t cluster_map(uint32_t local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_v2(uint32_t addr, float a, float b) {
    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b) : "memory");
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float a, float b, float c, float d) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// 2^x by the PTX ex2.approx instruction (one special-function-unit op; 2^-inf = 0)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

// Programmatic dependent launch: kernels of a step are launched so that a kernel's CTAs may
// start while its predecessor finishes.  pdl_wait() blocks until the predecessor grid has
// completed and its writes are visible (a no-op without the launch attribute); every kernel
// calls it before touching memory that a predecessor writes or reads.  pdl_trigger() lets
// the successor's CTAs be scheduled.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Entry of a kernel that touches predecessor data only after the wait.  With
// ALODLM_EARLY_TRIGGER=1 the successor may be scheduled before this kernel's own wait, so its
// input-independent prologue (barrier setup, weight or cached-K/V loads into its shared memory)
// overlaps this kernel and its predecessor.  This cannot deadlock: a successor is launched only
// once every CTA of this grid has started, and it reads nothing before its own wait.  Off by
// default: measured on a B200 it slows the few-row steps (Qwen3-8B shape bs 1: 10.39 vs 9.84
// ms; 1.7B: 5.16 vs 4.52 ms), the early successors taking SM slots from the kernels before them.
#ifndef ALODLM_EARLY_TRIGGER
#define ALODLM_EARLY_TRIGGER 0
#endif
__device__ __forceinline__ void pdl_enter() {
    if (ALODLM_EARLY_TRIGGER) {
        pdl_trigger();
        pdl_wait();
    } else {
        pdl_wait();
        pdl_trigger();
    }
}

// ---------------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the phase with the given parity has completed.  Returns false (and raises
// DEVERR_TIMEOUT) if that takes longer than WAIT_LIMIT_NS.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int *err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 0 && globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
            atomicOr(err, DEVERR_TIMEOUT);
            return false;
        }
    }
}

// named barrier of the 128 epilogue threads (warps 2-5) of a GEMM CTA
__device__ __forceinline__ void epilogue_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// the same barrier, returning whether `p` holds in every one of the 128 threads
__device__ __forceinline__ bool epilogue_all(bool p) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 1, 128, p;\n selp.u32 %0, 1, 0, q;\n}"
        : "=r"(r)
        : "r"((uint32_t)p)
        : "memory");
    return r != 0;
}

// ---------------------------------------------------------------------------------
// TMA (tiled, 2D, no multicast)
// ---------------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// Untiled bulk copy global -> this CTA's shared memory, completing on `bar` (no multicast):
// both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gsrc, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// orders this thread's view of global memory (generic proxy) before its later async-proxy
// (bulk copy) reads
__device__ __forceinline__ void fence_proxy_async_all() { asm volatile("fence.proxy.async;" ::: "memory"); }

// x = innermost (element) coordinate, y = row; x * sizeof(elem) must be a multiple of 16.
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(smem_dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tma_load_2d_hint(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int x, int y,
                                                 uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%3, "
        "%4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// ---------------------------------------------------------------------------------
// tcgen05: tensor memory and the 5th-generation MMA (cta_group::1)
// ---------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *smem_slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 inputs, f32 accumulate)
__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// arrive on an mbarrier once every tcgen05 op issued so far by this thread has completed
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 lanes x 16 columns of 32-bit TMEM words; thread i of the warp gets lane (base_lane + i)
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// One 32x32b.x16 TMEM load issued without waiting: several can be in flight, completed by
// one tmem_wait_ld(); reg_after_wait() then ties each register to that wait so that no use of
// it is scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld16_async(uint32_t taddr, uint32_t *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void reg_after_wait(uint32_t &x) { asm volatile("" : "+r"(x)); }

// Instruction descriptor, kind::f16: D f32, A and B bf16, both K-major, shape M x N.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
    return (1u << 4)                          // D format: f32
           | (1u << 7)                        // A format: bf16
           | (1u << 10)                       // B format: bf16
           | ((uint32_t)(N >> 3) << 17)       // N / 8
           | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// Shared-memory matrix descriptor for a K-major tile written by TMA with 128-byte swizzle:
// rows of 64 bf16 (128 B), 8-row swizzle atoms 1024 B apart.  Tile base 1024-aligned.
__device__ __forceinline__ uint64_t umma_sdesc_sw128(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4)      // start address
           | ((uint64_t)1 << 16)                    // leading byte offset (unused for swizzled K-major)
           | ((uint64_t)(1024 >> 4) << 32)          // stride byte offset: 8 rows x 128 B
           | ((uint64_t)1 << 46)                    // descriptor version (sm100)
           | ((uint64_t)2 << 61);                   // swizzle mode: 128 B
}

// ---------------------------------------------------------------------------------
// CTA pairs: tcgen05 with cta_group::2 (two CTAs of a cluster, ranks 2k and 2k+1, run one
// MMA of M = 256: each holds 128 rows of A and half of B in its own shared memory and gets its
// 128 accumulator rows in its own tensor memory).  No multicast anywhere: every load lands in
// the CTA that issues it.
// ---------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// allocate / release the same tensor-memory columns in both CTAs of the pair (one warp of each)
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *smem_slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D[tmem, both CTAs] (+)= A * B^T over the pair, kind::f16 (bf16 in, f32 accumulate); issued by
// one thread of the even CTA
__device__ __forceinline__ void umma_f16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// arrive on the mbarrier at shared::cluster address `bar` (this CTA's or its peer's) once every
// pair MMA issued so far by this thread has completed
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
// TMA 2D load into this CTA's shared memory whose completed bytes count on the mbarrier at
// shared::cluster address `bar`, which may be the peer's (the pair's MMA waits there)
__device__ __forceinline__ void tma_load_2d_pair(void *smem_dst, const CUtensorMap *map, uint32_t bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
        "%4}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(map), "r"(bar), "r"(x), "r"(y)
        : "memory");
}
// arrive (release, cluster scope) on the mbarrier at shared::cluster address `bar`
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}

// ---------------------------------------------------------------------------------
// misc math
// ---------------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Fixed-order block sum (deterministic): every warp reduces by a fixed butterfly, then
// warp 0 adds the warp partials in a fixed butterfly.  `red` holds >= 32 floats.
__device__ __forceinline__ float block_sum(float v, float *red) {
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = (blockDim.x + 31) >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    float t = (l < nw) ? red[l] : 0.f;
    if (w == 0) t = warp_sum(t);
    if (threadIdx.x == 0) red[0] = t;
    __syncthreads();
    float r = red[0];
    __syncthreads();
    return r;
}

__device__ __forceinline__ float silu_f(float x) { return x / (1.f + __expf(-x)); }

// ---------------------------------------------------------------------------------
// sampled commits: counter-based random numbers
// ---------------------------------------------------------------------------------

// Sampling state of a step (device memory, written by the step's first kernel): Gumbel noise
// is drawn under key (seed, step) when enabled.
struct SampleParams {
    unsigned long long seed, step;
    int enabled, pad;
};

// Philox4x64-10 (Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3",
// SC 2011): ten rounds, each two 64 x 64 -> 128-bit products of counter words with the
// round multipliers, the high halves xor-ed with the other counter words and the key; the key
// advances by the Weyl constants before every round but the first.  x: counter in, four
// random 64-bit words out.
__device__ __forceinline__ void philox4x64_10(uint64_t (&x)[4], uint64_t k0, uint64_t k1) {
    constexpr uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
    constexpr uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r) {
            k0 += W0;
            k1 += W1;
        }
        const uint64_t hi0 = __umul64hi(M0, x[0]), lo0 = M0 * x[0];
        const uint64_t hi1 = __umul64hi(M1, x[2]), lo1 = M1 * x[2];
        const uint64_t y0 = hi1 ^ x[1] ^ k0, y2 = hi0 ^ x[3] ^ k1;
        x[0] = y0;
        x[1] = lo1;
        x[2] = y2;
        x[3] = lo0;
    }
}

// Standard Gumbel variate from 64 random bits: u = (53 high bits + 1/2) * 2^-53 in (0, 1),
// g = -log(-log(u)), in double precision
__device__ __forceinline__ double gumbel_from_bits(uint64_t bits) {
    const double u = ((double)(bits >> 11) + 0.5) * 0x1.0p-53;
    return -log(-log(u));
}

// ---------------------------------------------------------------------------------
// q / k / v post-processing of one head (head_dim 128)
// ---------------------------------------------------------------------------------
// One head vector of head_dim 128 held by a warp, lane l owning d = 4l .. 4l+3: the per-head
// RMSNorm (weights w, when qk_norm) and rotate-half RoPE at the angles cs[e] of d % 64, for q
// and k heads (rope = true); v heads pass through.  Every path that prepares q, k or v calls
// this, so they all give the same bits.
__device__ __forceinline__ float4 head_post128(float4 x, bool rope, int qk_norm, float4 w, float eps,
                                               const float2 (&cs)[4], int lane) {
    float v[4] = {x.x, x.y, x.z, x.w};
    if (rope) {
        if (qk_norm) {
            float ss = v[0] * v[0] + v[1] * v[1] + v[2] * v[2] + v[3] * v[3];
            ss = warp_sum(ss);
            const float r = rsqrtf(ss / 128.f + eps);
            v[0] = v[0] * r * w.x;
            v[1] = v[1] * r * w.y;
            v[2] = v[2] * r * w.z;
            v[3] = v[3] * r * w.w;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float other = __shfl_xor_sync(0xffffffffu, v[e], 16);
            v[e] = (lane < 16) ? (v[e] * cs[e].x - other * cs[e].y) : (v[e] * cs[e].x + other * cs[e].y);
        }
    }
    return make_float4(v[0], v[1], v[2], v[3]);
}

// the RoPE angles (cos, sin) a lane needs for position pos (d = 4l + e, angle index d % 64)
__device__ __forceinline__ void rope_lane128(const float2 *rope, int pos, int lane, float2 (&cs)[4]) {
#pragma unroll
    for (int e = 0; e < 4; ++e) cs[e] = rope[(long long)pos * 64 + ((lane * 4 + e) & 63)];
}

__device__ __forceinline__ void store_bf16x4(bf16 *dst, float4 v) {
    __nv_bfloat162 b2[2] = {__floats2bfloat162_rn(v.x, v.y), __floats2bfloat162_rn(v.z, v.w)};
    *reinterpret_cast<uint2 *>(dst) = *reinterpret_cast<const uint2 *>(b2);
}

// row -> (sequence, position) of a batch of blocks laid out contiguously per sequence
struct RowMap {
    const int *seq_of;  // slot j -> sequence index b
    int rows_per_seq;   // N for a step, P for a prefill group (also the per-sequence packing stride of q)
    int pos0;           // position of row 0 of a sequence (P for a step, 0 for prefill)
    // Compacted rows (a prefill depth that runs only the positions whose exit depth reaches it),
    // all null otherwise: row m is the row_u[m]-th row of sequence slot row_seq[m], at position
    // pos0 + row_t[m]; slot j owns rows [seq_off[j], seq_off[j] + seq_cnt[j]).
    const int *row_seq = nullptr, *row_u = nullptr, *row_t = nullptr, *seq_off = nullptr, *seq_cnt = nullptr;
};

// sequence slot jj, index u among the slot's rows and position offset t of row m
__device__ __forceinline__ void row_of(const RowMap &mp, int m, int &jj, int &u, int &t) {
    if (mp.row_seq) {
        jj = mp.row_seq[m];
        u = mp.row_u[m];
        t = mp.row_t[m];
    } else {
        jj = m / mp.rows_per_seq;
        u = t = m % mp.rows_per_seq;
    }
}
