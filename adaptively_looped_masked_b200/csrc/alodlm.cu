// alodlm.cu — host side of the ALoDLM denoising-step library: the C ABI declared in
// include/alodlm.h, weight packing, the depth-aware KV arena, the prefill schedule and the
// looped denoising step.  Every step of the path runs in the kernels of this directory;
// the host only sizes launches and reads a 16-byte loop-control word per loop.
#include "../../include/alodlm.h"

#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <type_traits>
#include <vector>

#include "attention_pq.cuh"
#include "attention_tc.cuh"
#include "common.cuh"
#include "gemm_tc.cuh"
#include "kernels.cuh"

namespace {

// A named range on the host timeline (NVTX) around each phase of the library -- prefill,
// append, denoising step, loop s of a step (payload s), block decode -- so that a profiler
// which records NVTX (ncu --nvtx --nvtx-include) can pick out one phase's launches.  With no
// profiler attached each push and pop is a call that returns at once.
struct NvtxRange {
    explicit NvtxRange(const char *name, int payload = -1) {
        nvtxEventAttributes_t a = {};
        a.version = NVTX_VERSION;
        a.size = NVTX_EVENT_ATTRIB_STRUCT_SIZE;
        a.messageType = NVTX_MESSAGE_TYPE_ASCII;
        a.message.ascii = name;
        if (payload >= 0) {
            a.payloadType = NVTX_PAYLOAD_TYPE_INT32;
            a.payload.iValue = payload;
        }
        nvtxRangePushEx(&a);
    }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

// The step's linear layers and alodlm_gemm_bf16 use the per-tile kernel for few rows: on
// B200 it streams the weights faster than the stream-K kernel at 32-64 rows (0.77 vs 0.65 of
// the measured HBM bandwidth on the 24576 x 4096 gate/up shape).  Only the allocation-free
// entry point runs stream-K (its partials fit a fixed array there).
#ifndef ALODLM_MAX_SPLITS
#define ALODLM_MAX_SPLITS 8
#endif
// step attention may split keys over 16-CTA clusters (non-portable size) when they all fit
#ifndef ALODLM_ATTN_CLUSTER16
#define ALODLM_ATTN_CLUSTER16 1
#endif
// row count from which RMSNorm runs one warp per row (row in registers) instead of one block
// per row
#ifndef ALODLM_NORM_WARP_ROWS
#define ALODLM_NORM_WARP_ROWS 256
#endif
// RMSNorm folded into the residual-add and projection epilogues (1) or a norm kernel before
// every projection (0, the default: on a B200 the folded epilogues cost more than the norm
// launches they replace -- Qwen3-8B shape bs 1 10.24 vs 9.86 ms per step, bs 32 114.5 vs
// 110.6 ms -- although they pass the same parity tests)
#ifndef ALODLM_FOLD_NORM
#define ALODLM_FOLD_NORM 0
#endif

#ifndef ALODLM_PDL
#define ALODLM_PDL 1
#endif
#ifndef ALODLM_ATTN_PQ
#define ALODLM_ATTN_PQ 1
#endif

constexpr int NUM_SMS_HINT = 148;

// Launch with programmatic stream serialisation (the kernel may start while its predecessor
// on the stream finishes; the kernels order themselves with pdl_wait()).  Not on the legacy
// default stream.
template <typename... KArgs, typename... Args>
void klaunch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (ALODLM_PDL && st != nullptr && st != cudaStreamLegacy && st != cudaStreamPerThread) ? 1 : 0;
    cudaLaunchKernelEx(&cfg, kern, args...);
}

// The same with a thread-block cluster of (1, 1, cluster_z) CTAs.
template <typename... KArgs, typename... Args>
void klaunch_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster_z,
                     Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = cluster_z;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (ALODLM_PDL && st != nullptr && st != cudaStreamLegacy && st != cudaStreamPerThread) ? 2 : 1;
    cudaLaunchKernelEx(&cfg, kern, args...);
}
// The same with a thread-block cluster of (cluster_x, 1, 1) CTAs.
template <typename... KArgs, typename... Args>
void klaunch_cluster_x(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster_x,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster_x;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (ALODLM_PDL && st != nullptr && st != cudaStreamLegacy && st != cudaStreamPerThread) ? 2 : 1;
    cudaLaunchKernelEx(&cfg, kern, args...);
}
constexpr int PREFILL_ROWS = 16384;         // rows of one prefill group (sequences x P)

// KC_GEMM: linear layers on the pair and persistent kernels (many rows, tensor-bound);
// KC_GEMM_TILE: linear layers on the per-tile split-K kernel (few rows, weight streaming)
enum KClass { KC_GEMM = 0, KC_ATTN, KC_RGEMM, KC_RCOMB, KC_NORM, KC_QKV, KC_COMMIT, KC_OTHER, KC_GEMM_TILE };
const char *kclass_names[ALODLM_N_KCLASS] = {"gemm", "attention", "readout_gemm", "readout_combine",
                                             "norm", "qkv_rope", "commit", "other", "gemm_tile"};

std::mutex g_err_mu;
std::string g_create_err;

int round_up(int x, int m) { return (x + m - 1) / m * m; }
int cdiv(int a, int b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------------------------
// TMA descriptors (driver entry point fetched through the runtime)
// ---------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2D bf16 tensor [rows, inner] row-major, box [box_rows, 64], 128-byte swizzle, zero OOB fill
bool make_tmap(CUtensorMap *map, const void *ptr, int inner, int rows, int box_rows) {
    auto fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)inner * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// one-time per device: opt the big-shared-memory kernels in
template <int BN, int EPI>
void set_gemm_attr() {
    cudaFuncSetAttribute(gemm::gemm_tc_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)gemm::Cfg<BN>::SMEM_SPLIT);
}
template <int BN, int EPI>
void set_persist_attr() {
    cudaFuncSetAttribute(gemm::gemm_persist_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)gemm::Cfg<BN>::SMEM_PERSIST);
}
template <int EPI>
void set_pair_attr() {
    cudaFuncSetAttribute(gemm::gemm_pair_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)gemm::PairCfg::SMEM);
}
template <int BN, int EPI>
void set_sk_attr() {
    cudaFuncSetAttribute(gemm::gemm_sk_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)gemm::SkCfg<BN>::SMEM);
}
// CTA-pair kernel: clusters of two CTAs, as many pairs as the device holds at once (at most one
// per two SMs), each walking 256 x 256 tiles
#ifndef ALODLM_PAIR_GEMM
#define ALODLM_PAIR_GEMM 1
#endif
template <int EPI>
int pair_slots() {
    static int cached[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 0;
    if (!cached[dev]) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (NUM_SMS_HINT / 2));
        cfg.blockDim = dim3(192);
        cfg.dynamicSmemBytes = gemm::PairCfg::SMEM;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, gemm::gemm_pair_kernel<EPI>, &cfg) != cudaSuccess || n < 1) {
            cudaGetLastError();
            n = -1;  // the pair kernel cannot run here: the single-CTA kernels take its shapes
        }
        cached[dev] = n;
    }
    return cached[dev];
}

// How many 16-CTA clusters of the step attention can be resident at once (0: the
// non-portable cluster size is not available).  Looked up once per device, outside captures.
int attn_clusters16() {
    static int cached[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 0;
    if (!cached[dev]) {
        int n = 0;
        if (cudaFuncSetAttribute(attn_tc::attn_tc_kernel<128>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
            cudaSuccess) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(1, 16 * 8, 1);
            cfg.blockDim = dim3(192);
            cfg.dynamicSmemBytes = attn_tc::SMEM;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 1;
            attr[0].val.clusterDim.y = 16;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&n, attn_tc::attn_tc_kernel<128>, &cfg) != cudaSuccess) n = 0;
        }
        cudaGetLastError();
        cached[dev] = n > 0 ? n : -1;
    }
    return std::max(cached[dev], 0);
}

bool init_kernel_attrs() {
    static bool done[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return false;
    if (done[dev]) return true;
    set_gemm_attr<32, gemm::EPI_F32>();
    set_gemm_attr<32, gemm::EPI_ADD>();
    set_gemm_attr<32, gemm::EPI_SWIGLU>();
    set_gemm_attr<64, gemm::EPI_F32>();
    set_gemm_attr<64, gemm::EPI_ADD>();
    set_gemm_attr<64, gemm::EPI_SWIGLU>();
    set_gemm_attr<128, gemm::EPI_F32>();
    set_gemm_attr<128, gemm::EPI_ADD>();
    set_gemm_attr<128, gemm::EPI_SWIGLU>();
    set_gemm_attr<256, gemm::EPI_F32>();
    set_gemm_attr<256, gemm::EPI_ADD>();
    set_gemm_attr<256, gemm::EPI_SWIGLU>();
    set_persist_attr<128, gemm::EPI_F32>();
    set_persist_attr<128, gemm::EPI_ADD>();
    set_persist_attr<128, gemm::EPI_SWIGLU>();
    set_persist_attr<256, gemm::EPI_F32>();
    set_persist_attr<256, gemm::EPI_ADD>();
    set_persist_attr<256, gemm::EPI_SWIGLU>();
    set_persist_attr<256, gemm::EPI_READOUT>();
    set_pair_attr<gemm::EPI_F32>();
    set_pair_attr<gemm::EPI_ADD>();
    set_pair_attr<gemm::EPI_SWIGLU>();
    set_sk_attr<32, gemm::EPI_F32>();
    set_sk_attr<32, gemm::EPI_ADD>();
    set_sk_attr<32, gemm::EPI_SWIGLU>();
    set_sk_attr<64, gemm::EPI_F32>();
    set_sk_attr<64, gemm::EPI_ADD>();
    set_sk_attr<64, gemm::EPI_SWIGLU>();
    cudaFuncSetAttribute(attn_tc::attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)attn_tc::smem_bytes<128>());
    cudaFuncSetAttribute(attn_tc::attn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)attn_tc::smem_bytes<64>());
    cudaFuncSetAttribute(attn_pq::attn_pq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)attn_pq::SMEM);
    done[dev] = cudaGetLastError() == cudaSuccess;
    if (done[dev]) {  // occupancies, looked up here (never during a graph capture)
        pair_slots<gemm::EPI_F32>();
        pair_slots<gemm::EPI_ADD>();
        pair_slots<gemm::EPI_SWIGLU>();
        attn_clusters16();
    }
    return done[dev];
}

// Activation rows per tile: the smallest of 32/64/128 that covers them up to 128 rows; above,
// 256-row tiles only once they still give at least one tile per SM (fewer, fatter tiles
// leave SMs idle on mid-sized row counts).
int pick_bn(int M, int Nw) {
    if (M <= 32) return 32;
    if (M <= 64) return 64;
    if (M <= 128) return 128;
    return (cdiv(Nw, 128) * cdiv(M, 256) >= NUM_SMS_HINT) ? 256 : 128;
}

struct GemmShape {
    int bn, splits, kps, k_tiles;
};

// Tile/split choice: enough CTAs to cover the SMs (memory-bound small-M launches), at least
// four k-tiles per split, at most 8 splits (one cluster).
GemmShape plan_gemm(int M, int Nw, int K) {
    GemmShape g;
    g.bn = pick_bn(M, Nw);
    g.k_tiles = cdiv(K, gemm::BK);
    const int tiles = cdiv(Nw, gemm::BM) * cdiv(M, g.bn);
    const int per_sm = g.bn <= 64 ? 2 : 1;
    int splits = (NUM_SMS_HINT * per_sm) / tiles;
    // splits form one cluster (portable size <= 8, a power of two so that the ranks share the
    // 128 tile rows evenly in the reduction); at least 4 k-tiles each
    splits = std::max(1, std::min(std::min(splits, ALODLM_MAX_SPLITS), g.k_tiles / 4));
    while (splits & (splits - 1)) --splits;
    // equal k-ranges of cdiv(k_tiles, splits) must give exactly `splits` non-empty ranges (the
    // cluster reduction needs a power of two; e.g. 33 k-tiles in 8 ranges of 5 leave only 7)
    while (splits > 1 && cdiv(g.k_tiles, cdiv(g.k_tiles, splits)) != splits) splits >>= 1;
    g.kps = cdiv(g.k_tiles, splits);
    g.splits = splits;
    return g;
}

template <int BN, int EPI>
void launch_gemm_bn(const CUtensorMap &tA, const CUtensorMap &tB, int rowsA, int rowsB, int k_tiles, int kps,
                    int splits, int a_fastest, const gemm::EpiParams &ep, int *err, cudaStream_t st, int tiled) {
    dim3 grid;
    const int ta = cdiv(rowsA, gemm::BM), tb = cdiv(rowsB, BN);
    grid = a_fastest ? dim3(ta, tb, splits) : dim3(tb, ta, splits);
    if (splits > 1)
        klaunch_cluster(gemm::gemm_tc_kernel<BN, EPI>, grid, 192, gemm::Cfg<BN>::SMEM_SPLIT, st, splits, tA, tB, rowsA,
                        rowsB, (const int *)nullptr, k_tiles, kps, a_fastest, tiled, ep, err);
    else
        klaunch(gemm::gemm_tc_kernel<BN, EPI>, grid, 192, gemm::Cfg<BN>::SMEM, st, tA, tB, rowsA, rowsB,
                (const int *)nullptr, k_tiles, kps, a_fastest, tiled, ep, err);
}

// persistent kernel: one CTA per SM at most, walking whole tiles
template <int BN, int EPI>
void launch_persist(const CUtensorMap &tA, const CUtensorMap &tB, int rowsA, int rowsB, const int *rowsA_dyn,
                    int k_tiles, int a_fastest, const gemm::EpiParams &ep, int *err, cudaStream_t st, int num_sms,
                    int tiled) {
    const int tiles = cdiv(rowsA, gemm::BM) * cdiv(rowsB, BN);
    const int grid = std::max(1, std::min(num_sms, tiles));
    klaunch(gemm::gemm_persist_kernel<BN, EPI>, grid, 192, gemm::Cfg<BN>::SMEM_PERSIST, st, tA, tB, rowsA, rowsB, rowsA_dyn,
            k_tiles, a_fastest, tiled, ep, err);
}

template <int EPI>
void launch_pair(const CUtensorMap &tA, const CUtensorMap &tB, int rowsA, int rowsB, int k_tiles, int tiled_a,
                 const gemm::EpiParams &ep, int *err, cudaStream_t st, int n_pairs) {
    klaunch_cluster_x(gemm::gemm_pair_kernel<EPI>, dim3(2 * n_pairs), dim3(192), gemm::PairCfg::SMEM, st, 2, tA, tB,
                      rowsA, rowsB, k_tiles, tiled_a, ep, err);
}

template <int EPI>
void launch_gemm_epi(int bn, const CUtensorMap &tA, const CUtensorMap &tB, int rowsA, int rowsB, int k_tiles, int kps,
                     int splits, int a_fastest, const gemm::EpiParams &ep, int *err, cudaStream_t st, int tiled) {
    switch (bn) {
        case 32: launch_gemm_bn<32, EPI>(tA, tB, rowsA, rowsB, k_tiles, kps, splits, a_fastest, ep, err, st, tiled); break;
        case 64: launch_gemm_bn<64, EPI>(tA, tB, rowsA, rowsB, k_tiles, kps, splits, a_fastest, ep, err, st, tiled); break;
        case 128:
            launch_gemm_bn<128, EPI>(tA, tB, rowsA, rowsB, k_tiles, kps, splits, a_fastest, ep, err, st, tiled);
            break;
        default:
            launch_gemm_bn<256, EPI>(tA, tB, rowsA, rowsB, k_tiles, kps, splits, a_fastest, ep, err, st, tiled);
            break;
    }
}

// Where a GEMM may put its scratch: split-K / stream-K partials, stream-K tile counters
// (zero between launches; every launch leaves them zero), the device error word.
struct GemmEnv {
    float *ws;
    size_t ws_floats;
    int *counters;
    int n_counters;
    int *err;
    cudaStream_t st;
    int num_sms;
};

struct SkPlan {
    int bn, grid, upc, max_seg, n_tiles, k_tiles;
};

// Stream-K partition: at most one CTA per SM, equal numbers of (weight tile, k-tile) units.
SkPlan plan_sk(int M, int Nw, int K, int num_sms) {
    SkPlan p;
    p.bn = M <= 32 ? 32 : 64;
    p.k_tiles = cdiv(K, gemm::BK);
    p.n_tiles = cdiv(Nw, gemm::BM);
    const long long total = (long long)p.n_tiles * p.k_tiles;
    const int grid0 = (int)std::min<long long>(num_sms, total);
    p.upc = (int)((total + grid0 - 1) / grid0);
    p.grid = (int)((total + p.upc - 1) / p.upc);
    p.max_seg = 1;
    for (int t = 0; t < p.n_tiles; ++t) {
        const long long a = (long long)t * p.k_tiles, b = (long long)(t + 1) * p.k_tiles - 1;
        p.max_seg = std::max(p.max_seg, (int)(b / p.upc - a / p.upc + 1));
    }
    return p;
}

template <int BN, int EPI>
void launch_sk_bn(const SkPlan &p, const CUtensorMap &tW, const CUtensorMap &tB, int Nw, int M,
                  const gemm::EpiParams &ep, const GemmEnv &env) {
    klaunch(gemm::gemm_sk_kernel<BN, EPI>, p.grid, 192, gemm::SkCfg<BN>::SMEM, env.st, 
        tW, tB, Nw, M, p.k_tiles, p.n_tiles, p.upc, ep, env.ws, p.max_seg, env.counters, env.err);
}

template <int EPI>
void launch_sk(const SkPlan &p, const CUtensorMap &tW, const CUtensorMap &tB, int Nw, int M,
               const gemm::EpiParams &ep, const GemmEnv &env) {
    if (p.bn == 32)
        launch_sk_bn<32, EPI>(p, tW, tB, Nw, M, ep, env);
    else
        launch_sk_bn<64, EPI>(p, tW, tB, Nw, M, ep, env);
}

// The RMSNorm folded into the linear layers around it (see EpiParams): what a residual-add
// GEMM also writes for the next projection, and what a projection reads in its place.
struct Fold {
    bf16 *xg = nullptr;            // producer: bf16(x * g_next)
    const float *g_next = nullptr;
    float *ss = nullptr;           // producer: partial sums of x^2, [row][ss_ld]
    const float *ss_in = nullptr;  // consumer: the partials to scale by
    int ss_ld = 0, ss_n = 0;
    float norm_h = 0.f, eps = 0.f;
};

// out = act[M, K] x W[Nw, K]^T with epilogue `epi`: one CTA per 128 x BN tile with split-K
// inside a cluster when the tiles do not fill the SMs; otherwise the pair or the persistent
// kernel.  map_for_bn(bn) returns the activation's tensor map with BN-row boxes.  `ss_group`
// (if set) receives the number of features per partial sum a folding residual add writes on
// the path taken; `per_tile` (if set) whether the per-tile kernel ran.  Returns the number of
// kernels launched, or -1 (tensor map failure).
template <typename MapFn>
int run_gemm(const GemmEnv &env, const CUtensorMap &tmW, int Nw, MapFn map_for_bn, int M, int K, int epi, float *out,
             int ldo, bf16 *act_out, int ld_act, int w_tiled, const Fold &fold = Fold{}, int *ss_group = nullptr,
             bool *per_tile = nullptr) {
    if (per_tile) *per_tile = false;
    gemm::EpiParams ep{};
    ep.out = out;
    ep.ldo = ldo;
    ep.act = act_out;
    ep.ld_act = ld_act;
    ep.xg = fold.xg;
    ep.g_next = fold.g_next;
    ep.ss = fold.ss;
    ep.ss_in = fold.ss_in;
    ep.ss_ld = fold.ss_ld;
    ep.ss_n = fold.ss_n;
    ep.norm_h = fold.norm_h;
    ep.norm_eps = fold.eps;
    int group_dummy;
    int &group = ss_group ? *ss_group : group_dummy;
    group = 128;  // the staged epilogue of the pair and persistent kernels
    GemmShape g = plan_gemm(M, Nw, K);
    if (ALODLM_PAIR_GEMM && g.splits == 1 && g.bn >= 128 && M > 128) {
        // 256 x 256 tiles on CTA pairs once they fill every pair at least once
        const int slots = epi == gemm::EPI_F32 ? pair_slots<gemm::EPI_F32>()
                          : epi == gemm::EPI_ADD ? pair_slots<gemm::EPI_ADD>() : pair_slots<gemm::EPI_SWIGLU>();
        const int tiles = cdiv(Nw, 256) * cdiv(M, 256);
        if (slots > 0 && tiles >= slots) {
            const CUtensorMap *tB = map_for_bn(128);
            if (!tB) return -1;
            if (epi == gemm::EPI_F32)
                launch_pair<gemm::EPI_F32>(tmW, *tB, Nw, M, g.k_tiles, w_tiled, ep, env.err, env.st, slots);
            else if (epi == gemm::EPI_ADD)
                launch_pair<gemm::EPI_ADD>(tmW, *tB, Nw, M, g.k_tiles, w_tiled, ep, env.err, env.st, slots);
            else
                launch_pair<gemm::EPI_SWIGLU>(tmW, *tB, Nw, M, g.k_tiles, w_tiled, ep, env.err, env.st, slots);
            return 1;
        }
    }
    const CUtensorMap *tB = map_for_bn(g.bn);
    if (!tB) return -1;
    if (g.splits == 1 && g.bn >= 128) {
        auto go = [&](auto bn_tag) {
            constexpr int BN = decltype(bn_tag)::value;
            switch (epi) {
                case gemm::EPI_F32:
                    launch_persist<BN, gemm::EPI_F32>(tmW, *tB, Nw, M, nullptr, g.k_tiles, 0, ep, env.err, env.st,
                                                      env.num_sms, w_tiled);
                    break;
                case gemm::EPI_ADD:
                    launch_persist<BN, gemm::EPI_ADD>(tmW, *tB, Nw, M, nullptr, g.k_tiles, 0, ep, env.err, env.st,
                                                      env.num_sms, w_tiled);
                    break;
                default:
                    launch_persist<BN, gemm::EPI_SWIGLU>(tmW, *tB, Nw, M, nullptr, g.k_tiles, 0, ep, env.err, env.st,
                                                         env.num_sms, w_tiled);
                    break;
            }
        };
        if (g.bn == 128)
            go(std::integral_constant<int, 128>{});
        else
            go(std::integral_constant<int, 256>{});
        return 1;
    }
    group = g.splits > 1 ? 16 : 32;  // split-K owners: half-warps; one CTA per tile: warps
    if (per_tile) *per_tile = true;
    if (epi == gemm::EPI_F32)
        launch_gemm_epi<gemm::EPI_F32>(g.bn, tmW, *tB, Nw, M, g.k_tiles, g.kps, g.splits, 0, ep, env.err, env.st, w_tiled);
    else if (epi == gemm::EPI_ADD)
        launch_gemm_epi<gemm::EPI_ADD>(g.bn, tmW, *tB, Nw, M, g.k_tiles, g.kps, g.splits, 0, ep, env.err, env.st, w_tiled);
    else
        launch_gemm_epi<gemm::EPI_SWIGLU>(g.bn, tmW, *tB, Nw, M, g.k_tiles, g.kps, g.splits, 0, ep, env.err, env.st, w_tiled);
    return 1;
}

struct LayerDev {
    bf16 *wqkv = nullptr, *wo = nullptr, *wgu = nullptr, *wd = nullptr;
    float *attn_norm = nullptr, *mlp_norm = nullptr, *q_norm = nullptr, *k_norm = nullptr;
    CUtensorMap tm_qkv, tm_o, tm_gu, tm_d;
};

struct TimedLaunch {
    int cls;
    cudaEvent_t e0, e1;
};

// A loop's recorded graph bakes in everything below: the prefix length and the deepest built
// Core depth fix the attended positions and slots.
struct GraphKey {
    int s, n_act, cur, hi, N, K, rule, P, depth;
    float tau, lam;
    const void *p0, *p1, *p2, *p3, *p4, *p5, *p6, *p7;
    bool operator==(const GraphKey &o) const {
        return s == o.s && n_act == o.n_act && cur == o.cur && hi == o.hi && N == o.N && K == o.K &&
               rule == o.rule && P == o.P && depth == o.depth && tau == o.tau && lam == o.lam && p0 == o.p0 &&
               p1 == o.p1 && p2 == o.p2 && p3 == o.p3 && p4 == o.p4 && p5 == o.p5 && p6 == o.p6 && p7 == o.p7;
    }
};

struct LoopGraph {
    GraphKey key;
    cudaGraphExec_t exec;
    int n_kernels;
};

}  // namespace

// ---------------------------------------------------------------------------------
// the handle
// ---------------------------------------------------------------------------------
struct alodlm {
    alodlm_cfg cfg;
    cudaStream_t stream = nullptr;
    int device = 0;
    std::string err;
    std::vector<void *> allocs;
    size_t alloc_bytes = 0;

    // model
    int H = 0, nq = 0, nkv = 0, hd = 0, I = 0, V = 0, L = 0, n_qkv = 0;
    bf16 *embed = nullptr, *lm_head = nullptr;
    float *final_norm = nullptr, *exit_w = nullptr;
    float exit_b = 0.f;
    std::vector<LayerDev> layers;
    CUtensorMap tm_lm;

    // depth-aware KV arena: [slot][b][kvh][pos][hd]
    bf16 *kv_k = nullptr, *kv_v = nullptr;
    int n_slots = 0, pos_stride = 0;
    long long head_stride = 0, seq_stride = 0, slot_elems = 0;
    float2 *rope = nullptr;
    CUtensorMap tm_q, tm_kv_k, tm_kv_v;

    // prefill state
    int B = 0, P = 0, last_N = 0;
    bool prefilled = false;
    int depth_built = 0;  // Core depths 1..depth_built are materialised for every cached position
    int *exit_dev = nullptr;
    int *app_exit = nullptr;  // exit depths of the positions being appended [max_batch * max_block]
    // depth-on-demand prefill: the compacted rows of one depth (row tables rows_cap, slot tables max_batch)
    int *pf_row_seq = nullptr, *pf_row_u = nullptr, *pf_row_t = nullptr, *pf_gather = nullptr;
    int *pf_seq_off = nullptr, *pf_seq_cnt = nullptr;
    int *iota = nullptr;

    // activation scratch (rows_cap rows)
    int rows_cap = 0, step_rows_cap = 0;
    float *hbuf[2] = {nullptr, nullptr}, *hc = nullptr, *hexit = nullptr, *qkv = nullptr;
    bf16 *xn = nullptr, *qb = nullptr, *attn_out = nullptr, *act = nullptr;
    // folded RMSNorm: per-row partial sums of squares [rows_cap][ss_cap] (ss_cap = H / 16 rounded
    // up), and which layer's first norm the last residual add already prepared: layer fold_layer
    // over the M = fold_M rows of residual stream fold_x, with fold_n partials per row (-1: none)
    float *ss = nullptr;
    int ss_cap = 0, fold_layer = -1, fold_M = 0, fold_n = 0;
    const float *fold_x = nullptr;
    int norm_threads = 256;  // one float4 per thread per row where possible
    int num_sms = 148;

    // readout
    int R_cap = 0, n_vt = 0;
    bf16 *rb = nullptr;
    float *lam_rr = nullptr;
    float4 *part = nullptr;
    double2 *spart = nullptr;        // sampled commits: per (row, vocab tile) max of z + g and its id
    SampleParams *samp = nullptr;    // sampling state of the current step (device)
    int *ridx = nullptr, *rr_b = nullptr, *rr_i = nullptr;
    CUtensorMap tm_rb;

    // step state
    unsigned char *U = nullptr;
    float *a = nullptr, *cur_H = nullptr;
    int *cur_y = nullptr, *cont = nullptr, *ncommit = nullptr;
    int *seq_of[2] = {nullptr, nullptr}, *old_slot = nullptr;
    int *counts = nullptr, *counts_host = nullptr, *d_err = nullptr;

    // block decoding: two token buffers (a step's output is the next step's input), the
    // per-step outputs at fixed addresses (so the loop graphs are reused), the "masks left" flag
    int *dec_tok[2] = {nullptr, nullptr}, *dec_ex = nullptr, *dec_loops = nullptr, *dec_rows = nullptr;
    int *dec_left = nullptr, *dec_left_host = nullptr;
    float *dec_tr = nullptr;

    // debug copies [K][maxB][maxN][H]
    float *dbg[4] = {nullptr, nullptr, nullptr, nullptr};

    // activation tensor maps by (pointer, inner, rows, box rows)
    std::map<std::tuple<const void *, int, int, int>, CUtensorMap> tmcache;


    // CUDA graphs of the loop body
    bool use_graphs = true;
    std::vector<LoopGraph> graphs;

    // launch accounting
    int launches = 0;
    bool timing = false;
    std::vector<cudaEvent_t> ev_pool;
    size_t ev_next = 0;
    std::vector<TimedLaunch> timed;
    double cls_bytes[ALODLM_N_KCLASS] = {0}, cls_flops[ALODLM_N_KCLASS] = {0};
    int cls_launches[ALODLM_N_KCLASS] = {0};
    cudaEvent_t pending_e0 = nullptr;
};

namespace {

int fail(alodlm *h, int code, const std::string &msg) {
    if (h)
        h->err = msg;
    else {
        std::lock_guard<std::mutex> lk(g_err_mu);
        g_create_err = msg;
    }
    return code;
}

int cuda_fail(alodlm *h, cudaError_t e, const char *what) {
    return fail(h, ALODLM_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

void clear_graphs(alodlm *h) {
    for (auto &g : h->graphs) cudaGraphExecDestroy(g.exec);
    h->graphs.clear();
}

template <typename T>
int dalloc(alodlm *h, T **p, size_t count) {
    const size_t bytes = std::max<size_t>(count * sizeof(T), 256);
    if (h->cfg.mem_limit_bytes && h->alloc_bytes + bytes > h->cfg.mem_limit_bytes)
        return fail(h, ALODLM_ENOMEM, "allocation would pass cfg.mem_limit_bytes");
    void *q = nullptr;
    cudaError_t e = cudaMalloc(&q, bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(h, ALODLM_ENOMEM, std::string("cudaMalloc: ") + cudaGetErrorString(e));
    }
    h->allocs.push_back(q);
    h->alloc_bytes += bytes;
    *p = static_cast<T *>(q);
    return ALODLM_OK;
}

// launch bookkeeping: count, optional CUDA-event timing per kernel class, algorithmic work
void kbegin(alodlm *h) {
    if (!h->timing) return;
    if (h->ev_next + 2 > h->ev_pool.size()) {
        for (int i = 0; i < 64; ++i) {
            cudaEvent_t e;
            cudaEventCreate(&e);
            h->ev_pool.push_back(e);
        }
    }
    h->pending_e0 = h->ev_pool[h->ev_next++];
    cudaEventRecord(h->pending_e0, h->stream);
}
void kend(alodlm *h, int cls, double bytes, double flops) {
    h->launches++;
    h->cls_bytes[cls] += bytes;
    h->cls_flops[cls] += flops;
    h->cls_launches[cls]++;
    if (!h->timing) return;
    cudaEvent_t e1 = h->ev_pool[h->ev_next++];
    cudaEventRecord(e1, h->stream);
    h->timed.push_back({cls, h->pending_e0, e1});
}
void reset_stats(alodlm *h) {
    h->launches = 0;
    h->ev_next = 0;
    h->timed.clear();
    for (int c = 0; c < ALODLM_N_KCLASS; ++c) {
        h->cls_bytes[c] = h->cls_flops[c] = 0;
        h->cls_launches[c] = 0;
    }
}

#define LAUNCH(cls, bytes, flops, ...)   \
    do {                                 \
        kbegin(h);                       \
        __VA_ARGS__;                     \
        kend(h, cls, (bytes), (flops));  \
    } while (0)

const CUtensorMap *act_map(alodlm *h, const void *ptr, int inner, int rows, int box_rows) {
    auto key = std::make_tuple(ptr, inner, rows, box_rows);
    auto it = h->tmcache.find(key);
    if (it != h->tmcache.end()) return &it->second;
    CUtensorMap m;
    if (!make_tmap(&m, ptr, inner, rows, box_rows)) return nullptr;
    return &(h->tmcache[key] = m);
}

// C = act[M, K] x W[Nw, K]^T with a fused epilogue (tiled weights on the MMA's M side)
int linear(alodlm *h, const CUtensorMap &tmW, int Nw, const bf16 *actp, int M, int K, int epi, float *out, int ldo,
           bf16 *act_out, int ld_act, const Fold &fold = Fold{}, int *ss_group = nullptr) {
    const double bytes = 2.0 * Nw * K + 2.0 * M * K +
                         (epi == gemm::EPI_ADD ? 8.0 : (epi == gemm::EPI_SWIGLU ? 1.0 : 4.0)) * M * Nw;
    const double flops = 2.0 * M * Nw * K;
    const GemmEnv env{nullptr, 0, nullptr, 0, h->d_err, h->stream, h->num_sms};
    auto map_for_bn = [&](int bn) { return act_map(h, actp, K, h->rows_cap, bn); };
    int n = 0;
    bool per_tile = false;
    kbegin(h);
    n = run_gemm(env, tmW, Nw, map_for_bn, M, K, epi, out, ldo, act_out, ld_act, 1, fold, ss_group, &per_tile);
    kend(h, per_tile ? KC_GEMM_TILE : KC_GEMM, bytes, flops);
    if (n < 0) return fail(h, ALODLM_ECUDA, "cuTensorMapEncodeTiled failed (activation)");
    h->launches += n - 1;
    return ALODLM_OK;
}

// Work partition of one attention launch: RP packed query rows per (sequence, KV head), n_seq
// sequences, keys [0, kv_len).  pq_ok: the two-tile kernel may serve this launch (head_dim 128,
// unmasked rows without row tables); cap16: 16-CTA clusters fit for the one-tile grid.
struct AttnPlan {
    int qtiles;          // 128-row query tiles per (sequence, KV head)
    int two_tile;        // 1: the two-tile kernel, ceil(qtiles / 2) CTAs per (sequence, KV head)
    int splits;          // key splits per query tile (one cluster); a power of two
    int keys_per_split;  // a multiple of the 128-key tile
    int last_to_end;     // the last split also takes the keys past splits * keys_per_split
};

AttnPlan plan_attention(int RP, int nkv, int n_seq, int kv_len, int causal, int num_sms, int pq_ok, int cap16) {
    AttnPlan a{};
    a.qtiles = cdiv(RP, attn_tc::BQ);
    const int base = a.qtiles * nkv * n_seq;
    const int ktiles = cdiv(kv_len, attn_tc::BKV);
    // two query tiles per CTA (K/V loaded once for both, softmax warpgroups in turn) where a
    // (sequence, KV head) has two and the pairs still cover half the SMs without a key split
    const int qpairs = cdiv(a.qtiles, 2);
    if (pq_ok && !causal && ALODLM_ATTN_PQ && a.qtiles >= 2 && 2 * qpairs * nkv * n_seq >= num_sms) {
        a.two_tile = 1;
        a.splits = 1;
        a.keys_per_split = ktiles * attn_tc::BKV;
        return a;
    }
    // splits of a query tile form one cluster (a power of two so that they share the 128
    // rows evenly; 8 CTAs, or 16 where that many 16-CTA clusters fit at once): enough CTAs
    // to cover the SMs, rounded up to the next power of two while the grid still fits in
    // one wave, so that a latency-bound launch walks one key tile per CTA
    // causal rows: no key split (each query tile walks keys [0, its last position]; a
    // prefill's query tiles alone fill the SMs)
    const int cap = cap16 ? 16 : 8;
    const int want = causal ? 1 : std::max(1, std::min(std::min(ktiles, cdiv(num_sms, base)), cap));
    int splits = 1;
    while (splits < want) splits <<= 1;
    if (splits > cap || (splits > 1 && (long long)splits * base > num_sms)) splits >>= 1;
    int kps = cdiv(ktiles, splits);  // trailing ranks may get no keys (empty partials)
    // a remainder shorter than a key tile rides on the last rank when that saves every other
    // rank a tile: e.g. 8 full tiles + 32 keys over 8 ranks -> one tile each, the last two
    const int full = kv_len / attn_tc::BKV, kps_full = std::max(1, cdiv(full, splits));
    if (splits > 1 && kps_full < kps && (long long)splits * kps_full * attn_tc::BKV >= (long long)full * attn_tc::BKV &&
        kv_len - (long long)splits * kps_full * attn_tc::BKV < attn_tc::BKV) {
        kps = kps_full;
        a.last_to_end = 1;
    }
    a.splits = splits;
    a.keys_per_split = kps * attn_tc::BKV;
    return a;
}

// attention of M rows (n_seq sequences x rows_per_seq) against slot `slot`, keys [0, kv_len)
int attention(alodlm *h, int slot, int M, const RowMap &map, int n_seq, int kv_len, int causal) {
    attn_tc::Params p{};
    // keys before the rows' own: the step's cached prefix, or the positions an append extends
    p.static_keys = std::max(0, kv_len - map.rows_per_seq);
    p.causal = causal;
    p.pos0 = map.pos0;
    p.row_t = map.row_t;
    p.seq_off = map.seq_off;
    p.seq_cnt = map.seq_cnt;
    p.G = h->nq / h->nkv;
    p.RP = p.G * map.rows_per_seq;
    p.nkv = h->nkv;
    p.nq = h->nq;
    p.Tq = map.rows_per_seq;
    p.kv_len = kv_len;
    p.slot = slot;
    p.max_batch = h->cfg.max_batch;
    p.pos_stride = h->pos_stride;
    p.seq_of = map.seq_of;
    p.out = h->attn_out;
    p.out_ld = h->nq * h->hd;
    p.m_rows = M;
    p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)h->hd));
    p.err = h->d_err;
    const int qtiles = cdiv(p.RP, attn_tc::BQ);
    const int base = qtiles * h->nkv * n_seq;
    const double bytes = 4.0 * n_seq * h->nkv * (double)kv_len * h->hd + 4.0 * M * h->nq * h->hd;
    const double flops = 4.0 * M * h->nq * (double)kv_len * h->hd * (causal ? 0.5 : 1.0);
    const AttnPlan plan =
        plan_attention(p.RP, h->nkv, n_seq, kv_len, causal, h->num_sms, h->hd == attn_tc::HD && !map.seq_cnt,
                       h->hd == 128 && ALODLM_ATTN_CLUSTER16 && attn_clusters16() >= base);
    p.n_splits = plan.splits;
    p.keys_per_split = plan.keys_per_split;
    p.last_to_end = plan.last_to_end;
    if (plan.two_tile) {
        LAUNCH(KC_ATTN, bytes, flops,
               klaunch(attn_pq::attn_pq_kernel, dim3(cdiv(qtiles, 2), h->nkv, n_seq), attn_pq::THREADS,
                       attn_pq::SMEM, h->stream, h->tm_q, h->tm_kv_k, h->tm_kv_v, p));
        return ALODLM_OK;
    }
    const int splits = plan.splits;
    // one instance per head_dim (one or two 64-wide halves per head vector)
    auto *const kern = h->hd == 128 ? attn_tc::attn_tc_kernel<128> : attn_tc::attn_tc_kernel<64>;
    const size_t smem = h->hd == 128 ? attn_tc::smem_bytes<128>() : attn_tc::smem_bytes<64>();
    if (splits > 1) {
        // cluster along y: the `splits` consecutive y indices of one kv head
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(qtiles, h->nkv * splits, n_seq);
        cfg.blockDim = dim3(192);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = h->stream;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 1;
        attr[0].val.clusterDim.y = splits;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = ALODLM_PDL ? 2 : 1;
        LAUNCH(KC_ATTN, bytes, flops,
               cudaLaunchKernelEx(&cfg, kern, h->tm_q, h->tm_kv_k, h->tm_kv_v, p));
    } else {
        LAUNCH(KC_ATTN, bytes, flops,
               klaunch(kern, dim3(qtiles, h->nkv, n_seq), 192, smem, h->stream, h->tm_q, h->tm_kv_k, h->tm_kv_v,
                       p));
    }
    return ALODLM_OK;
}

int slot_prelude(const alodlm *h, int l) { return l; }
int slot_core(const alodlm *h, int c, int d) { return h->cfg.n_prelude + (d - 1) * h->cfg.n_core + c; }
int slot_coda(const alodlm *h, int j) { return h->cfg.n_prelude + h->cfg.k_max * h->cfg.n_core + j; }

// Depth fallback of one Core layer at depth `depth` during a prefill or an append: rows of
// sequences b0 .. b0+nb-1, positions pos0 .. pos0+n-1 with exit depths exit[b * n + t]
struct Fallback {
    const int *exit;
    int n, pos0, b0, nb, depth, src_slot;
};

// xn = RMSNorm(x) * g (bf16) over M rows of the hidden size: one block per row for few rows
// (the whole GPU works on each), one warp per row once the rows alone fill it
int rmsnorm(alodlm *h, const float *x, const float *g, bf16 *xn, int M) {
    const int H = h->H;
    if (M >= ALODLM_NORM_WARP_ROWS && H % 128 == 0 && H <= 128 * 32)
        LAUNCH(KC_NORM, 6.0 * M * H, 0.0,
               (klaunch(k::rmsnorm_row_regs_kernel<32>, cdiv(M, 4), 128, 0, h->stream, x, g, xn, M, H,
                        h->cfg.rms_eps)));
    else if (M >= 256 && H % 128 == 0)
        LAUNCH(KC_NORM, 6.0 * M * H, 0.0,
               (klaunch(k::rmsnorm_warp_kernel, cdiv(M, 8), 256, 0, h->stream, x, g, xn, M, H, h->cfg.rms_eps)));
    else
        LAUNCH(KC_NORM, 6.0 * M * H, 0.0,
               (klaunch(k::rmsnorm_kernel, M, h->norm_threads, 0, h->stream, x, g, xn, H, h->cfg.rms_eps)));
    return ALODLM_OK;
}

// one pre-norm Qwen3 decoder layer over M rows, residual stream `x` updated in place.  With the
// RMSNorm folded (ALODLM_FOLD_NORM), the two residual adds write the next projection's operand
// bf16(x * g) and per-row partial sums of x^2, and the Q/K/V and gate/up projections scale their
// rows by 1 / rms: no separate norm kernel runs except where the layer's input did not come from
// the previous layer's residual add on the same rows (the first layer of a chain).
int run_layer(alodlm *h, int li, int slot, int M, const RowMap &map, int n_seq, int kv_len, int causal, float *x,
              const Fallback *fb) {
    const LayerDev &Lw = h->layers[li];
    const int H = h->H, qd = h->nq * h->hd;
    const bool fold = ALODLM_FOLD_NORM != 0;
    int rc;
    auto consumer = [&](int n_parts) {
        Fold f;
        f.ss_in = h->ss;
        f.ss_ld = h->ss_cap;
        f.ss_n = n_parts;
        f.norm_h = (float)H;
        f.eps = h->cfg.rms_eps;
        return f;
    };
    auto producer = [&](const float *g_next) {
        Fold f;
        f.xg = h->xn;
        f.g_next = g_next;
        f.ss = h->ss;
        f.ss_ld = h->ss_cap;
        return f;
    };
    Fold f_qkv;
    if (fold && h->fold_layer == li && h->fold_x == x && h->fold_M == M)
        f_qkv = consumer(h->fold_n);
    else if ((rc = rmsnorm(h, x, Lw.attn_norm, h->xn, M)))
        return rc;
    h->fold_layer = -1;
    bf16 *kc = h->kv_k + (long long)slot * h->slot_elems, *vc = h->kv_v + (long long)slot * h->slot_elems;
    if ((rc = linear(h, Lw.tm_qkv, h->n_qkv, h->xn, M, H, gemm::EPI_F32, h->qkv, h->n_qkv, nullptr, 0, f_qkv)))
        return rc;
    const int n_heads = h->nq + 2 * h->nkv;
    if (h->hd == 128 && n_heads <= 64) {
        LAUNCH(KC_QKV, 6.0 * M * h->n_qkv, 0.0,
               (klaunch(k::qkv_post128_kernel, M, 256, 0, h->stream, h->qkv, h->nq, h->nkv, cdiv(n_heads, 8),
                        Lw.q_norm, Lw.k_norm, h->cfg.qk_norm, h->cfg.rms_eps, h->rope, map, h->qb, kc, vc,
                        h->seq_stride, h->head_stride)));
    } else {
        LAUNCH(KC_QKV, 6.0 * M * h->n_qkv, 0.0,
               (klaunch(k::qkv_post_kernel, dim3(M, cdiv(n_heads, 8)), 256, 0, h->stream, h->qkv, h->nq, h->nkv,
                        h->hd, Lw.q_norm, Lw.k_norm, h->cfg.qk_norm, h->cfg.rms_eps, h->rope, map, h->qb, kc, vc,
                        h->seq_stride, h->head_stride)));
    }
    if (fb) {
        const long long so = (long long)fb->src_slot * h->slot_elems;
        LAUNCH(KC_OTHER, 8.0 * fb->nb * h->nkv * fb->n * h->hd, 0.0,
               (klaunch(k::kv_fallback_kernel, dim3(fb->nb, h->nkv), 256, 0, h->stream, fb->exit, fb->n, fb->pos0,
                        fb->b0, fb->depth, h->kv_k + so, h->kv_v + so, kc, vc, h->seq_stride, h->head_stride,
                        h->hd)));
    }
    if ((rc = attention(h, slot, M, map, n_seq, kv_len, causal))) return rc;
    int group = 0;
    if ((rc = linear(h, Lw.tm_o, H, h->attn_out, M, qd, gemm::EPI_ADD, x, H, nullptr, 0,
                     fold ? producer(Lw.mlp_norm) : Fold{}, &group)))
        return rc;
    Fold f_gu;
    if (fold)
        f_gu = consumer(cdiv(H, group));
    else if ((rc = rmsnorm(h, x, Lw.mlp_norm, h->xn, M)))
        return rc;
    if ((rc = linear(h, Lw.tm_gu, 2 * h->I, h->xn, M, H, gemm::EPI_SWIGLU, nullptr, 0, h->act, h->I, f_gu)))
        return rc;
    // the next layer in the stack takes its first norm from this residual add (the callers
    // invalidate it wherever something else runs in between)
    const bool chain = fold && li + 1 < h->L;
    if ((rc = linear(h, Lw.tm_d, H, h->act, M, h->I, gemm::EPI_ADD, x, H, nullptr, 0,
                     chain ? producer(h->layers[li + 1].attn_norm) : Fold{}, &group)))
        return rc;
    if (chain) {
        h->fold_layer = li + 1;
        h->fold_x = x;
        h->fold_M = M;
        h->fold_n = cdiv(H, group);
    }
    return ALODLM_OK;
}

// the depth fallback of one Core slot on its own (a depth that no position runs)
void launch_fallback(alodlm *h, int slot, const Fallback &fb) {
    const long long so = (long long)fb.src_slot * h->slot_elems;
    bf16 *kc = h->kv_k + (long long)slot * h->slot_elems, *vc = h->kv_v + (long long)slot * h->slot_elems;
    LAUNCH(KC_OTHER, 8.0 * fb.nb * h->nkv * fb.n * h->hd, 0.0,
           (klaunch(k::kv_fallback_kernel, dim3(fb.nb, h->nkv), 256, 0, h->stream, fb.exit, fb.n, fb.pos0, fb.b0,
                    fb.depth, (const bf16 *)(h->kv_k + so), (const bf16 *)(h->kv_v + so), kc, vc, h->seq_stride,
                    h->head_stride, h->hd)));
}

int check_launch(alodlm *h, const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(h, e, what);
    return ALODLM_OK;
}

int validate_cfg(const alodlm_cfg *c, std::string &why) {
    auto bad = [&](const char *m) {
        why = m;
        return ALODLM_EINVAL;
    };
    if (c->hidden < 64 || c->hidden % 16) return bad("hidden must be >= 64 and a multiple of 16");
    if (c->head_dim != 64 && c->head_dim != 128) return bad("head_dim must be 64 or 128");
    if (c->n_q_heads < 1 || c->n_kv_heads < 1 || c->n_q_heads % c->n_kv_heads)
        return bad("n_q_heads must be a positive multiple of n_kv_heads");
    if (c->inter < 16 || c->inter % 16) return bad("inter must be a positive multiple of 16");
    if (c->vocab < 2) return bad("vocab must be >= 2");
    if (c->n_core < 1 || c->n_prelude < 0 || c->n_coda < 0) return bad("layer counts out of range");
    if (c->k_max < 1 || c->k_max > 64) return bad("k_max must be in 1..64");
    if (c->max_batch < 1 || c->max_batch > 1024) return bad("max_batch must be in 1..1024");
    if (c->max_block < 1 || c->max_block > 1024) return bad("max_block must be in 1..1024");
    if ((long long)c->max_batch * c->max_block > 65536) return bad("max_batch * max_block must be <= 65536");
    if (c->max_prefix < 1) return bad("max_prefix must be >= 1");
    if (c->mask_id < 0 || c->mask_id >= c->vocab) return bad("mask_id out of range");
    if (!(c->rms_eps > 0.f) || !(c->rope_base > 1.f)) return bad("rms_eps/rope_base out of range");
    return ALODLM_OK;
}

}  // namespace

// ---------------------------------------------------------------------------------
// ABI
// ---------------------------------------------------------------------------------
extern "C" {

const char *alodlm_kernel_class_name(int k) {
    return (k >= 0 && k < ALODLM_N_KCLASS) ? kclass_names[k] : "";
}

const char *alodlm_last_error(const alodlm_t *h) {
    if (h) return h->err.c_str();
    std::lock_guard<std::mutex> lk(g_err_mu);
    return g_create_err.c_str();
}

void alodlm_destroy(alodlm_t *h) {
    if (!h) return;
    cudaStreamSynchronize(h->stream);
    clear_graphs(h);
    for (void *p : h->allocs) cudaFree(p);
    for (auto e : h->ev_pool) cudaEventDestroy(e);
    if (h->counts_host) cudaFreeHost(h->counts_host);
    if (h->dec_left_host) cudaFreeHost(h->dec_left_host);
    delete h;
}

int alodlm_create(const alodlm_cfg *cfg, const alodlm_weights *w, void *stream, alodlm_t **out) {
    if (out) *out = nullptr;
    if (!cfg || !w || !out || !w->layers || !w->embed || !w->lm_head || !w->final_norm || !w->exit_w)
        return fail(nullptr, ALODLM_EINVAL, "null argument");
    std::string why;
    if (validate_cfg(cfg, why)) return fail(nullptr, ALODLM_EINVAL, why);
    if (w->matrix_dtype != ALODLM_DTYPE_BF16 && w->matrix_dtype != ALODLM_DTYPE_F32)
        return fail(nullptr, ALODLM_EINVAL, "matrix_dtype must be ALODLM_DTYPE_BF16 or ALODLM_DTYPE_F32");
    const int L = cfg->n_prelude + cfg->n_core + cfg->n_coda;
    for (int l = 0; l < L; ++l) {
        const alodlm_layer_w &lw = w->layers[l];
        if (!lw.attn_norm || !lw.q || !lw.k || !lw.v || !lw.o || !lw.mlp_norm || !lw.gate || !lw.up || !lw.down ||
            (cfg->qk_norm && (!lw.q_norm || !lw.k_norm)))
            return fail(nullptr, ALODLM_EINVAL, "null layer weight pointer");
    }
    if (!get_encode_fn()) return fail(nullptr, ALODLM_ECUDA, "cuTensorMapEncodeTiled unavailable");
    if (!init_kernel_attrs()) return fail(nullptr, ALODLM_ECUDA, "cudaFuncSetAttribute failed");

    alodlm *h = new alodlm();
    h->cfg = *cfg;
    h->stream = static_cast<cudaStream_t>(stream);
    cudaGetDevice(&h->device);
    cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device);
    h->norm_threads = std::max(32, std::min(1024, round_up(cfg->hidden / 4, 32)));

    h->H = cfg->hidden;
    h->nq = cfg->n_q_heads;
    h->nkv = cfg->n_kv_heads;
    h->hd = cfg->head_dim;
    h->I = cfg->inter;
    h->V = cfg->vocab;
    h->L = L;
    h->n_qkv = (h->nq + 2 * h->nkv) * h->hd;
    const int H = h->H, qd = h->nq * h->hd;
    const int f32 = w->matrix_dtype == ALODLM_DTYPE_F32;
    int rc = ALODLM_OK;
    auto cleanup = [&](int code) {
        std::string msg = h->err;
        alodlm_destroy(h);
        fail(nullptr, code, msg);
        return code;
    };

    // ---- weights: pack to bf16 (rows padded with zeros), then store every matrix the GEMMs
    // stream in the tiled layout (each [tile rows x 64] tile contiguous) ----
    const size_t stage_elems =
        std::max({(size_t)round_up(h->V, 256) * H, (size_t)round_up(h->n_qkv, 128) * H, (size_t)round_up(H, 128) * qd,
                  (size_t)round_up(2 * h->I, 128) * H, (size_t)round_up(H, 128) * h->I});
    bf16 *stage = nullptr;
    if (cudaMalloc(&stage, stage_elems * 2) != cudaSuccess) {
        cudaGetLastError();
        h->err = "cudaMalloc failed (weight staging)";
        return cleanup(ALODLM_ENOMEM);
    }
    struct StageGuard {
        bf16 *p;
        ~StageGuard() { cudaFree(p); }
    } stage_guard{stage};
    auto stage_rows = [&](int rows_pad, int cols, const void *src, int src_rows) -> int {
        cudaMemsetAsync(stage, 0, (size_t)rows_pad * cols * 2, h->stream);
        k::pack_rows_kernel<<<src_rows, 256, 0, h->stream>>>(src, f32, cols, nullptr, src_rows, cols, stage, cols);
        return check_launch(h, "pack_rows_kernel");
    };
    // stage (rows_pad x cols, row-major) -> tiled copy in handle memory + its tensor map
    auto tile_from_stage = [&](bf16 **dst, CUtensorMap *map, int rows_pad, int cols, int RT) -> int {
        const int KT = cdiv(cols, 64), n_rt = rows_pad / RT;
        int r;
        if ((r = dalloc(h, dst, (size_t)n_rt * KT * RT * 64))) return r;
        k::tile_matrix_kernel<<<n_rt * KT, 256, 0, h->stream>>>(stage, rows_pad, cols, RT, KT, *dst);
        if ((r = check_launch(h, "tile_matrix_kernel"))) return r;
        if (!make_tmap(map, *dst, 64, n_rt * KT * RT, RT)) return fail(h, ALODLM_ECUDA, "cuTensorMapEncodeTiled failed");
        return ALODLM_OK;
    };
    auto copy_vec = [&](float **dst, const void *src, int n) -> int {
        int r;
        if ((r = dalloc(h, dst, n))) return r;
        cudaMemcpyAsync(*dst, src, n * sizeof(float), cudaMemcpyDeviceToDevice, h->stream);
        return ALODLM_OK;
    };
    // the embedding is gathered by rows: plain layout
    if ((rc = dalloc(h, &h->embed, (size_t)h->V * H))) return cleanup(rc);
    k::pack_rows_kernel<<<h->V, 256, 0, h->stream>>>(w->embed, f32, H, nullptr, h->V, H, h->embed, H);
    if ((rc = check_launch(h, "pack embed"))) return cleanup(rc);
    if ((rc = stage_rows(round_up(h->V, 256), H, w->lm_head, h->V)) ||
        (rc = tile_from_stage(&h->lm_head, &h->tm_lm, round_up(h->V, 256), H, 256)))
        return cleanup(rc);
    if ((rc = copy_vec(&h->final_norm, w->final_norm, H))) return cleanup(rc);
    if ((rc = copy_vec(&h->exit_w, w->exit_w, H))) return cleanup(rc);
    h->exit_b = w->exit_b;
    h->layers.resize(L);
    for (int l = 0; l < L; ++l) {
        const alodlm_layer_w &lw = w->layers[l];
        LayerDev &d = h->layers[l];
        // fused QKV: rows [q; k; v]
        cudaMemsetAsync(stage, 0, (size_t)round_up(h->n_qkv, 128) * H * 2, h->stream);
        k::pack_rows_kernel<<<qd, 256, 0, h->stream>>>(lw.q, f32, H, nullptr, qd, H, stage, H);
        k::pack_rows_kernel<<<h->nkv * h->hd, 256, 0, h->stream>>>(lw.k, f32, H, nullptr, h->nkv * h->hd, H,
                                                                   stage + (size_t)qd * H, H);
        k::pack_rows_kernel<<<h->nkv * h->hd, 256, 0, h->stream>>>(
            lw.v, f32, H, nullptr, h->nkv * h->hd, H, stage + (size_t)(qd + h->nkv * h->hd) * H, H);
        if ((rc = check_launch(h, "pack qkv"))) return cleanup(rc);
        if ((rc = tile_from_stage(&d.wqkv, &d.tm_qkv, round_up(h->n_qkv, 128), H, 128))) return cleanup(rc);
        if ((rc = stage_rows(round_up(H, 128), qd, lw.o, H)) ||
            (rc = tile_from_stage(&d.wo, &d.tm_o, round_up(H, 128), qd, 128)))
            return cleanup(rc);
        cudaMemsetAsync(stage, 0, (size_t)round_up(2 * h->I, 128) * H * 2, h->stream);
        k::pack_gate_up_kernel<<<2 * h->I, 256, 0, h->stream>>>(lw.gate, lw.up, f32, h->I, H, stage);
        if ((rc = check_launch(h, "pack gate/up"))) return cleanup(rc);
        if ((rc = tile_from_stage(&d.wgu, &d.tm_gu, round_up(2 * h->I, 128), H, 128))) return cleanup(rc);
        if ((rc = stage_rows(round_up(H, 128), h->I, lw.down, H)) ||
            (rc = tile_from_stage(&d.wd, &d.tm_d, round_up(H, 128), h->I, 128)))
            return cleanup(rc);
        if ((rc = copy_vec(&d.attn_norm, lw.attn_norm, H))) return cleanup(rc);
        if ((rc = copy_vec(&d.mlp_norm, lw.mlp_norm, H))) return cleanup(rc);
        if (cfg->qk_norm) {
            if ((rc = copy_vec(&d.q_norm, lw.q_norm, h->hd))) return cleanup(rc);
            if ((rc = copy_vec(&d.k_norm, lw.k_norm, h->hd))) return cleanup(rc);
        }
    }
    if (cudaStreamSynchronize(h->stream) != cudaSuccess) {
        h->err = "weight packing failed";
        return cleanup(ALODLM_ECUDA);
    }

    // ---- depth-aware KV arena ----
    h->n_slots = cfg->n_prelude + cfg->k_max * cfg->n_core + cfg->n_coda;
    h->pos_stride = cfg->max_prefix + cfg->max_block;
    h->head_stride = (long long)h->pos_stride * h->hd;
    h->seq_stride = h->head_stride * h->nkv;
    h->slot_elems = h->seq_stride * cfg->max_batch;
    if ((rc = dalloc(h, &h->kv_k, (size_t)h->slot_elems * h->n_slots))) return cleanup(rc);
    if ((rc = dalloc(h, &h->kv_v, (size_t)h->slot_elems * h->n_slots))) return cleanup(rc);
    if ((rc = dalloc(h, &h->rope, (size_t)h->pos_stride * (h->hd / 2)))) return cleanup(rc);
    {
        const long long n = (long long)h->pos_stride * (h->hd / 2);
        k::rope_table_kernel<<<(unsigned)((n + 255) / 256), 256, 0, h->stream>>>(h->rope, h->pos_stride, h->hd / 2,
                                                                                (double)cfg->rope_base);
        if ((rc = check_launch(h, "rope_table_kernel"))) return cleanup(rc);
    }

    // ---- scratch ----
    const int g_max = std::max(1, std::min(cfg->max_batch, PREFILL_ROWS / std::max(1, cfg->max_prefix)));
    h->step_rows_cap = cfg->max_batch * cfg->max_block;
    h->rows_cap = round_up(std::max(h->step_rows_cap, g_max * cfg->max_prefix), 256);
    const size_t R = h->rows_cap;
    if ((rc = dalloc(h, &h->hbuf[0], R * H)) || (rc = dalloc(h, &h->hbuf[1], R * H)) ||
        (rc = dalloc(h, &h->hc, R * H)) || (rc = dalloc(h, &h->hexit, R * H)) ||
        (rc = dalloc(h, &h->qkv, R * h->n_qkv)) || (rc = dalloc(h, &h->xn, R * H)) ||
        (rc = dalloc(h, &h->qb, R * qd)) || (rc = dalloc(h, &h->attn_out, R * qd)) ||
        (rc = dalloc(h, &h->act, R * h->I)))
        return cleanup(rc);
    h->ss_cap = cdiv(H, 16);
    if ((rc = dalloc(h, &h->ss, R * h->ss_cap))) return cleanup(rc);
    // zero the activation buffers once so rows past the live ones never hold NaN patterns
    cudaMemsetAsync(h->xn, 0, R * H * 2, h->stream);
    cudaMemsetAsync(h->attn_out, 0, R * qd * 2, h->stream);
    cudaMemsetAsync(h->act, 0, R * h->I * 2, h->stream);

    // never-written arena positions are read (and masked) by 128-key tiles: keep them finite
    cudaMemsetAsync(h->kv_k, 0, (size_t)h->slot_elems * h->n_slots * 2, h->stream);
    cudaMemsetAsync(h->kv_v, 0, (size_t)h->slot_elems * h->n_slots * 2, h->stream);
    {
        // the attention's tensor maps address head vectors by 32-bit row coordinates
        const long long arena_rows = (long long)h->n_slots * cfg->max_batch * h->nkv * h->pos_stride;
        if (arena_rows + 256 >= (1ll << 31) || (long long)R * h->nq >= (1ll << 31)) {
            h->err = "KV arena or query rows beyond 2^31 head vectors";
            return cleanup(ALODLM_EINVAL);
        }
        if (!make_tmap(&h->tm_q, h->qb, h->hd, (int)(R * h->nq), attn_tc::BQ) ||
            !make_tmap(&h->tm_kv_k, h->kv_k, h->hd, (int)arena_rows, attn_tc::BKV) ||
            !make_tmap(&h->tm_kv_v, h->kv_v, h->hd, (int)arena_rows, attn_tc::BKV)) {
            h->err = "cuTensorMapEncodeTiled failed (attention)";
            return cleanup(ALODLM_ECUDA);
        }
    }

    h->R_cap = round_up(h->step_rows_cap, 128);
    h->n_vt = cdiv(h->V, 256);
    if ((rc = dalloc(h, &h->rb, (size_t)h->R_cap * H)) || (rc = dalloc(h, &h->lam_rr, h->R_cap)) ||
        (rc = dalloc(h, &h->part, (size_t)h->R_cap * h->n_vt)) || (rc = dalloc(h, &h->ridx, h->step_rows_cap)) ||
        (rc = dalloc(h, &h->spart, (size_t)h->R_cap * h->n_vt)) || (rc = dalloc(h, &h->samp, 1)) ||
        (rc = dalloc(h, &h->rr_b, h->R_cap)) || (rc = dalloc(h, &h->rr_i, h->R_cap)))
        return cleanup(rc);
    cudaMemsetAsync(h->rb, 0, (size_t)h->R_cap * H * 2, h->stream);
    if (!make_tmap(&h->tm_rb, h->rb, H, h->R_cap, 128)) {
        h->err = "cuTensorMapEncodeTiled failed (readout rows)";
        return cleanup(ALODLM_ECUDA);
    }
    const size_t BN_ = (size_t)cfg->max_batch * cfg->max_block;
    if ((rc = dalloc(h, &h->U, BN_)) || (rc = dalloc(h, &h->a, BN_)) || (rc = dalloc(h, &h->cur_H, BN_)) ||
        (rc = dalloc(h, &h->cur_y, BN_)) || (rc = dalloc(h, &h->cont, cfg->max_batch)) ||
        (rc = dalloc(h, &h->ncommit, cfg->max_batch)) || (rc = dalloc(h, &h->seq_of[0], cfg->max_batch)) ||
        (rc = dalloc(h, &h->seq_of[1], cfg->max_batch)) || (rc = dalloc(h, &h->old_slot, cfg->max_batch)) ||
        (rc = dalloc(h, &h->counts, 4)) || (rc = dalloc(h, &h->d_err, 1)) || (rc = dalloc(h, &h->iota, cfg->max_batch)) ||
        (rc = dalloc(h, &h->exit_dev, (size_t)cfg->max_batch * cfg->max_prefix)) ||
        (rc = dalloc(h, &h->app_exit, BN_)) || (rc = dalloc(h, &h->pf_row_seq, h->rows_cap)) ||
        (rc = dalloc(h, &h->pf_row_u, h->rows_cap)) || (rc = dalloc(h, &h->pf_row_t, h->rows_cap)) ||
        (rc = dalloc(h, &h->pf_gather, h->rows_cap)) || (rc = dalloc(h, &h->pf_seq_off, cfg->max_batch)) ||
        (rc = dalloc(h, &h->pf_seq_cnt, cfg->max_batch)) ||
        (rc = dalloc(h, &h->dec_tok[0], BN_)) || (rc = dalloc(h, &h->dec_tok[1], BN_)) ||
        (rc = dalloc(h, &h->dec_ex, BN_)) || (rc = dalloc(h, &h->dec_loops, cfg->max_batch)) ||
        (rc = dalloc(h, &h->dec_rows, 2 * (size_t)cfg->k_max)) || (rc = dalloc(h, &h->dec_left, 1)) ||
        (rc = dalloc(h, &h->dec_tr, 3 * (size_t)cfg->k_max * BN_)))
        return cleanup(rc);
    {
        std::vector<int> io(cfg->max_batch);
        for (int i = 0; i < cfg->max_batch; ++i) io[i] = i;
        cudaMemcpyAsync(h->iota, io.data(), io.size() * sizeof(int), cudaMemcpyHostToDevice, h->stream);
        cudaMemsetAsync(h->d_err, 0, sizeof(int), h->stream);
    }
    if (cfg->debug_dump) {
        for (int i = 0; i < 4; ++i)
            if ((rc = dalloc(h, &h->dbg[i], (size_t)cfg->k_max * BN_ * H))) return cleanup(rc);
    }
    if (cudaMallocHost(&h->counts_host, 4 * sizeof(int)) != cudaSuccess ||
        cudaMallocHost(&h->dec_left_host, sizeof(int)) != cudaSuccess) {
        h->err = "cudaMallocHost failed";
        return cleanup(ALODLM_ENOMEM);
    }
    cudaError_t e = cudaStreamSynchronize(h->stream);
    if (e != cudaSuccess) {
        cuda_fail(h, e, "create");
        return cleanup(ALODLM_ECUDA);
    }
    *out = h;
    return ALODLM_OK;
}

}  // extern "C"

namespace {

int denoise_step_impl(alodlm *h, const int32_t *block_ids, int B, int N, float tau_H, float lambda, int k_max,
                      int rule, const SampleParams &sp, const alodlm_step_out *out);

int decode_block_impl(alodlm *h, const int32_t *block_ids, int B, int N, float tau_H, float lambda, int k_max,
                      int rule, int max_steps, bool sampled, uint64_t seed, const alodlm_decode_out *out,
                      int *steps_taken) {
    const NvtxRange range("alodlm decode_block");
    if (steps_taken) *steps_taken = 0;
    if (!h || !block_ids || !out || !out->tokens || !out->commit_step || !out->commit_depth || !out->steps_run ||
        !out->loops || !out->rows)
        return fail(h, ALODLM_EINVAL, "null argument");
    if (max_steps < 1) return fail(h, ALODLM_EINVAL, "max_steps must be >= 1");
    if (!h->prefilled) return fail(h, ALODLM_ESTATE, "decode_block before prefill");
    if (B != h->B) return fail(h, ALODLM_ESTATE, "batch differs from the prefill's");
    if (N < 1 || N > h->cfg.max_block) return fail(h, ALODLM_EINVAL, "N out of range");
    if (k_max < 1 || k_max > h->cfg.k_max) return fail(h, ALODLM_EINVAL, "k_max out of range");
    const long long BN = (long long)B * N;
    const unsigned grid = (unsigned)std::min<long long>((BN + 255) / 256, 1024);
    cudaError_t ce = cudaSuccess;  // first error of the asynchronous calls
    auto ck = [&](cudaError_t e) {
        if (ce == cudaSuccess) ce = e;
    };
    ck(cudaMemsetAsync(out->commit_step, 0, BN * sizeof(int32_t), h->stream));
    ck(cudaMemsetAsync(out->commit_depth, 0, BN * sizeof(int32_t), h->stream));
    ck(cudaMemsetAsync(out->steps_run, 0, (size_t)B * sizeof(int32_t), h->stream));
    ck(cudaMemsetAsync(out->loops, 0, (size_t)max_steps * B * sizeof(int32_t), h->stream));
    ck(cudaMemsetAsync(out->rows, 0, (size_t)max_steps * 2 * k_max * sizeof(int32_t), h->stream));
    ck(cudaMemcpyAsync(out->tokens, block_ids, BN * sizeof(int32_t), cudaMemcpyDeviceToDevice, h->stream));
    // a block without masks takes no step
    ck(cudaMemsetAsync(h->dec_left, 0, sizeof(int), h->stream));
    klaunch(k::any_mask_kernel, grid, 256, 0, h->stream, (const int *)block_ids, BN, h->cfg.mask_id, h->dec_left);
    ck(cudaGetLastError());
    if (ce != cudaSuccess) return cuda_fail(h, ce, "decode_block: set-up");
    const size_t KBN = (size_t)k_max * BN;
    alodlm_step_out so{};
    so.exit_depth = h->dec_ex;
    so.entropy = h->dec_tr;
    so.halt = h->dec_tr + KBN;
    so.cum_halt = h->dec_tr + 2 * KBN;
    so.loops_run = h->dec_loops;
    so.active_rows = h->dec_rows;
    so.readout_rows = h->dec_rows + k_max;
    const int32_t *in = block_ids;
    int t = 0;
    for (;;) {
        ck(cudaMemcpyAsync(h->dec_left_host, h->dec_left, sizeof(int), cudaMemcpyDeviceToHost, h->stream));
        ck(cudaStreamSynchronize(h->stream));
        if (ce != cudaSuccess) return cuda_fail(h, ce, "decode_block: read the masks-left flag");
        if (*h->dec_left_host == 0 || t == max_steps) break;
        ++t;
        so.tokens = h->dec_tok[t & 1];
        const SampleParams sp{(unsigned long long)seed, (unsigned long long)t, sampled ? 1 : 0, 0};
        const int rc = denoise_step_impl(h, in, B, N, tau_H, lambda, k_max, rule, sp, &so);
        if (rc) return rc;
        ck(cudaMemsetAsync(h->dec_left, 0, sizeof(int), h->stream));
        klaunch(k::decode_update_kernel, grid, 256, 0, h->stream, (const int *)in, (const int *)so.tokens,
                (const int *)h->dec_ex, t, B, N, h->cfg.mask_id, out->commit_step, out->commit_depth, out->steps_run,
                h->dec_left);
        ck(cudaGetLastError());
        ck(cudaMemcpyAsync(out->loops + (size_t)(t - 1) * B, h->dec_loops, (size_t)B * sizeof(int32_t),
                           cudaMemcpyDeviceToDevice, h->stream));
        ck(cudaMemcpyAsync(out->rows + (size_t)(t - 1) * 2 * k_max, h->dec_rows, 2 * (size_t)k_max * sizeof(int32_t),
                           cudaMemcpyDeviceToDevice, h->stream));
        in = so.tokens;
    }
    if (t > 0) ck(cudaMemcpyAsync(out->tokens, in, BN * sizeof(int32_t), cudaMemcpyDeviceToDevice, h->stream));
    ck(cudaGetLastError());
    if (ce != cudaSuccess) return cuda_fail(h, ce, "decode_block");
    if (steps_taken) *steps_taken = t;
    return ALODLM_OK;
}

}  // namespace

extern "C" {

int alodlm_decode_block(alodlm_t *h, const int32_t *block_ids, int B, int N, float tau_H, float lambda, int k_max,
                        int rule, int max_steps, const alodlm_decode_out *out, int *steps_taken) {
    return decode_block_impl(h, block_ids, B, N, tau_H, lambda, k_max, rule, max_steps, false, 0, out, steps_taken);
}

int alodlm_decode_block_sampled(alodlm_t *h, const int32_t *block_ids, int B, int N, float tau_H, float lambda,
                                int k_max, int rule, int max_steps, uint64_t seed, const alodlm_decode_out *out,
                                int *steps_taken) {
    return decode_block_impl(h, block_ids, B, N, tau_H, lambda, k_max, rule, max_steps, true, seed, out, steps_taken);
}

int alodlm_set_timing(alodlm_t *h, int on) {
    if (!h) return ALODLM_EINVAL;
    h->timing = on != 0;
    return ALODLM_OK;
}

int alodlm_inject_wait_timeout(alodlm_t *h) {
    if (!h) return ALODLM_EINVAL;
    k::wait_expiry_kernel<<<1, 32, 0, h->stream>>>(h->d_err);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ALODLM_OK : cuda_fail(h, e, "wait_expiry_kernel");
}

int alodlm_plan_gemm(int M, int N, int K, int32_t *out) {
    if (!out || M < 1 || N < 1 || K < 1) return fail(nullptr, ALODLM_EINVAL, "plan_gemm: bad argument");
    const GemmShape g = plan_gemm(M, N, K);
    out[0] = g.bn;
    out[1] = g.splits;
    out[2] = g.kps;
    out[3] = g.k_tiles;
    return ALODLM_OK;
}

int alodlm_plan_gemm_noalloc(int M, int N, int K, int num_sms, int32_t *out) {
    if (!out || M < 1 || M > 64 || N < 1 || K < 1 || num_sms < 1)
        return fail(nullptr, ALODLM_EINVAL, "plan_gemm_noalloc: bad argument");
    const SkPlan p = plan_sk(M, N, K, num_sms);
    out[0] = p.bn;
    out[1] = p.grid;
    out[2] = p.upc;
    out[3] = p.max_seg;
    out[4] = p.n_tiles;
    out[5] = p.k_tiles;
    return ALODLM_OK;
}

int alodlm_plan_attention(int packed_rows, int n_kv_heads, int n_seq, int kv_len, int causal, int num_sms,
                          int two_tile_ok, int cluster16_ok, int32_t *out) {
    if (!out || packed_rows < 1 || n_kv_heads < 1 || n_seq < 1 || kv_len < 1 || num_sms < 1)
        return fail(nullptr, ALODLM_EINVAL, "plan_attention: bad argument");
    const AttnPlan a = plan_attention(packed_rows, n_kv_heads, n_seq, kv_len, causal, num_sms, two_tile_ok, cluster16_ok);
    out[0] = a.qtiles;
    out[1] = a.two_tile;
    out[2] = a.splits;
    out[3] = a.keys_per_split;
    out[4] = a.last_to_end;
    return ALODLM_OK;
}

int alodlm_sync(alodlm_t *h) {
    if (!h) return ALODLM_EINVAL;
    cudaError_t e = cudaStreamSynchronize(h->stream);
    if (e != cudaSuccess) return cuda_fail(h, e, "sync");
    int dev_err = 0;
    e = cudaMemcpy(&dev_err, h->d_err, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(h, e, "sync: read error word");
    if (dev_err) {
        // no kernel of a step keeps state across launches that a kernel giving up could leave
        // part-way (cluster merges only): clearing the error word re-arms the handle
        cudaMemsetAsync(h->d_err, 0, sizeof(int), h->stream);
        e = cudaStreamSynchronize(h->stream);
        if (e != cudaSuccess) return cuda_fail(h, e, "sync: clear the error word");
        if (dev_err & DEVERR_TIMEOUT) return fail(h, ALODLM_ETIMEOUT, "a bounded device wait timed out");
        return fail(h, ALODLM_EDEVICE, "a kernel flagged an out-of-range value (token id or exit depth)");
    }
    return ALODLM_OK;
}

}  // extern "C"

namespace {

// Prefix rows through the whole stack, writing their K/V into Core depths 1..n_depths of the
// arena: sequences b0 .. b0+nb-1, positions pos0 .. pos0+n-1 holding ids[b * n + t], attending
// causally to keys [0, pos0 + n) (the positions before pos0 are already in the arena, every
// slot resolved to its depth).  A position with exit depth e runs the Core e times: at depth
// d > e its Core K/V is the depth-e K/V (copied from slot d-1), and the Coda runs once on its
// depth-e state.  Depth on demand: at depth d only the positions with e >= d run the Core (the
// rows are compacted to them), and no depth beyond n_depths is built.  exit: device [B, n]
// exit depths in 1..k_max with e_host its host copy (rows b * n + t), or nullptr / empty for
// k_max everywhere (then n_depths = k_max and every row runs every depth).
int build_prefix_rows(alodlm *h, const int32_t *ids, int b0, int nb, int n, int pos0, const int *exit,
                      const std::vector<int> &e_host, int n_depths) {
    h->fold_layer = -1;  // the stream's contents come from elsewhere
    const alodlm_cfg &c = h->cfg;
    const int M = nb * n, kv_len = pos0 + n;
    RowMap full_map{h->iota + b0, n, pos0};
    float *x = h->hbuf[0];
    int rc;
    LAUNCH(KC_OTHER, 6.0 * M * h->H, 0.0,
           (klaunch(k::embed_kernel, M, 256, 0, h->stream, ids, n, full_map, h->embed, h->V, h->H, x, h->d_err)));
    for (int l = 0; l < c.n_prelude; ++l)
        if ((rc = run_layer(h, l, slot_prelude(h, l), M, full_map, nb, kv_len, 1, x, nullptr))) return rc;
    // rows of the current depth as (slot, position) pairs, in slot then position order
    std::vector<int> cur_seq, cur_t;
    for (int jj = 0; jj < nb; ++jj)
        for (int t = 0; t < n; ++t) {
            cur_seq.push_back(jj);
            cur_t.push_back(t);
        }
    int par = 0;  // x = hbuf[par]
    for (int d = 1; d <= n_depths; ++d) {
        RowMap map = full_map;
        int Md = (int)cur_seq.size();
        if (exit) {
            // the rows that still run at depth d
            std::vector<int> nseq, nt, gather, off(nb, 0), cnt(nb, 0), u;
            for (int m = 0; m < Md; ++m)
                if (e_host[(size_t)(b0 + cur_seq[m]) * n + cur_t[m]] >= d) {
                    gather.push_back(m);
                    nseq.push_back(cur_seq[m]);
                    nt.push_back(cur_t[m]);
                    u.push_back(cnt[cur_seq[m]]++);
                }
            const int Mn = (int)nseq.size();
            if (Mn != Md && Mn > 0) {
                cudaMemcpyAsync(h->pf_gather, gather.data(), Mn * sizeof(int), cudaMemcpyHostToDevice, h->stream);
                LAUNCH(KC_OTHER, 8.0 * Mn * h->H, 0.0,
                       (klaunch(k::gather_idx_rows_kernel, Mn, 256, 0, h->stream, (const float *)h->hbuf[par],
                                h->hbuf[par ^ 1], (const int *)h->pf_gather, h->H)));
                par ^= 1;
                x = h->hbuf[par];
            }
            cur_seq.swap(nseq);
            cur_t.swap(nt);
            Md = Mn;
            if (Md < M) {  // compacted: this depth's row tables
                for (int jj = 1; jj < nb; ++jj) off[jj] = off[jj - 1] + cnt[jj - 1];
                if (Md > 0) {
                    cudaMemcpyAsync(h->pf_row_seq, cur_seq.data(), Md * sizeof(int), cudaMemcpyHostToDevice, h->stream);
                    cudaMemcpyAsync(h->pf_row_t, cur_t.data(), Md * sizeof(int), cudaMemcpyHostToDevice, h->stream);
                    cudaMemcpyAsync(h->pf_row_u, u.data(), Md * sizeof(int), cudaMemcpyHostToDevice, h->stream);
                }
                cudaMemcpyAsync(h->pf_seq_off, off.data(), nb * sizeof(int), cudaMemcpyHostToDevice, h->stream);
                cudaMemcpyAsync(h->pf_seq_cnt, cnt.data(), nb * sizeof(int), cudaMemcpyHostToDevice, h->stream);
                map.row_seq = h->pf_row_seq;
                map.row_u = h->pf_row_u;
                map.row_t = h->pf_row_t;
                map.seq_off = h->pf_seq_off;
                map.seq_cnt = h->pf_seq_cnt;
            }
        }
        for (int cc = 0; cc < c.n_core; ++cc) {
            Fallback fb{exit, n, pos0, b0, nb, d, d > 1 ? slot_core(h, cc, d - 1) : 0};
            const bool use_fb = exit && d > 1;
            if (Md == 0) {  // nothing runs this deep: every position's K/V is its shallower one
                if (use_fb) launch_fallback(h, slot_core(h, cc, d), fb);
                continue;
            }
            if ((rc = run_layer(h, c.n_prelude + cc, slot_core(h, cc, d), Md, map, nb, kv_len, 1, x,
                                use_fb ? &fb : nullptr)))
                return rc;
        }
        if (exit && Md > 0) {
            if (Md == M)
                LAUNCH(KC_OTHER, 8.0 * M * h->H / c.k_max, 0.0,
                       (klaunch(k::capture_exit_kernel, M, 256, 0, h->stream, exit, n, b0, d, x, h->hexit, h->H)));
            else
                LAUNCH(KC_OTHER, 8.0 * Md * h->H / c.k_max, 0.0,
                       (klaunch(k::scatter_exit_kernel, Md, 256, 0, h->stream, exit, n, b0, d, (const int *)h->pf_row_seq,
                                (const int *)h->pf_row_t, (const float *)x, h->hexit, h->H)));
        }
    }
    if (exit) x = h->hexit;
    for (int j = 0; j < c.n_coda; ++j)
        if ((rc = run_layer(h, c.n_prelude + c.n_core + j, slot_coda(h, j), M, full_map, nb, kv_len, 1, x, nullptr)))
            return rc;
    return check_launch(h, "prefix rows");
}

// Core depths (from, to] of every cached position [0, n_pos) of every sequence become copies of
// depth `from`: a depth that no position had reached, filled when a longer-looping position
// joins the prefix.
void fill_depths(alodlm *h, int from, int to, int n_pos) {
    for (int d = from + 1; d <= to; ++d)
        for (int cc = 0; cc < h->cfg.n_core; ++cc) {
            const long long so = (long long)slot_core(h, cc, from) * h->slot_elems;
            const long long dst = (long long)slot_core(h, cc, d) * h->slot_elems;
            LAUNCH(KC_OTHER, 8.0 * h->B * h->nkv * n_pos * h->hd, 0.0,
                   (klaunch(k::copy_positions_kernel, dim3(h->B, h->nkv), 256, 0, h->stream,
                            (const bf16 *)(h->kv_k + so), (const bf16 *)(h->kv_v + so), h->kv_k + dst, h->kv_v + dst,
                            n_pos, h->seq_stride, h->head_stride, h->hd)));
        }
}

// host copy of device exit depths and their maximum (0 when exit is null)
int exit_depths_to_host(alodlm *h, const int *exit, long long n, std::vector<int> &e_host, int &max_e) {
    max_e = 0;
    e_host.clear();
    if (!exit) return ALODLM_OK;
    e_host.resize(n);
    cudaError_t e = cudaMemcpyAsync(e_host.data(), exit, n * sizeof(int), cudaMemcpyDeviceToHost, h->stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(h->stream);
    if (e != cudaSuccess) return cuda_fail(h, e, "exit depths");
    for (int v : e_host) {
        if (v < 1 || v > h->cfg.k_max) return fail(h, ALODLM_EDEVICE, "exit depth outside 1..k_max");
        max_e = std::max(max_e, v);
    }
    return ALODLM_OK;
}

}  // namespace

extern "C" {

int alodlm_prefill(alodlm_t *h, const int32_t *prefix_ids, int B, int P, const int32_t *exit_depth) {
    const NvtxRange range("alodlm prefill");
    if (!h || !prefix_ids) return fail(h, ALODLM_EINVAL, "null argument");
    const alodlm_cfg &c = h->cfg;
    if (B < 1 || B > c.max_batch || P < 1 || P > c.max_prefix)
        return fail(h, ALODLM_EINVAL, "prefill: B or P out of range");
    reset_stats(h);
    h->prefilled = false;
    std::vector<int> e_host;
    int max_e = 0, rc;
    if (exit_depth) {
        cudaMemcpyAsync(h->exit_dev, exit_depth, (size_t)B * P * sizeof(int), cudaMemcpyDeviceToDevice, h->stream);
        if ((rc = exit_depths_to_host(h, h->exit_dev, (long long)B * P, e_host, max_e))) return rc;
    }
    // depth on demand: no Core depth beyond the deepest exit depth is built
    const int depths = exit_depth ? max_e : c.k_max;
    const int g = std::max(1, std::min(B, h->rows_cap / P));
    for (int b0 = 0; b0 < B; b0 += g)
        if ((rc = build_prefix_rows(h, prefix_ids, b0, std::min(g, B - b0), P, 0, exit_depth ? h->exit_dev : nullptr,
                                    e_host, depths)))
            return rc;
    h->B = B;
    h->P = P;
    h->depth_built = depths;
    h->prefilled = true;
    return ALODLM_OK;
}

int alodlm_append(alodlm_t *h, const int32_t *ids, int B, int N, const int32_t *exit_depth) {
    const NvtxRange range("alodlm append");
    if (!h || !ids) return fail(h, ALODLM_EINVAL, "null argument");
    const alodlm_cfg &c = h->cfg;
    if (!h->prefilled) return fail(h, ALODLM_ESTATE, "append before prefill");
    if (B != h->B) return fail(h, ALODLM_ESTATE, "batch differs from the prefill's");
    if (N < 1 || N > c.max_block) return fail(h, ALODLM_EINVAL, "append: N out of range (1..max_block)");
    if (h->P + N > c.max_prefix) return fail(h, ALODLM_EINVAL, "append: the prefix would pass max_prefix");
    reset_stats(h);
    std::vector<int> e_host;
    int max_e = 0, rc;
    if (exit_depth) {
        cudaMemcpyAsync(h->app_exit, exit_depth, (size_t)B * N * sizeof(int), cudaMemcpyDeviceToDevice, h->stream);
        if ((rc = exit_depths_to_host(h, h->app_exit, (long long)B * N, e_host, max_e))) return rc;
    }
    const int need = exit_depth ? max_e : c.k_max;
    if (need > h->depth_built) {  // the cached positions get the depths the new ones reach first
        fill_depths(h, h->depth_built, need, h->P);
        h->depth_built = need;
    }
    if ((rc = build_prefix_rows(h, ids, 0, B, N, h->P, exit_depth ? h->app_exit : nullptr, e_host,
                                h->depth_built))) {
        h->prefilled = false;  // the arena may hold part of the new positions
        return rc;
    }
    h->P += N;
    return ALODLM_OK;
}

}  // extern "C"

namespace {

int denoise_step_impl(alodlm *h, const int32_t *block_ids, int B, int N, float tau_H, float lambda, int k_max,
                      int rule, const SampleParams &sp, const alodlm_step_out *out) {
    const NvtxRange range("alodlm step");
    if (!h || !block_ids || !out || !out->tokens || !out->exit_depth || !out->entropy || !out->halt ||
        !out->cum_halt || !out->loops_run || !out->active_rows || !out->readout_rows)
        return fail(h, ALODLM_EINVAL, "null argument");
    const alodlm_cfg &c = h->cfg;
    if (!h->prefilled) return fail(h, ALODLM_ESTATE, "denoise_step before prefill");
    if (B != h->B) return fail(h, ALODLM_ESTATE, "batch differs from the prefill's");
    if (N < 1 || N > c.max_block) return fail(h, ALODLM_EINVAL, "N out of range");
    if (k_max < 1 || k_max > c.k_max) return fail(h, ALODLM_EINVAL, "k_max out of range");
    if (rule != ALODLM_RULE_PAPER && rule != ALODLM_RULE_PER_TOKEN) return fail(h, ALODLM_EINVAL, "unknown rule");
    if (std::isnan(tau_H) || std::isnan(lambda)) return fail(h, ALODLM_EINVAL, "tau_H/lambda is NaN");
    reset_stats(h);
    const int H = h->H, P = h->P;
    const int K = k_max;
    h->last_N = N;
    k::StepState st;
    st.tokens = out->tokens;
    st.exit_depth = out->exit_depth;
    st.tr_H = out->entropy;
    st.tr_lam = out->halt;
    st.tr_a = out->cum_halt;
    st.loops_run = out->loops_run;
    st.active_rows = out->active_rows;
    st.readout_rows = out->readout_rows;
    st.U = h->U;
    st.a = h->a;
    st.cur_H = h->cur_H;
    st.cur_y = h->cur_y;
    st.cont = h->cont;
    st.n_commit = h->ncommit;

    int cur = 0, hi = 0, rc;
    const long long BNt = (long long)B * N;
    LAUNCH(KC_COMMIT, 16.0 * BNt, 0.0,
           (klaunch(k::step_init_kernel, (unsigned)std::min<long long>((BNt + 255) / 256, 1024), 256, 0, h->stream, 
               block_ids, B, N, K, c.mask_id, st, sp, h->samp)));
    LAUNCH(KC_COMMIT, 8.0 * BNt, 0.0,
           (klaunch(k::plan_kernel, 1, 1024, 0, h->stream, B, h->iota, N, h->cont, h->U, h->seq_of[0], h->old_slot,
                                                      h->ridx, h->rr_b, h->rr_i, h->counts, 1, K, out->active_rows,
                                                      out->readout_rows, h->d_err)));
    int n_act = B;
    RowMap map{h->seq_of[0], N, P};
    int M = n_act * N;
    float *x = h->hbuf[hi];
    LAUNCH(KC_OTHER, 6.0 * M * H, 0.0,
           (klaunch(k::embed_kernel, M, 256, 0, h->stream, block_ids, N, map, h->embed, h->V, H, x, h->d_err)));
    h->fold_layer = -1;
    for (int l = 0; l < c.n_prelude; ++l)
        if ((rc = run_layer(h, l, slot_prelude(h, l), M, map, n_act, P + N, 0, x, nullptr))) return rc;

    // One loop: Core, Coda, readout over the U rows (their count is read on the device, the
    // grids are sized for every row of the looping sequences), commit/merge and the plan of the
    // next loop, then the 16-byte control word to the host.  With a capture-capable stream the
    // loop is recorded once per (loop, looping sequences, buffer parity, outputs, thresholds)
    // as a CUDA graph and replayed.
    auto enqueue_loop = [&](int s, int n_act_, int cur_, int hi_) -> int {
        RowMap mp{h->seq_of[cur_], N, P};
        const int Ml = n_act_ * N;
        // loop 1 continues the Prelude's rows; later loops start from the merged (and possibly
        // compacted) states
        if (s > 1) h->fold_layer = -1;
        float *xl = h->hbuf[hi_];
        const long long dbg_off = (long long)(s - 1) * c.max_batch * c.max_block * H;
        int r;
        if (c.debug_dump)
            LAUNCH(KC_OTHER, 0.0, 0.0,
                   (klaunch(k::dump_rows_kernel, Ml, 256, 0, h->stream, xl, mp, H, h->dbg[0] + dbg_off)));
        for (int cc = 0; cc < c.n_core; ++cc) {
            if ((r = run_layer(h, c.n_prelude + cc, slot_core(h, cc, std::min(s, h->depth_built)), Ml, mp, n_act_,
                               P + N, 0, xl, nullptr)))
                return r;
            if (cc == 0 && c.debug_dump)
                LAUNCH(KC_OTHER, 0.0, 0.0,
                       (klaunch(k::dump_rows_kernel, Ml, 256, 0, h->stream, xl, mp, H, h->dbg[3] + dbg_off)));
        }
        if (c.debug_dump)
            LAUNCH(KC_OTHER, 0.0, 0.0,
                   (klaunch(k::dump_rows_kernel, Ml, 256, 0, h->stream, xl, mp, H, h->dbg[1] + dbg_off)));
        cudaMemcpyAsync(h->hc, xl, (size_t)Ml * H * sizeof(float), cudaMemcpyDeviceToDevice, h->stream);
        if (h->fold_x == xl) h->fold_x = h->hc;  // the Coda runs on a copy of the same rows
        for (int j = 0; j < c.n_coda; ++j)
            if ((r = run_layer(h, c.n_prelude + c.n_core + j, slot_coda(h, j), Ml, mp, n_act_, P + N, 0, h->hc,
                               nullptr)))
                return r;
        float *dbg_r = c.debug_dump ? h->dbg[2] + dbg_off : nullptr;
        LAUNCH(KC_NORM, 4.0 * Ml * H + 2.0 * Ml * H, 0.0,
               (klaunch(k::final_norm_kernel, Ml, 256, 0, h->stream, h->hc, h->final_norm, h->exit_w, h->exit_b, H,
                        c.rms_eps, mp, h->ridx, h->rb, h->lam_rr, dbg_r)));
        {
            gemm::EpiParams ep{};
            ep.partials = h->part;
            ep.n_btiles = h->n_vt;
            ep.spartials = h->spart;
            ep.samp = h->samp;
            ep.rr_b = h->rr_b;
            ep.rr_i = h->rr_i;
            ep.N = N;
            ep.loop = s;
            const double R_est = Ml;  // upper bound on the readout rows (exact counts are on the device)
            const double bytes = 2.0 * h->V * H + 2.0 * R_est * H + 16.0 * R_est * h->n_vt;
            LAUNCH(KC_RGEMM, bytes, 2.0 * R_est * h->V * (double)H,
                   (launch_persist<256, gemm::EPI_READOUT>(h->tm_rb, h->tm_lm, Ml, h->V, h->counts + 1,
                                                           cdiv(H, gemm::BK), 1, ep, h->d_err, h->stream,
                                                           h->num_sms, 2)));
            LAUNCH(KC_RCOMB, 16.0 * R_est * h->n_vt, 0.0,
                   (klaunch(k::readout_combine_kernel, cdiv(Ml, 8), 256, 0, h->stream, h->part,
                            (const double2 *)h->spart, (const SampleParams *)h->samp, h->n_vt, h->counts + 1, h->rr_b, h->rr_i, h->lam_rr, N, K, s, h->a, h->cur_H,
                       h->cur_y, out->entropy, out->halt, out->cum_halt)));
        }
        LAUNCH(KC_COMMIT, 16.0 * Ml, 0.0,
               (klaunch(k::commit_kernel, n_act_, 256, 0, h->stream, mp, s, K, rule, tau_H, lambda, h->embed, H, xl,
                                                               st)));
        LAUNCH(KC_COMMIT, 8.0 * Ml, 0.0,
               (klaunch(k::plan_kernel, 1, 1024, 0, h->stream, n_act_, h->seq_of[cur_], N, h->cont, h->U,
                                                          h->seq_of[cur_ ^ 1], h->old_slot, h->ridx, h->rr_b,
                                                          h->rr_i, h->counts, s + 1, K, out->active_rows,
                                                          out->readout_rows, h->d_err)));
        cudaMemcpyAsync(h->counts_host, h->counts, 4 * sizeof(int), cudaMemcpyDeviceToHost, h->stream);
        return ALODLM_OK;
    };

    const bool graphs = h->use_graphs && !h->timing && h->stream != nullptr && h->stream != cudaStreamLegacy &&
                        h->stream != cudaStreamPerThread;
    for (int s = 1; s <= K; ++s) {
        const NvtxRange loop_range("alodlm loop", s);
        if (graphs) {
            const GraphKey key{s, n_act, cur, hi, N, K, rule, P, h->depth_built, tau_H, lambda, out->tokens, out->exit_depth,
                               out->entropy, out->halt, out->cum_halt, out->loops_run, out->active_rows,
                               out->readout_rows};
            cudaGraphExec_t exec = nullptr;
            for (auto &g : h->graphs)
                if (g.key == key) exec = g.exec;
            if (!exec) {
                if (h->graphs.size() >= 512) clear_graphs(h);
                const int launches_before = h->launches;
                cudaError_t e = cudaStreamBeginCapture(h->stream, cudaStreamCaptureModeThreadLocal);
                if (e != cudaSuccess) return cuda_fail(h, e, "graph capture begin");
                rc = enqueue_loop(s, n_act, cur, hi);
                cudaGraph_t graph = nullptr;
                e = cudaStreamEndCapture(h->stream, &graph);
                if (rc) {
                    if (graph) cudaGraphDestroy(graph);
                    return rc;
                }
                if (e != cudaSuccess) return cuda_fail(h, e, "graph capture end");
                e = cudaGraphInstantiate(&exec, graph, 0);
                cudaGraphDestroy(graph);
                if (e != cudaSuccess) return cuda_fail(h, e, "graph instantiate");
                h->graphs.push_back({key, exec, h->launches - launches_before});
            } else {
                for (auto &g : h->graphs)
                    if (g.exec == exec) h->launches += g.n_kernels;
            }
            cudaError_t e = cudaGraphLaunch(exec, h->stream);
            if (e != cudaSuccess) return cuda_fail(h, e, "graph launch");
        } else {
            if ((rc = enqueue_loop(s, n_act, cur, hi))) return rc;
        }
        cudaError_t e = cudaStreamSynchronize(h->stream);
        if (e != cudaSuccess) return cuda_fail(h, e, "step: loop control");
        if ((rc = check_launch(h, "step"))) return rc;
        if (h->counts_host[2]) return alodlm_sync(h);
        const int n_next = h->counts_host[0];
        if (n_next == 0) break;
        if (n_next != n_act) {
            x = h->hbuf[hi];
            LAUNCH(KC_COMMIT, 8.0 * n_next * N * H, 0.0,
                   (klaunch(k::gather_rows_kernel, n_next * N, 256, 0, h->stream, x, h->hbuf[hi ^ 1], h->old_slot, N, H)));
            hi ^= 1;
        }
        cur ^= 1;
        n_act = n_next;
    }
    return check_launch(h, "step end");
}

}  // namespace

extern "C" {

int alodlm_denoise_step(alodlm_t *h, const int32_t *block_ids, int B, int N, float tau_H, float lambda, int k_max,
                        int rule, const alodlm_step_out *out) {
    const SampleParams greedy{0ull, 0ull, 0, 0};
    return denoise_step_impl(h, block_ids, B, N, tau_H, lambda, k_max, rule, greedy, out);
}

int alodlm_denoise_step_sampled(alodlm_t *h, const int32_t *block_ids, int B, int N, float tau_H, float lambda,
                                int k_max, int rule, uint64_t seed, uint64_t step, const alodlm_step_out *out) {
    const SampleParams sp{(unsigned long long)seed, (unsigned long long)step, 1, 0};
    return denoise_step_impl(h, block_ids, B, N, tau_H, lambda, k_max, rule, sp, out);
}

int alodlm_set_graphs(alodlm_t *h, int on) {
    if (!h) return ALODLM_EINVAL;
    h->use_graphs = on != 0;
    if (!h->use_graphs) clear_graphs(h);
    return ALODLM_OK;
}

int alodlm_debug_state(alodlm_t *h, int which, int loop, float *dst) {
    if (!h || !dst) return ALODLM_EINVAL;
    if (!h->cfg.debug_dump) return fail(h, ALODLM_EINVAL, "debug_dump is off");
    if (which < 0 || which > 3 || loop < 1 || loop > h->cfg.k_max || h->last_N < 1)
        return fail(h, ALODLM_EINVAL, "debug_state: out of range or no step yet");
    const float *src = h->dbg[which] + (size_t)(loop - 1) * h->cfg.max_batch * h->cfg.max_block * h->H;
    cudaError_t e = cudaMemcpyAsync(dst, src, (size_t)h->B * h->last_N * h->H * sizeof(float),
                                    cudaMemcpyDeviceToDevice, h->stream);
    return e == cudaSuccess ? ALODLM_OK : cuda_fail(h, e, "debug_state");
}

int alodlm_kv_slot(alodlm_t *h, int which, int slot, int b, int n_pos, void *dst) {
    if (!h || !dst || which < 0 || which > 1 || slot < 0 || slot >= h->n_slots || b < 0 ||
        b >= h->cfg.max_batch || n_pos < 1 || n_pos > h->pos_stride)
        return h ? fail(h, ALODLM_EINVAL, "kv_slot: out of range") : ALODLM_EINVAL;
    // a Core depth beyond the deepest built one is served by the deepest built one
    const int core0 = h->cfg.n_prelude, core_end = core0 + h->cfg.k_max * h->cfg.n_core;
    if (slot >= core0 && slot < core_end && h->depth_built > 0) {
        const int d = (slot - core0) / h->cfg.n_core + 1, cc = (slot - core0) % h->cfg.n_core;
        if (d > h->depth_built) slot = slot_core(h, cc, h->depth_built);
    }
    const bf16 *base = (which ? h->kv_v : h->kv_k) + (long long)slot * h->slot_elems + (long long)b * h->seq_stride;
    cudaError_t e = cudaMemcpy2DAsync(dst, (size_t)n_pos * h->hd * 2, base, (size_t)h->head_stride * 2,
                                      (size_t)n_pos * h->hd * 2, h->nkv, cudaMemcpyDeviceToDevice, h->stream);
    return e == cudaSuccess ? ALODLM_OK : cuda_fail(h, e, "kv_slot");
}

int alodlm_step_stats(const alodlm_t *hc, int *kernel_launches, double *times_ms, int *launches, double *bytes,
                      double *flops) {
    alodlm *h = const_cast<alodlm *>(hc);
    if (!h) return ALODLM_EINVAL;
    if (kernel_launches) *kernel_launches = h->launches;
    for (int c = 0; c < ALODLM_N_KCLASS; ++c) {
        if (times_ms) times_ms[c] = 0.0;
        if (launches) launches[c] = h->cls_launches[c];
        if (bytes) bytes[c] = h->cls_bytes[c];
        if (flops) flops[c] = h->cls_flops[c];
    }
    if (times_ms && !h->timed.empty()) {
        cudaError_t e = cudaStreamSynchronize(h->stream);
        if (e != cudaSuccess) return cuda_fail(h, e, "stats");
        for (const auto &t : h->timed) {
            float ms = 0.f;
            cudaEventElapsedTime(&ms, t.e0, t.e1);
            times_ms[t.cls] += ms;
        }
    }
    return ALODLM_OK;
}

int alodlm_gemm_bf16(const void *A, const void *W, float *C, int M, int N, int K, float *workspace,
                     size_t workspace_bytes, void *stream) {
    if (!A || !W || !C || !workspace || workspace_bytes < 256 || M < 1 || N < 1 || K < 8 || K % 8)
        return ALODLM_EINVAL;
    if (!get_encode_fn() || !init_kernel_attrs()) return ALODLM_ECUDA;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // workspace: the status word (split-K reduces inside a cluster; nothing else is needed)
    GemmEnv env{};
    env.err = reinterpret_cast<int *>(workspace);
    env.st = static_cast<cudaStream_t>(stream);
    env.num_sms = sms;
    CUtensorMap tW, tA;
    if (!make_tmap(&tW, W, K, N, gemm::BM)) return ALODLM_ECUDA;
    auto map_for_bn = [&](int bn) -> const CUtensorMap * { return make_tmap(&tA, A, K, M, bn) ? &tA : nullptr; };
    if (run_gemm(env, tW, N, map_for_bn, M, K, gemm::EPI_F32, C, N, nullptr, 0, 0) < 0)
        return ALODLM_ECUDA;
    return cudaGetLastError() == cudaSuccess ? ALODLM_OK : ALODLM_ECUDA;
}

// ---------------------------------------------------------------------------------
// Allocation-free GEMM.  Its scratch (status word, tile counters, split partials) is a fixed
// array compiled into the library; host code reaches it only through the device address
// looked up once per device.
// ---------------------------------------------------------------------------------
}  // extern "C"

namespace {
constexpr size_t NOALLOC_HEAD_FLOATS = 64;       // status word + spare
constexpr size_t NOALLOC_COUNTER_FLOATS = 1024;  // tile counters (N <= 32768 -> <= 256 tiles)
constexpr size_t NOALLOC_PARTIAL_FLOATS = 4u << 20;
constexpr size_t NOALLOC_FLOATS = NOALLOC_HEAD_FLOATS + NOALLOC_COUNTER_FLOATS + NOALLOC_PARTIAL_FLOATS;
constexpr int NOALLOC_MAX_M = 64, NOALLOC_MAX_N = 32768, NOALLOC_MAX_K = 32768;

std::mutex g_noalloc_mu;
// per device: the context the address was looked up in, and the address
CUcontext g_noalloc_ctx[64] = {nullptr};
float *g_noalloc_addr[64] = {nullptr};

// the driver's cuCtxGetCurrent, fetched through the runtime like the tensor-map encoder
using CtxGetCurrentFn = CUresult (*)(CUcontext *);
CtxGetCurrentFn get_ctx_fn() {
    static CtxGetCurrentFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    }
    return fn;
}
}  // namespace

static __device__ __align__(256) float g_noalloc_scratch[NOALLOC_FLOATS];

extern "C" {

int alodlm_gemm_bf16_noalloc(const void *A, const void *W, float *C, int M, int N, int K, int32_t *status,
                             void *stream) {
    if (!A || !W || !C) return fail(nullptr, ALODLM_EINVAL, "gemm_bf16_noalloc: null pointer");
    if (M < 1 || M > NOALLOC_MAX_M || N < 1 || N > NOALLOC_MAX_N || K < 8 || K > NOALLOC_MAX_K || K % 8)
        return fail(nullptr, ALODLM_EINVAL,
                    "gemm_bf16_noalloc: needs 1 <= M <= 64, 1 <= N <= 32768, 8 <= K <= 32768, K % 8 == 0");
    if (!get_encode_fn() || !init_kernel_attrs() || !get_ctx_fn())
        return fail(nullptr, ALODLM_ECUDA, "gemm_bf16_noalloc: driver entry points or kernel attributes");
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return fail(nullptr, ALODLM_ECUDA, "gemm_bf16_noalloc: device index");
    CUcontext ctx = nullptr;
    if (get_ctx_fn()(&ctx) != CUDA_SUCCESS || !ctx)
        return fail(nullptr, ALODLM_ECUDA, "gemm_bf16_noalloc: no current context");
    float *scratch = nullptr;
    {
        // first call on this device (or in a new context of it, e.g. after cudaDeviceReset):
        // look up the device address of the scratch array -- its name in host code is only a
        // stand-in for it
        std::lock_guard<std::mutex> lk(g_noalloc_mu);
        if (!g_noalloc_addr[dev] || g_noalloc_ctx[dev] != ctx) {
            void *p = nullptr;
            cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
            if (e != cudaSuccess) {
                cudaGetLastError();
                return fail(nullptr, ALODLM_ECUDA, std::string("gemm_bf16_noalloc: cudaGetSymbolAddress: ") +
                                                       cudaGetErrorString(e));
            }
            g_noalloc_addr[dev] = static_cast<float *>(p);
            g_noalloc_ctx[dev] = ctx;
        }
        scratch = g_noalloc_addr[dev];
    }
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const SkPlan plan = plan_sk(M, N, K, sms);
    if ((size_t)plan.n_tiles > NOALLOC_COUNTER_FLOATS ||
        (size_t)plan.n_tiles * plan.max_seg * gemm::BM * plan.bn > NOALLOC_PARTIAL_FLOATS)
        return fail(nullptr, ALODLM_EINVAL, "gemm_bf16_noalloc: shape needs more scratch than the fixed array holds");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the array keeps the previous call's contents: the status word and the counters must start at zero
    cudaError_t e = cudaMemsetAsync(scratch, 0, (NOALLOC_HEAD_FLOATS + NOALLOC_COUNTER_FLOATS) * sizeof(float), st);
    if (e != cudaSuccess) return fail(nullptr, ALODLM_ECUDA, std::string("gemm_bf16_noalloc: ") + cudaGetErrorString(e));
    CUtensorMap tW, tA;
    if (!make_tmap(&tW, W, K, N, gemm::BM) || !make_tmap(&tA, A, K, M, plan.bn))
        return fail(nullptr, ALODLM_ECUDA, "gemm_bf16_noalloc: cuTensorMapEncodeTiled failed");
    GemmEnv env{};
    env.err = reinterpret_cast<int *>(scratch);
    env.counters = reinterpret_cast<int *>(scratch + NOALLOC_HEAD_FLOATS);
    env.n_counters = (int)NOALLOC_COUNTER_FLOATS;
    env.ws = scratch + NOALLOC_HEAD_FLOATS + NOALLOC_COUNTER_FLOATS;
    env.ws_floats = NOALLOC_PARTIAL_FLOATS;
    env.st = st;
    env.num_sms = sms;
    gemm::EpiParams ep{};
    ep.out = C;
    ep.ldo = N;
    launch_sk<gemm::EPI_F32>(plan, tW, tA, N, M, ep, env);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(nullptr, ALODLM_ECUDA, std::string("gemm_bf16_noalloc: ") + cudaGetErrorString(e));
    // hand the call's status word to the caller before the next call clears it
    if (status) {
        e = cudaMemcpyAsync(status, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess)
            return fail(nullptr, ALODLM_ECUDA, std::string("gemm_bf16_noalloc: status copy: ") + cudaGetErrorString(e));
    }
    return ALODLM_OK;
}

}  // extern "C"
