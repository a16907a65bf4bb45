// C ABI of the MoE layer forward pass (include/moe.h): argument checks,
// workspace layout, TMA tensor maps and the launch sequence.  Host code only.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "../../include/moe.h"
#include "moe_launch.h"

#ifdef MOE_DEBUG
constexpr bool kDebugBuild = true;   // the checking build (libmoe_b200_debug.so)
#else
constexpr bool kDebugBuild = false;
#endif

// Checking build: the one-shot table corruption armed by moe_debug_corrupt_next
// (tests of the bounds checks).  The regular build never arms it.
struct DebugCorruption {
    int table = -1, index = 0, value = 0;
};
static std::mutex g_debug_mu;
static DebugCorruption g_debug_corruption;

using namespace moe;

namespace {

// ------------------------------------------------------------------ checks
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status check_config(const moe_config* c) {
    if (!c) return MOE_ERR_INVALID_ARG;
    if (c->d <= 0 || c->d % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (c->n_experts <= 0 || c->n_experts > 1024) return MOE_ERR_INVALID_ARG;
    if (c->n_groups <= 0 || c->n_groups > 32 || c->n_experts % c->n_groups != 0) return MOE_ERR_INVALID_ARG;
    const int gs = c->n_experts / c->n_groups;
    if (gs < 2) return MOE_ERR_INVALID_ARG;
    if (c->topk_groups < 1 || c->topk_groups > c->n_groups) return MOE_ERR_INVALID_ARG;
    if (c->top_k < 1 || c->top_k > 32 || c->top_k > c->topk_groups * gs) return MOE_ERR_INVALID_ARG;
    if (c->hidden <= 0 || c->hidden % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (c->n_shared != 0 && c->n_shared != 1) return MOE_ERR_INVALID_ARG;
    if (c->n_shared == 1 && (c->shared_hidden <= 0 || c->shared_hidden % 128 != 0)) return MOE_ERR_INVALID_ARG;
    if (c->act_dtype != MOE_F32 && c->act_dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (c->weight_dtype != MOE_BF16 && c->weight_dtype != MOE_E4M3) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

struct DevInfo {
    int sm_count = 0;
    int major = 0;
};

DevInfo dev_info() {
    static std::mutex mu;
    static DevInfo cache[64];
    static bool have[64] = {};
    int dev = 0;
    DevInfo info;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return info;
    std::lock_guard<std::mutex> g(mu);
    if (dev < 64 && have[dev]) return cache[dev];
    cudaDeviceGetAttribute(&info.sm_count, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&info.major, cudaDevAttrComputeCapabilityMajor, dev);
    if (dev < 64) {
        cache[dev] = info;
        have[dev] = true;
    }
    return info;
}

moe_status check_device(DevInfo* out) {
    DevInfo i = dev_info();
    if (i.major != 10 || i.sm_count <= 0) return MOE_ERR_UNSUPPORTED;
    *out = i;
    return MOE_OK;
}

// ------------------------------------------------------------------ TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D row-major [rows, cols] map, box [box_rows, box_cols], 128-byte swizzle,
// out-of-bounds elements read as zero.
bool map_2d(CUtensorMap* m, CUtensorMapDataType dt, int elem_bytes, const void* ptr, uint64_t rows, uint64_t cols,
            uint32_t box_rows, uint32_t box_cols) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * (uint64_t)elem_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool map_bf16(CUtensorMap* m, const void* p, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    return map_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p, rows, cols, box_rows, 64);
}

// ------------------------------------------------------------------ tiles
// Token-chunk width BN of the grouped GEMMs from the mean rows per expert.
// An item loads only the rows it has (32-row boxes), so a wide BN costs no
// traffic, only pipeline depth and TMEM double buffering: small BN for decode
// (a few tokens per expert, deep pipeline), 256 once experts hold ~100 rows,
// so that an expert's weights are streamed once and never split in chunks.
int pick_bn(long long rows_per_expert) {
    if (rows_per_expert <= 16) return 32;
    if (rows_per_expert <= 40) return 64;
    if (rows_per_expert <= 96) return 128;
    return 256;
}

constexpr int kBoxRows = 32;  // token rows per B-operand TMA box
constexpr int kFp8MaxBn = 64;  // FP8 GEMMs hold their promoted sums in registers
constexpr int kPermuteMultiMinT = 1024;  // tokens above which the permutation runs on many CTAs
constexpr int kPairBoxRows = 64;  // token rows per B box in the CTA-pair GEMMs (PAIR_BOX_ROWS)

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Router GEMM tiling: token chunk and K splits.  At decode sizes the whole
// router weight would be streamed by a handful of CTAs; splitting K spreads it
// over about one item per SM.  The partial logits are summed in a fixed order
// by the selection kernel, so the logits do not depend on scheduling.
int router_bn(int T) { return T <= 256 ? 32 : 128; }
int router_splits(int T, int n_sm) {
    const int items = (T + router_bn(T) - 1) / router_bn(T);
    int s = n_sm / items;
    return s < 1 ? 1 : (s > 16 ? 16 : s);
}
// Rows of partial logits to reserve: an upper bound of splits x T that does
// not decrease with T (a workspace sized for T_max serves every T <= T_max):
// splits <= 16, and splits x chunks <= 148 when splits > 1.
size_t router_part_rows(int T) {
    const size_t t = (size_t)T;
    if (T <= 256) return t * 16 < 148 * 32 ? t * 16 : 148 * 32;
    const size_t b = t * 16 < 148 * 128 ? t * 16 : 148 * 128;
    return b > t ? b : t;
}

bool map_u8(CUtensorMap* m, const void* p, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    return map_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p, rows, cols, box_rows, 128);
}

struct Workspace {
    float* logits;
    float* part;             // split-K partial router logits
    int32_t* hist;           // per-CTA expert histograms of the multi-CTA permutation
    int32_t* idx;
    float* w;
    int32_t* counts;
    int32_t* offsets;
    int32_t* src;
    int32_t* inv;
    int32_t* row_tok;
    float* row_coef;
    int32_t* row_off;
    int32_t* item_gu;
    int32_t* item_dn;
    __nv_bfloat16* x_perm;   // bf16 weights: permuted activations [rows, d]
    __nv_bfloat16* h_perm;   // bf16 weights: SwiGLU output [rows, ldh]
    uint8_t* x_q;            // e4m3 weights: quantised x [T, d] and its scales [T, d/128]
    float* sx;
    uint8_t* xq_perm;        // permuted codes [rows, d] and scales [d/128][rows]
    float* sxT;
    uint8_t* hq;             // h codes [rows, ldh] and scales [ldh/128][rows]
    float* shT;
    float* y_acc;
    size_t bytes;
};

// Lays out the workspace for T tokens from `base` (NULL: sizes only).
Workspace layout(const moe_config* c, int T, void* base) {
    Workspace w;
    memset(&w, 0, sizeof(w));
    const size_t E = c->n_experts, k = c->top_k, NG = E + c->n_shared;
    const size_t rows = (size_t)T * k + (size_t)c->n_shared * T;
    const size_t ldh = c->hidden > c->shared_hidden ? c->hidden : c->shared_hidden;
    size_t off = 0;
    uint8_t* b = static_cast<uint8_t*>(base);
    auto take = [&](size_t bytes) -> void* {
        void* p = base ? b + off : nullptr;
        off = align_up(off + bytes, 1024);
        return p;
    };
    w.logits = (float*)take((size_t)T * E * 4);
    w.part = (float*)take(router_part_rows(T) * E * 4);
    w.idx = (int32_t*)take((size_t)T * k * 4);
    w.w = (float*)take((size_t)T * k * 4);
    w.hist = (int32_t*)take((size_t)permute_blocks(T) * E * 4);
    w.counts = (int32_t*)take(E * 4);
    w.offsets = (int32_t*)take((E + 1) * 4);
    w.src = (int32_t*)take((size_t)T * k * 4);
    w.inv = (int32_t*)take((size_t)T * k * 4);
    w.row_tok = (int32_t*)take(rows * 4);
    w.row_coef = (float*)take(rows * 4);
    w.row_off = (int32_t*)take((NG + 1) * 4);
    w.item_gu = (int32_t*)take((NG + 1) * 4);
    w.item_dn = (int32_t*)take((NG + 1) * 4);
    if (c->weight_dtype == MOE_E4M3) {
        w.x_q = (uint8_t*)take((size_t)T * c->d);
        w.sx = (float*)take((size_t)T * (c->d / 128) * 4);
        w.xq_perm = (uint8_t*)take(rows * (size_t)c->d);
        w.sxT = (float*)take(rows * (size_t)(c->d / 128) * 4);
        w.hq = (uint8_t*)take(rows * ldh);
        w.shT = (float*)take(rows * (ldh / 128) * 4);
    } else {
        w.x_perm = (__nv_bfloat16*)take(rows * (size_t)c->d * 2);
        w.h_perm = (__nv_bfloat16*)take(rows * ldh * 2);
    }
    w.y_acc = (float*)take((size_t)T * c->d * 4);
    w.bytes = off;
    return w;
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// NVTX ranges around the host-side enqueue of each stage (names "moe.<stage>"),
// nested in one range per entry point: a profiler's timeline groups the kernels
// by stage, and ncu can select them with --nvtx-include.  Header-only NVTX: with
// no tool attached each push/pop is a call through a null stub.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

// Consecutive stages of one call: next() closes the open stage range, if any,
// and opens the named one; the destructor closes the last.
class NvtxStages {
    bool open_ = false;

public:
    NvtxStages() = default;
    NvtxStages(const NvtxStages&) = delete;
    NvtxStages& operator=(const NvtxStages&) = delete;
    void next(const char* name) {
        if (open_) nvtxRangePop();
        nvtxRangePushA(name);
        open_ = true;
    }
    ~NvtxStages() {
        if (open_) nvtxRangePop();
    }
};

// The kernels one forward call runs, decided from the shapes and the SM count.
struct Plan {
    int bn;              // token rows per grouped-GEMM tile
    bool fp8;            // e4m3 expert weights
    bool pair;           // bf16 grouped GEMMs on CTA pairs
    bool pair8;          // e4m3 grouped GEMMs on CTA pairs
    int router_parts;    // K splits of the router GEMM (1 with fp32 activations)
    bool permute_multi;  // many-CTA permutation
};

Plan make_plan(const moe_config* c, int T, int n_sm) {
    Plan p;
    p.fp8 = c->weight_dtype == MOE_E4M3;
    const int H = c->hidden, Hs = c->n_shared ? c->shared_hidden : c->hidden, d = c->d;
    // token rows per group: the routed experts' average, or all T rows of the one
    // dense group when there is no routed expert
    p.bn = pick_bn(c->n_experts ? ((long long)T * c->top_k + c->n_experts - 1) / c->n_experts : T);
    // wide token tiles run on CTA pairs (2-SM MMA), each SM loading half of the
    // token rows.  bf16: 256 rows per item, 256 features per gate/up item, 512
    // rows per down item.  FP8: 128 rows per item (the promoted sums live in
    // registers), 128 features per gate/up item, 256 rows per down item.
    p.pair = !p.fp8 && p.bn == 256 && H % 256 == 0 && Hs % 256 == 0 && d % 512 == 0 && n_sm >= 2;
    p.pair8 = p.fp8 && p.bn >= 128 && n_sm >= 2;
    if (p.pair8) p.bn = 128;
    else if (p.fp8 && p.bn > kFp8MaxBn) p.bn = kFp8MaxBn;
    p.router_parts = 1;
    if (c->act_dtype != MOE_F32 && c->n_experts <= 256) {
        p.router_parts = router_splits(T, n_sm);
        if (p.router_parts > d / 64) p.router_parts = d / 64;  // every split owns at least one K block
    }
    // a single CTA sorts decode-sized batches in one launch; large batches use many CTAs
    p.permute_multi = T > kPermuteMultiMinT;
    return p;
}

// Router logits on tensor cores (bf16 x) or CUDA cores (fp32 x), then selection.
moe_status route_impl(const moe_config* c, const DevInfo& di, const void* x, const void* w_router, float* logits,
                      const float* bias, int T, int32_t* idx, float* w, cudaStream_t s, float* part = nullptr,
                      int n_parts = 1) {
    if (!part) n_parts = 1;
    if (x) {
        if (c->act_dtype == MOE_F32) {
            n_parts = 1;
            cudaError_t e = launch_router_f32(static_cast<const float*>(x),
                                              static_cast<const __nv_bfloat16*>(w_router), T, c->d, c->n_experts,
                                              logits, s);
            if (e != cudaSuccess) return MOE_ERR_CUDA;
        } else {
            GemmArgs a;
            memset(&a, 0, sizeof(a));
            const int bn = router_bn(T);
            if (!map_bf16(&a.a0, w_router, c->n_experts, c->d, 128)) return MOE_ERR_CUDA;
            a.a1 = a.s0 = a.s1 = a.a0;
            if (!map_bf16(&a.b, x, T, c->d, kBoxRows)) return MOE_ERR_CUDA;
            a.item_off = nullptr;
            a.n_rows_single = T;
            a.K_routed = a.K_shared = c->d;
            a.mt_routed = (c->n_experts + 255) / 256;
            a.logits = logits;
            a.n_logit_cols = c->n_experts;
            a.k_splits = n_parts;
            a.part = part;
            const int items = a.mt_routed * ((T + bn - 1) / bn) * n_parts;
            const int grid = items < di.sm_count ? items : di.sm_count;
            if (launch_gemm(MODE_LOGITS, bn, &a, grid, s) != cudaSuccess) return MOE_ERR_CUDA;
        }
    }
    return cuda_status(launch_select(logits, bias, T, c->n_experts, c->n_groups, c->topk_groups, c->top_k, idx, w, s,
                                     part, n_parts));
}

size_t xhat_bytes(const moe_config* c, int T) { return ((size_t)T * c->d * 2 + 255) & ~(size_t)255; }

// The checks moe_forward makes before it enqueues anything (T == 0 passes).
moe_status check_forward_args(const moe_config* cfg, const moe_weights* wt, const void* x, const float* bias, int T,
                              const void* y, moe_dtype y_dtype, int accumulate, const void* workspace,
                              size_t ws_bytes) {
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (T < 0 || (y_dtype != MOE_F32 && y_dtype != MOE_BF16) || (accumulate != 0 && accumulate != 1))
        return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!wt || !x || !bias || !y || !workspace) return MOE_ERR_INVALID_ARG;
    if (!wt->w_router || !wt->w_gate || !wt->w_up || !wt->w_down) return MOE_ERR_INVALID_ARG;
    if (cfg->n_shared && (!wt->ws_gate || !wt->ws_up || !wt->ws_down)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y) || !aligned16(wt->w_router) || !aligned16(wt->w_gate) ||
        !aligned16(wt->w_up) || !aligned16(wt->w_down) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return MOE_ERR_INVALID_ARG;
    if (cfg->n_shared && (!aligned16(wt->ws_gate) || !aligned16(wt->ws_up) || !aligned16(wt->ws_down)))
        return MOE_ERR_INVALID_ARG;
    if (cfg->weight_dtype == MOE_E4M3) {
        if (cfg->act_dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
        if (!wt->s_gate || !wt->s_up || !wt->s_down) return MOE_ERR_INVALID_ARG;
        if (cfg->n_shared && (!wt->ss_gate || !wt->ss_up || !wt->ss_down)) return MOE_ERR_INVALID_ARG;
    }
    if (ws_bytes < layout(cfg, T, nullptr).bytes) return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

// The layer restricted to a block of n_local routed experts (expert parallelism):
// no selection (the routing is given), no shared expert, bf16 rows.
bool local_cfg(const moe_config* cfg, int n_local, moe_config* c) {
    if (check_config(cfg) != MOE_OK || n_local < 1 || n_local > cfg->n_experts) return false;
    *c = *cfg;
    c->n_experts = n_local;
    c->n_groups = 1;
    c->topk_groups = 1;
    c->n_shared = 0;
    c->shared_hidden = cfg->hidden;
    c->act_dtype = MOE_BF16;
    return true;
}
size_t dtype_bytes(moe_dtype t) { return t == MOE_F32 ? 4 : t == MOE_BF16 ? 2 : 1; }

moe_status forward_impl(const moe_config* cfg, const moe_weights* wt, const void* x, const float* bias, int T,
                        void* y, moe_dtype y_dtype, int accumulate, void* workspace, size_t ws_bytes,
                        moe_stream_t stream, const moe_stage_events* events, const moe_routing_out* routing,
                        const void* norm_g, float eps);
moe_status run_experts(const moe_config* cfg, const moe_weights* wt, const Workspace& W, const Plan& plan,
                       const DevInfo& di, int T, const void* x, bool act_quantised, void* y, moe_dtype y_dtype,
                       int accumulate, const void* residual, cudaStream_t s, const moe_stage_events* events,
                       int dn_splits);

}  // namespace

extern "C" {

int moe_abi_version(void) { return MOE_ABI_VERSION; }

int moe_debug_build(void) { return kDebugBuild ? 1 : 0; }

moe_status moe_debug_corrupt_next(int table, int index, int value) {
    if (table != -1 && table != MOE_DEBUG_TABLE_ROW_TOK && table != MOE_DEBUG_TABLE_ROW_OFF)
        return MOE_ERR_INVALID_ARG;
    if (!kDebugBuild) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> g(g_debug_mu);
    g_debug_corruption.table = table;
    g_debug_corruption.index = index;
    g_debug_corruption.value = value;
    return MOE_OK;
}

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
        case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    }
    return "MOE_ERR_UNKNOWN";
}

size_t moe_workspace_size(const moe_config* cfg, int T_max) {
    if (check_config(cfg) != MOE_OK || T_max < 0) return 0;
    return layout(cfg, T_max, nullptr).bytes;
}

moe_status moe_route(const moe_config* cfg, const void* x, const void* w_router, float* logits, const float* bias,
                     int T, int32_t* topk_idx, float* topk_w, moe_stream_t stream) {
    NvtxRange nvtx_call("moe_route");
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (T < 0) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!logits || !bias || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    if (x && (!w_router || !aligned16(x) || !aligned16(w_router))) return MOE_ERR_INVALID_ARG;
    DevInfo di;
    if ((st = check_device(&di)) != MOE_OK) return st;
    return route_impl(cfg, di, x, w_router, logits, bias, T, topk_idx, topk_w, (cudaStream_t)stream);
}

moe_status moe_quantize_act(const void* x, int T, int d, uint8_t* q, float* sx, moe_stream_t stream) {
    if (T < 0 || d <= 0 || d % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !q || !sx || (reinterpret_cast<uintptr_t>(x) & 7u) || (reinterpret_cast<uintptr_t>(q) & 3u))
        return MOE_ERR_INVALID_ARG;
    DevInfo di;
    moe_status st = check_device(&di);
    if (st != MOE_OK) return st;
    return cuda_status(launch_quant_act(static_cast<const __nv_bfloat16*>(x), T, d, q, sx, (cudaStream_t)stream));
}

unsigned long long moe_launch_count(void) { return launch_count(); }

moe_status moe_selftest_wait_timeout(unsigned long long limit_ns, moe_stream_t stream) {
    if (limit_ns == 0 || limit_ns > 1000000000ull) return MOE_ERR_INVALID_ARG;
    DevInfo di;
    moe_status st = check_device(&di);
    if (st != MOE_OK) return st;
    return cuda_status(launch_wait_selftest(limit_ns, (cudaStream_t)stream));
}

moe_status moe_forward_plan(const moe_config* cfg, int T, moe_dtype y_dtype, moe_plan* out) {
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (!out || T < 0 || (y_dtype != MOE_F32 && y_dtype != MOE_BF16)) return MOE_ERR_INVALID_ARG;
    DevInfo di;
    if ((st = check_device(&di)) != MOE_OK) return st;
    memset(out, 0, sizeof(*out));
    if (T == 0) return MOE_OK;
    const Plan p = make_plan(cfg, T, di.sm_count);
    out->token_tile = p.bn;
    out->cta_pair = (p.pair || p.pair8) ? 1 : 0;
    out->fp8 = p.fp8 ? 1 : 0;
    out->router_splits = p.router_parts;
    out->permute_ctas = p.permute_multi ? permute_blocks(T) : 1;
    // router + selection, permutation, copy into expert order (with the quantisation), two
    // GEMMs, bf16 cast
    out->launches = 2 + (p.permute_multi ? 3 : 1) + 1 + 2 + (y_dtype == MOE_BF16 ? 1 : 0);
    return MOE_OK;
}

moe_status moe_update_bias(const moe_config* cfg, const int32_t* counts, float* bias, float gamma,
                           moe_stream_t stream) {
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (!counts || !bias || !(gamma == gamma)) return MOE_ERR_INVALID_ARG;
    DevInfo di;
    if ((st = check_device(&di)) != MOE_OK) return st;
    return cuda_status(launch_update_bias(counts, cfg->n_experts, bias, gamma, (cudaStream_t)stream));
}

moe_status moe_permute(const moe_config* cfg, const int32_t* topk_idx, int T, int32_t* counts, int32_t* offsets,
                       int32_t* src, int32_t* inv, moe_stream_t stream) {
    NvtxRange nvtx_call("moe_permute");
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (T < 0) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!topk_idx || !counts || !offsets || !src || !inv) return MOE_ERR_INVALID_ARG;
    DevInfo di;
    if ((st = check_device(&di)) != MOE_OK) return st;
    PermuteArgs a;
    memset(&a, 0, sizeof(a));
    a.idx = topk_idx;
    a.T = T;
    a.k = cfg->top_k;
    a.E = cfg->n_experts;
    a.counts = counts;
    a.offsets = offsets;
    a.src = src;
    a.inv = inv;
    return cuda_status(launch_permute(a, (cudaStream_t)stream));
}

moe_status moe_forward(const moe_config* cfg, const moe_weights* wt, const void* x, const float* bias, int T,
                       void* y, moe_dtype y_dtype, int accumulate, void* workspace, size_t ws_bytes,
                       moe_stream_t stream) {
    return moe_forward_ex(cfg, wt, x, bias, T, y, y_dtype, accumulate, workspace, ws_bytes, stream, nullptr,
                          nullptr);
}

moe_status moe_forward_ex(const moe_config* cfg, const moe_weights* wt, const void* x, const float* bias, int T,
                          void* y, moe_dtype y_dtype, int accumulate, void* workspace, size_t ws_bytes,
                          moe_stream_t stream, const moe_stage_events* events, const moe_routing_out* routing) {
    NvtxRange nvtx_call("moe_forward");
    return forward_impl(cfg, wt, x, bias, T, y, y_dtype, accumulate, workspace, ws_bytes, stream, events, routing,
                        nullptr, 0.0f);
}

size_t moe_block_workspace_size(const moe_config* cfg, int T_max) {
    const size_t base = moe_workspace_size(cfg, T_max);
    return base ? base + xhat_bytes(cfg, T_max) : 0;
}

moe_status moe_rmsnorm(const void* h, const void* g, float eps, int T, int d, void* out, uint8_t* q, float* sx,
                       moe_stream_t stream) {
    if (T < 0 || d <= 0 || d % 8 || d > 8 * NORM_MAX_VEC * NORM_THREADS || !(eps >= 0.0f)) return MOE_ERR_INVALID_ARG;
    if ((q != nullptr) != (sx != nullptr) || (q && d % 128)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!h || !g || !out || !aligned16(h) || !aligned16(g) || !aligned16(out) || (q && (!aligned16(q) || !aligned16(sx))))
        return MOE_ERR_INVALID_ARG;
    DevInfo di;
    moe_status st = check_device(&di);
    if (st != MOE_OK) return st;
    return cuda_status(launch_rmsnorm(static_cast<const __nv_bfloat16*>(h), static_cast<const __nv_bfloat16*>(g), T,
                                      d, eps, static_cast<__nv_bfloat16*>(out), q, sx, (cudaStream_t)stream));
}

// The dense FFN runs as the layer's expert stages with no routed expert: one
// group of all T rows in the always-on slot (hidden = the dense width).
static moe_config dense_config(int d, int hidden, moe_dtype act_dtype, moe_dtype weight_dtype) {
    moe_config c;
    memset(&c, 0, sizeof(c));
    c.d = d;
    c.n_experts = 0;
    c.n_groups = 1;
    c.topk_groups = 1;
    c.top_k = 0;
    c.hidden = hidden;
    c.n_shared = 1;
    c.shared_hidden = hidden;
    c.routed_scale = 1.0f;
    c.act_dtype = act_dtype;
    c.weight_dtype = weight_dtype;
    return c;
}

static bool dense_shape_ok(int d, int hidden, moe_dtype act_dtype, moe_dtype weight_dtype) {
    if (d <= 0 || hidden <= 0 || d % 128 || hidden % 128) return false;
    if (act_dtype != MOE_F32 && act_dtype != MOE_BF16) return false;
    if (weight_dtype != MOE_BF16 && weight_dtype != MOE_E4M3) return false;
    return !(weight_dtype == MOE_E4M3 && act_dtype != MOE_BF16);
}

size_t moe_dense_workspace_size(int d, int hidden, moe_dtype act_dtype, moe_dtype weight_dtype, int T_max) {
    if (!dense_shape_ok(d, hidden, act_dtype, weight_dtype) || T_max < 0) return 0;
    const moe_config c = dense_config(d, hidden, act_dtype, weight_dtype);
    return layout(&c, T_max, nullptr).bytes;
}

moe_status moe_dense_ffn(int d, int hidden, moe_dtype act_dtype, moe_dtype weight_dtype, const void* w_gate,
                         const void* w_up, const void* w_down, const float* s_gate, const float* s_up,
                         const float* s_down, const void* x, int T, void* y, moe_dtype y_dtype, int accumulate,
                         void* workspace, size_t ws_bytes, moe_stream_t stream, const moe_stage_events* events) {
    NvtxRange nvtx_call("moe_dense_ffn");
    if (!dense_shape_ok(d, hidden, act_dtype, weight_dtype)) {
        const bool bad_shape = d <= 0 || hidden <= 0 || d % 128 || hidden % 128;
        return bad_shape ? MOE_ERR_INVALID_ARG : MOE_ERR_UNSUPPORTED;
    }
    if (T < 0 || (y_dtype != MOE_F32 && y_dtype != MOE_BF16) || (accumulate != 0 && accumulate != 1))
        return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    const bool fp8 = weight_dtype == MOE_E4M3;
    if (!w_gate || !w_up || !w_down || !x || !y || !workspace) return MOE_ERR_INVALID_ARG;
    if (fp8 && (!s_gate || !s_up || !s_down)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) || !aligned16(x) || !aligned16(y) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return MOE_ERR_INVALID_ARG;
    const moe_config c = dense_config(d, hidden, act_dtype, weight_dtype);
    if (ws_bytes < layout(&c, T, nullptr).bytes) return MOE_ERR_WORKSPACE;
    DevInfo di;
    moe_status st = check_device(&di);
    if (st != MOE_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    moe_weights w;
    memset(&w, 0, sizeof(w));
    w.ws_gate = w_gate;
    w.ws_up = w_up;
    w.ws_down = w_down;
    w.ss_gate = s_gate;
    w.ss_up = s_up;
    w.ss_down = s_down;
    const Workspace W = layout(&c, T, workspace);
    const Plan plan = make_plan(&c, T, di.sm_count);
    const int mt_gu = plan.pair ? hidden / 256 : hidden / 128;
    const int mt_dn = plan.pair ? d / 512 : (d + 255) / 256;
    // a few token chunks leave most SMs without a down tile (d / 512 = 14 pair tiles at
    // d = 7168): split the long K (= hidden) of the down GEMM so that one wave fills the
    // GPU; the splits add into y by the combine's atomics.  bf16 kernels only.
    int dn_splits = 1;
    if (!plan.fp8) {
        const int units = plan.pair ? di.sm_count / 2 : di.sm_count;
        const int tiles = ((T + plan.bn - 1) / plan.bn) * mt_dn;
        const int max_splits = hidden / 64 / 4;  // at least four 64-wide K blocks a split
        if (tiles < units) dn_splits = units / tiles;
        if (dn_splits > max_splits) dn_splits = max_splits;
        if (dn_splits < 1) dn_splits = 1;
    }
    for (int i = 0; i < 2; ++i)  // no router: the first two stage marks coincide
        if (events && events->ev[i]) cudaEventRecord((cudaEvent_t)events->ev[i], s);
    if (launch_dense_schedule(T, plan.bn, mt_gu, mt_dn * dn_splits, W.row_off, W.item_gu, W.item_dn, W.row_tok,
                              W.row_coef, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return run_experts(&c, &w, W, plan, di, T, x, false, y, y_dtype, accumulate, accumulate ? y : nullptr, s,
                       events, dn_splits);
}

moe_status moe_forward_block(const moe_config* cfg, const moe_weights* wt, const void* norm_g, float eps,
                             const void* h, const float* bias, int T, void* y, void* workspace, size_t ws_bytes,
                             moe_stream_t stream, const moe_stage_events* events, const moe_routing_out* routing) {
    NvtxRange nvtx_call("moe_forward_block");
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (cfg->act_dtype != MOE_BF16 || cfg->d > 8 * NORM_MAX_VEC * NORM_THREADS) return MOE_ERR_UNSUPPORTED;
    if (T < 0 || !(eps >= 0.0f)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!norm_g || !aligned16(norm_g)) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_block_workspace_size(cfg, T)) return MOE_ERR_WORKSPACE;
    return forward_impl(cfg, wt, h, bias, T, y, MOE_BF16, 0, workspace, ws_bytes, stream, events, routing, norm_g, eps);
}

size_t moe_host_workspace_size(const moe_config* cfg, int T_max, moe_dtype y_dtype) {
    if (y_dtype != MOE_F32 && y_dtype != MOE_BF16) return 0;
    const size_t base = moe_workspace_size(cfg, T_max);
    if (!base) return 0;
    const size_t n = (size_t)T_max * cfg->d;
    return round256(base) + round256(n * dtype_bytes(cfg->act_dtype)) + round256(n * dtype_bytes(y_dtype));
}

moe_status moe_forward_host(const moe_config* cfg, const moe_weights* wt, const void* x_host, const float* bias,
                            int T, void* y_host, moe_dtype y_dtype, int accumulate, void* workspace, size_t ws_bytes,
                            moe_stream_t stream) {
    NvtxRange nvtx_call("moe_forward_host");
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (T < 0 || (y_dtype != MOE_F32 && y_dtype != MOE_BF16)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return check_forward_args(cfg, wt, x_host, bias, 0, y_host, y_dtype, accumulate, workspace, ws_bytes);
    if (!x_host || !y_host || !workspace) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_host_workspace_size(cfg, T, y_dtype)) return MOE_ERR_WORKSPACE;
    // the device copies of x and y sit behind the layer's own workspace
    const size_t fw = round256(moe_workspace_size(cfg, T));
    const size_t xb = (size_t)T * cfg->d * dtype_bytes(cfg->act_dtype);
    const size_t yb = (size_t)T * cfg->d * dtype_bytes(y_dtype);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    void* xd = ws + fw;
    void* yd = ws + fw + round256(xb);
    if ((st = check_forward_args(cfg, wt, xd, bias, T, yd, y_dtype, accumulate, ws, fw)) != MOE_OK) return st;
    DevInfo di;
    if ((st = check_device(&di)) != MOE_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(xd, x_host, xb, cudaMemcpyHostToDevice, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (accumulate && cudaMemcpyAsync(yd, y_host, yb, cudaMemcpyHostToDevice, s) != cudaSuccess) return MOE_ERR_CUDA;
    st = forward_impl(cfg, wt, xd, bias, T, yd, y_dtype, accumulate, ws, fw, stream, nullptr, nullptr, nullptr, 0.0f);
    if (st != MOE_OK) return st;
    return cudaMemcpyAsync(y_host, yd, yb, cudaMemcpyDeviceToHost, s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_ep_max_send_rows(const moe_config* cfg, int T, int n_ranks) {
    if (check_config(cfg) != MOE_OK || T < 0 || n_ranks < 1) return 0;
    return T * (cfg->top_k < n_ranks ? cfg->top_k : n_ranks);
}

moe_status moe_ep_dispatch(const moe_config* cfg, int n_ranks, const int32_t* topk_idx, const float* topk_w,
                           const void* x, int T, int32_t* send_counts, int32_t* send_offsets, int32_t* send_tok,
                           void* send_x, int32_t* send_idx, float* send_w, moe_stream_t stream) {
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (T < 0 || n_ranks < 1 || n_ranks > 32 || cfg->n_experts % n_ranks != 0) return MOE_ERR_INVALID_ARG;
    if (!send_counts || !send_offsets) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!topk_idx || !topk_w || !x || !send_tok || !send_x || !send_idx || !send_w || !aligned16(x) ||
                  !aligned16(send_x)))
        return MOE_ERR_INVALID_ARG;
    DevInfo di;
    if ((st = check_device(&di)) != MOE_OK) return st;
    return cuda_status(launch_ep_dispatch(topk_idx, topk_w, T, cfg->top_k, cfg->n_experts, n_ranks, x,
                                          cfg->act_dtype == MOE_F32, cfg->d, send_counts, send_offsets, send_tok,
                                          static_cast<__nv_bfloat16*>(send_x), send_idx, send_w, di.sm_count,
                                          (cudaStream_t)stream));
}

size_t moe_ep_packed_row_bytes(const moe_config* cfg) {
    if (check_config(cfg) != MOE_OK) return 0;
    return align_up((size_t)cfg->d * 2 + (size_t)cfg->top_k * 8, 16);
}

moe_status moe_ep_dispatch_packed(const moe_config* cfg, int n_ranks, int capacity, const int32_t* topk_idx,
                                  const float* topk_w, const void* x, int T, int32_t* send_counts, int32_t* send_tok,
                                  void* packed, moe_stream_t stream) {
    NvtxRange nvtx_call("moe_ep_dispatch_packed");
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (T < 0 || capacity < T || capacity < 1 || n_ranks < 1 || n_ranks > 32 || cfg->n_experts % n_ranks != 0 ||
        (long long)n_ranks * capacity > INT32_MAX)
        return MOE_ERR_INVALID_ARG;
    if (!send_counts || !send_tok || !packed || !aligned16(packed)) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!topk_idx || !topk_w || !x || !aligned16(x))) return MOE_ERR_INVALID_ARG;
    DevInfo di;
    if ((st = check_device(&di)) != MOE_OK) return st;
    return cuda_status(launch_ep_dispatch_packed(topk_idx, topk_w, T, cfg->top_k, cfg->n_experts, n_ranks, capacity,
                                                 x, cfg->act_dtype == MOE_F32, cfg->d, send_counts, send_tok,
                                                 static_cast<uint8_t*>(packed), (int)moe_ep_packed_row_bytes(cfg),
                                                 (cudaStream_t)stream));
}

moe_status moe_ep_dispatch_peer(const moe_config* cfg, int n_ranks, int capacity, int my_rank, const int32_t* topk_idx,
                                const float* topk_w, const void* x, int T, int32_t* send_counts, int32_t* send_tok,
                                void* const* recv_bufs, moe_stream_t stream) {
    NvtxRange nvtx_call("moe_ep_dispatch_peer");
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (T < 0 || capacity < T || capacity < 1 || n_ranks < 1 || n_ranks > 32 || cfg->n_experts % n_ranks != 0 ||
        my_rank < 0 || my_rank >= n_ranks || (long long)n_ranks * capacity > INT32_MAX)
        return MOE_ERR_INVALID_ARG;
    if (!send_counts || !send_tok || !recv_bufs || (reinterpret_cast<uintptr_t>(recv_bufs) & 7u))
        return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!topk_idx || !topk_w || !x || !aligned16(x))) return MOE_ERR_INVALID_ARG;
    DevInfo di;
    if ((st = check_device(&di)) != MOE_OK) return st;
    return cuda_status(launch_ep_dispatch_packed(
        topk_idx, topk_w, T, cfg->top_k, cfg->n_experts, n_ranks, capacity, x, cfg->act_dtype == MOE_F32, cfg->d,
        send_counts, send_tok, nullptr, (int)moe_ep_packed_row_bytes(cfg), (cudaStream_t)stream,
        reinterpret_cast<uint8_t* const*>(recv_bufs), my_rank * capacity));
}

moe_status moe_ep_unpack(const moe_config* cfg, int n_rows, const void* packed, void* x_rows, int32_t* topk_idx,
                         float* topk_w, moe_stream_t stream) {
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (n_rows < 0) return MOE_ERR_INVALID_ARG;
    if (n_rows == 0) return MOE_OK;
    if (!packed || !x_rows || !topk_idx || !topk_w || !aligned16(packed) || !aligned16(x_rows))
        return MOE_ERR_INVALID_ARG;
    DevInfo di;
    if ((st = check_device(&di)) != MOE_OK) return st;
    return cuda_status(launch_ep_unpack(static_cast<const uint8_t*>(packed), n_rows, (int)moe_ep_packed_row_bytes(cfg),
                                        cfg->d, cfg->top_k, static_cast<__nv_bfloat16*>(x_rows), topk_idx, topk_w,
                                        (cudaStream_t)stream));
}

size_t moe_experts_routed_workspace_size(const moe_config* cfg, int n_local, int n_rows_max) {
    moe_config c;
    if (!local_cfg(cfg, n_local, &c) || n_rows_max < 0) return 0;
    return layout(&c, n_rows_max, nullptr).bytes;
}

moe_status moe_experts_routed(const moe_config* cfg, const moe_weights* wl, int expert_lo, int n_local,
                              const void* x_rows, int n_rows, const int32_t* topk_idx, const float* topk_w,
                              float* y_rows, void* workspace, size_t ws_bytes, moe_stream_t stream) {
    moe_status st = check_config(cfg);
    if (st != MOE_OK) return st;
    moe_config c;
    if (!local_cfg(cfg, n_local, &c) || expert_lo < 0 || expert_lo > cfg->n_experts - n_local || n_rows < 0)
        return MOE_ERR_INVALID_ARG;
    if (n_rows == 0) return MOE_OK;
    if (!wl || !x_rows || !topk_idx || !topk_w || !y_rows || !workspace) return MOE_ERR_INVALID_ARG;
    if (!wl->w_gate || !wl->w_up || !wl->w_down || !aligned16(wl->w_gate) || !aligned16(wl->w_up) ||
        !aligned16(wl->w_down) || !aligned16(x_rows) || !aligned16(y_rows) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return MOE_ERR_INVALID_ARG;
    if (c.weight_dtype == MOE_E4M3 && (!wl->s_gate || !wl->s_up || !wl->s_down)) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < layout(&c, n_rows, nullptr).bytes) return MOE_ERR_WORKSPACE;
    DevInfo di;
    if ((st = check_device(&di)) != MOE_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const Workspace W = layout(&c, n_rows, workspace);
    const Plan plan = make_plan(&c, n_rows, di.sm_count);
    const int H = c.hidden, d = c.d;
    // the permutation of the rows' slots of this block (other blocks' slots skipped) and the tile schedules
    PermuteArgs pa;
    memset(&pa, 0, sizeof(pa));
    pa.idx = topk_idx;
    pa.T = n_rows;
    pa.k = c.top_k;
    pa.E = n_local;
    pa.id_lo = expert_lo;
    pa.foreign_ok = 1;
    pa.counts = W.counts;
    pa.offsets = W.offsets;
    pa.src = W.src;
    pa.inv = W.inv;
    pa.topk_w = topk_w;
    pa.routed_scale = c.routed_scale;
    pa.n_shared = 0;
    pa.row_tok = W.row_tok;
    pa.row_coef = W.row_coef;
    pa.row_off = W.row_off;
    pa.item_off_gu = W.item_gu;
    pa.item_off_dn = W.item_dn;
    pa.bn_gu = pa.bn_dn = plan.bn;
    pa.mt_gu_routed = pa.mt_gu_shared = plan.pair ? H / 256 : H / 128;
    pa.mt_dn = plan.pair ? d / 512 : (d + 255) / 256;
    const cudaError_t ep = plan.permute_multi ? launch_permute_multi(pa, W.hist, s) : launch_permute(pa, s);
    if (ep != cudaSuccess) return MOE_ERR_CUDA;
    return run_experts(&c, wl, W, plan, di, n_rows, x_rows, false, y_rows, MOE_F32, 0, nullptr, s, nullptr, 1);
}

moe_status moe_ep_combine(int T, int d, int n_rows, const float* back_rows, const int32_t* send_tok, float* y_acc,
                          void* y, const void* residual, moe_stream_t stream) {
    if (T < 0 || d <= 0 || d % 8 != 0 || n_rows < 0) return MOE_ERR_INVALID_ARG;
    if (T == 0) return n_rows == 0 ? MOE_OK : MOE_ERR_INVALID_ARG;
    if (!y_acc || !aligned16(y_acc) || (n_rows > 0 && (!back_rows || !send_tok || !aligned16(back_rows))) ||
        (y && !aligned16(y)) || (residual && !aligned16(residual)))
        return MOE_ERR_INVALID_ARG;
    DevInfo di;
    moe_status st = check_device(&di);
    if (st != MOE_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    if (launch_ep_combine(back_rows, send_tok, n_rows, T, d, y_acc, di.sm_count, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (y && launch_finalize_bf16(y_acc, static_cast<const __nv_bfloat16*>(residual), static_cast<__nv_bfloat16*>(y),
                                  (size_t)T * d, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

moe_status moe_ep_combine_peer(int T, int d, int n_ranks, int capacity, int my_rank, const float* const* result_bufs,
                               const int32_t* send_tok, float* y_acc, void* y, const void* residual,
                               moe_stream_t stream) {
    if (T < 0 || d <= 0 || d % 8 != 0 || n_ranks < 1 || n_ranks > 32 || capacity < 1 || capacity < T ||
        my_rank < 0 || my_rank >= n_ranks || (long long)n_ranks * capacity > INT32_MAX)
        return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!y_acc || !aligned16(y_acc) || !send_tok || !result_bufs || (reinterpret_cast<uintptr_t>(result_bufs) & 7u) ||
        (y && !aligned16(y)) || (residual && !aligned16(residual)))
        return MOE_ERR_INVALID_ARG;
    DevInfo di;
    moe_status st = check_device(&di);
    if (st != MOE_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    if (launch_ep_combine(nullptr, send_tok, n_ranks * capacity, T, d, y_acc, di.sm_count, s, result_bufs, capacity,
                          my_rank * capacity) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (y && launch_finalize_bf16(y_acc, static_cast<const __nv_bfloat16*>(residual), static_cast<__nv_bfloat16*>(y),
                                  (size_t)T * d, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

}  // extern "C"

namespace {

// Stages (3b)-(5) of the layer on tables the caller has built: the gather of
// the activations in group order (FP8: quantised first unless act_quantised),
// the gate/up and down grouped GEMMs, the combine and the output cast.  Used by
// the MoE forward (groups = routed experts + the shared one) and by the dense
// FFN (one group of all T rows in the shared-expert slot, n_experts = 0).
moe_status run_experts(const moe_config* cfg, const moe_weights* wt, const Workspace& W, const Plan& plan,
                       const DevInfo& di, int T, const void* x, bool act_quantised, void* y, moe_dtype y_dtype,
                       int accumulate, const void* residual, cudaStream_t s, const moe_stage_events* events,
                       int dn_splits) {
    const bool fp8 = cfg->weight_dtype == MOE_E4M3;
    const int E = cfg->n_experts, k = cfg->top_k, d = cfg->d, H = cfg->hidden;
    const int Hs = cfg->n_shared ? cfg->shared_hidden : H;
    const int NG = E + cfg->n_shared;
    const int rows_max = T * k + cfg->n_shared * T;
    const int ldh = H > Hs ? H : Hs;
    const int bn = plan.bn;
    const bool pair = plan.pair, pair8 = plan.pair8;
    const int box_rows = (pair || pair8) ? kPairBoxRows : kBoxRows;
    const int mt_dn = pair ? d / 512 : (d + 255) / 256;
    auto mark = [&](int i) {
        if (events && events->ev[i]) cudaEventRecord((cudaEvent_t)events->ev[i], s);
    };
    // one group of all T rows in token order (the dense FFN) with bf16 x: the token
    // operand is x itself, no gathered copy
    const bool direct_b = E == 0 && !fp8 && cfg->act_dtype == MOE_BF16;
    NvtxStages nv;
    nv.next(fp8 ? "moe.quantize+gather" : "moe.gather");
    if (fp8) {
        if (launch_quant_scatter_fp8(act_quantised ? nullptr : static_cast<const __nv_bfloat16*>(x),
                                     act_quantised ? W.x_q : nullptr, W.sx, d, T, k, W.inv,
                                     cfg->n_shared ? W.row_off + E : nullptr, rows_max, W.xq_perm, W.sxT, di.sm_count,
                                     s) != cudaSuccess)
            return MOE_ERR_CUDA;
    } else if (!direct_b && launch_scatter_rows(x, cfg->act_dtype == MOE_F32, d, T, k, W.inv,
                                                cfg->n_shared ? W.row_off + E : nullptr, rows_max, W.x_perm,
                                                di.sm_count, s) != cudaSuccess) {
        return MOE_ERR_CUDA;
    }
    mark(2);

    // (4) gate/up grouped GEMM with the SwiGLU epilogue -> h_perm
    nv.next("moe.gate_up");
    auto wmap = [&](CUtensorMap* m, const void* p, uint64_t rows, uint64_t cols, uint32_t box_rows) {
        return fp8 ? map_u8(m, p, rows, cols, box_rows) : map_bf16(m, p, rows, cols, box_rows);
    };
    GemmArgs g;
    memset(&g, 0, sizeof(g));
    // weight rows per TMA box: the FP8 pair kernel stacks 64 gate over 64 up rows per CTA
    const uint32_t gu_box = pair8 ? 64 : 128;
    if (E && (!wmap(&g.a0, wt->w_gate, (uint64_t)E * H, d, gu_box) ||
              !wmap(&g.a1, wt->w_up, (uint64_t)E * H, d, gu_box)))
        return MOE_ERR_CUDA;
    if (cfg->n_shared) {
        if (!wmap(&g.s0, wt->ws_gate, Hs, d, gu_box) || !wmap(&g.s1, wt->ws_up, Hs, d, gu_box)) return MOE_ERR_CUDA;
        if (!E) {
            g.a0 = g.s0;
            g.a1 = g.s1;
        }
    } else {
        g.s0 = g.a0;
        g.s1 = g.a1;
    }
    if (!(fp8 ? map_u8(&g.b, W.xq_perm, rows_max, d, box_rows)
              : map_bf16(&g.b, direct_b ? x : W.x_perm, rows_max, d, box_rows)))
        return MOE_ERR_CUDA;
    g.item_off = W.item_gu;
    g.row_off = W.row_off;
    g.rows_cap = rows_max;
    g.chunk_major = pair ? 1 : 0;  // the bf16 CTA-pair kernels
    g.n_groups = NG;
    g.n_routed = E;
    g.K_routed = g.K_shared = d;
    g.mt_routed = pair ? H / 256 : H / 128;
    g.mt_shared = pair ? Hs / 256 : Hs / 128;
    g.rows_per_expert = H;
    g.h = W.h_perm;
    g.ldh = ldh;
    if (fp8) {
        g.sa0 = E ? wt->s_gate : wt->ss_gate;
        g.sa1 = E ? wt->s_up : wt->ss_up;
        g.ss0 = cfg->n_shared ? wt->ss_gate : wt->s_gate;
        g.ss1 = cfg->n_shared ? wt->ss_up : wt->s_up;
        g.a_rb_routed = H / 128;
        g.a_rb_shared = Hs / 128;
        g.sbT = W.sxT;
        g.sb_ld = rows_max;
        g.hq = W.hq;
        g.hsT = W.shT;
        g.hs_ld = rows_max;
    }
    const cudaError_t egu = pair8  ? launch_gemm2_fp8(MODE_GATEUP, &g, di.sm_count, s)
                            : fp8  ? launch_gemm_fp8(MODE_GATEUP, bn, &g, di.sm_count, s)
                            : pair ? launch_gemm2(MODE_GATEUP, &g, di.sm_count, s)
                                   : launch_gemm(MODE_GATEUP, bn, &g, di.sm_count, s);
    if (egu != cudaSuccess) return MOE_ERR_CUDA;
    mark(3);

    // (5) down GEMM, routing-weight scale and un-permute scatter into fp32
    nv.next("moe.down+combine");
    float* yacc = y_dtype == MOE_F32 ? static_cast<float*>(y) : W.y_acc;
    if ((y_dtype == MOE_BF16 || !accumulate) &&
        cudaMemsetAsync(yacc, 0, (size_t)T * d * sizeof(float), s) != cudaSuccess)
        return MOE_ERR_CUDA;
    GemmArgs dn;
    memset(&dn, 0, sizeof(dn));
    if (E && !wmap(&dn.a0, wt->w_down, (uint64_t)E * d, H, 128)) return MOE_ERR_CUDA;
    if (cfg->n_shared) {
        if (!wmap(&dn.s0, wt->ws_down, d, Hs, 128)) return MOE_ERR_CUDA;
        if (!E) dn.a0 = dn.s0;
    } else {
        dn.s0 = dn.a0;
    }
    dn.a1 = dn.a0;
    dn.s1 = dn.s0;
    if (!(fp8 ? map_u8(&dn.b, W.hq, rows_max, ldh, box_rows) : map_bf16(&dn.b, W.h_perm, rows_max, ldh, box_rows)))
        return MOE_ERR_CUDA;
    dn.item_off = W.item_dn;
    dn.row_off = W.row_off;
    dn.rows_cap = rows_max;
    dn.chunk_major = pair ? 1 : 0;
    dn.y_rows = T;
    dn.n_groups = NG;
    dn.n_routed = E;
    dn.K_routed = H;
    dn.K_shared = Hs;
    dn.mt_routed = dn.mt_shared = mt_dn;
    dn.k_splits = dn_splits;  // bf16 kernels only: the tables count mt_dn * dn_splits tiles per chunk
    dn.rows_per_expert = d;
    dn.y = yacc;
    dn.row_coef = W.row_coef;
    dn.row_tok = W.row_tok;
    dn.ldy = d;
    if (fp8) {
        dn.sa0 = dn.sa1 = E ? wt->s_down : wt->ss_down;
        dn.ss0 = dn.ss1 = cfg->n_shared ? wt->ss_down : wt->s_down;
        dn.a_rb_routed = dn.a_rb_shared = d / 128;
        dn.sbT = W.shT;
        dn.sb_ld = rows_max;
    }
    const cudaError_t edn = pair8  ? launch_gemm2_fp8(MODE_DOWN, &dn, di.sm_count, s)
                            : fp8  ? launch_gemm_fp8(MODE_DOWN, bn, &dn, di.sm_count, s)
                            : pair ? launch_gemm2(MODE_DOWN, &dn, di.sm_count, s)
                                   : launch_gemm(MODE_DOWN, bn, &dn, di.sm_count, s);
    if (edn != cudaSuccess) return MOE_ERR_CUDA;
    mark(4);

    nv.next("moe.cast");
    if (y_dtype == MOE_BF16 &&
        launch_finalize_bf16(W.y_acc, static_cast<const __nv_bfloat16*>(residual), static_cast<__nv_bfloat16*>(y),
                             (size_t)T * d, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    mark(5);
    return MOE_OK;
}

// Applies (and disarms) an armed corruption to this call's tables, on the stream,
// after the permutation has written them.  An index outside the table does nothing.
cudaError_t apply_debug_corruption(const Workspace& W, int rows_max, int n_groups, cudaStream_t s) {
    if (!kDebugBuild) return cudaSuccess;
    DebugCorruption c;
    {
        std::lock_guard<std::mutex> g(g_debug_mu);
        c = g_debug_corruption;
        g_debug_corruption.table = -1;
    }
    int32_t* base = nullptr;
    int n = 0;
    if (c.table == MOE_DEBUG_TABLE_ROW_TOK) {
        base = W.row_tok;
        n = rows_max;
    } else if (c.table == MOE_DEBUG_TABLE_ROW_OFF) {
        base = W.row_off;
        n = n_groups + 1;
    }
    if (!base || c.index < 0 || c.index >= n) return cudaSuccess;
    return launch_debug_poke(base + c.index, c.value, s);
}

moe_status forward_impl(const moe_config* cfg, const moe_weights* wt, const void* x, const float* bias, int T,
                        void* y, moe_dtype y_dtype, int accumulate, void* workspace, size_t ws_bytes,
                        moe_stream_t stream, const moe_stage_events* events, const moe_routing_out* routing,
                        const void* norm_g, float eps) {
    moe_status st = check_forward_args(cfg, wt, x, bias, T, y, y_dtype, accumulate, workspace, ws_bytes);
    if (st != MOE_OK || T == 0) return st;
    const bool fp8 = cfg->weight_dtype == MOE_E4M3;
    DevInfo di;
    if ((st = check_device(&di)) != MOE_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;

    Workspace W = layout(cfg, T, workspace);
    if (routing) {
        if ((routing->logits && (reinterpret_cast<uintptr_t>(routing->logits) & 3u)) ||
            (routing->topk_idx && (reinterpret_cast<uintptr_t>(routing->topk_idx) & 3u)) ||
            (routing->topk_w && (reinterpret_cast<uintptr_t>(routing->topk_w) & 3u)))
            return MOE_ERR_INVALID_ARG;
        // the layer routes through the caller's buffers instead of the workspace
        if (routing->logits) W.logits = routing->logits;
        if (routing->topk_idx) W.idx = routing->topk_idx;
        if (routing->topk_w) W.w = routing->topk_w;
        if ((routing->counts && (reinterpret_cast<uintptr_t>(routing->counts) & 3u)) ||
            (routing->offsets && (reinterpret_cast<uintptr_t>(routing->offsets) & 3u)) ||
            (routing->src && (reinterpret_cast<uintptr_t>(routing->src) & 3u)) ||
            (routing->inv && (reinterpret_cast<uintptr_t>(routing->inv) & 3u)))
            return MOE_ERR_INVALID_ARG;
        if (routing->counts) W.counts = routing->counts;
        if (routing->offsets) W.offsets = routing->offsets;
        if (routing->src) W.src = routing->src;
        if (routing->inv) W.inv = routing->inv;
    }
    const int E = cfg->n_experts, k = cfg->top_k, d = cfg->d, H = cfg->hidden;
    const int Hs = cfg->n_shared ? cfg->shared_hidden : H;
    const Plan plan = make_plan(cfg, T, di.sm_count);
    const int bn = plan.bn;
    const bool pair = plan.pair;

    auto mark = [&](int i) {
        if (events && events->ev[i]) cudaEventRecord((cudaEvent_t)events->ev[i], s);
    };
    NvtxStages nv;
    // (0) pre-norm of the sublayer: the layer runs on x = RMSNorm(h) and adds h back at
    //     the end; in the FP8 layer the same pass writes the activation codes and scales
    mark(0);
    const void* residual = accumulate ? y : nullptr;
    if (norm_g) {
        nv.next("moe.rmsnorm");
        __nv_bfloat16* xhat = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(workspace) + W.bytes);
        if (launch_rmsnorm(static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(norm_g), T, d,
                           eps, xhat, fp8 ? W.x_q : nullptr, fp8 ? W.sx : nullptr, s) != cudaSuccess)
            return MOE_ERR_CUDA;
        residual = x;
        x = xhat;
    }
    // (1)+(2) router and selection
    nv.next("moe.route");
    st = route_impl(cfg, di, x, wt->w_router, W.logits, bias, T, W.idx, W.w, s, W.part, plan.router_parts);
    if (st != MOE_OK) return st;
    mark(1);

    // (3) permutation + tile schedules
    nv.next("moe.permute");
    PermuteArgs pa;
    memset(&pa, 0, sizeof(pa));
    pa.idx = W.idx;
    pa.T = T;
    pa.k = k;
    pa.E = E;
    pa.counts = W.counts;
    pa.offsets = W.offsets;
    pa.src = W.src;
    pa.inv = W.inv;
    pa.topk_w = W.w;
    pa.routed_scale = cfg->routed_scale;
    pa.n_shared = cfg->n_shared;
    pa.row_tok = W.row_tok;
    pa.row_coef = W.row_coef;
    pa.row_off = W.row_off;
    pa.item_off_gu = W.item_gu;
    pa.item_off_dn = W.item_dn;
    pa.bn_gu = pa.bn_dn = bn;
    pa.mt_gu_routed = pair ? H / 256 : H / 128;
    pa.mt_gu_shared = pair ? Hs / 256 : Hs / 128;
    pa.mt_dn = pair ? d / 512 : (d + 255) / 256;  // pair8: 256 down rows per item, as the 1-CTA kernels
    const cudaError_t ep = plan.permute_multi ? launch_permute_multi(pa, W.hist, s) : launch_permute(pa, s);
    if (ep != cudaSuccess) return MOE_ERR_CUDA;
    if (apply_debug_corruption(W, T * k + cfg->n_shared * T, E + cfg->n_shared, s) != cudaSuccess) return MOE_ERR_CUDA;
    return run_experts(cfg, wt, W, plan, di, T, x, norm_g != nullptr, y, y_dtype, accumulate, residual, s, events, 1);
}

}  // namespace

extern "C" {

moe_status moe_device_error(unsigned int* flags, moe_stream_t stream) {
    if (!flags) return MOE_ERR_INVALID_ARG;
    DevInfo di;
    moe_status st = check_device(&di);
    if (st != MOE_OK) return st;
    if (read_clear_dev_error(flags, (cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
    return *flags ? MOE_ERR_DEVICE : MOE_OK;
}

}  // extern "C"
