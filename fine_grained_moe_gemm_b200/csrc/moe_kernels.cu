// Kernels of the MoE layer forward pass (sm_100a) and their launchers.
//
//   router_f32_kernel     fp32-activation router logits (CUDA cores)
//   select_kernel         sigmoid, selection bias, group-limited top-k, weights
//   permute_kernel        histogram / prefix sum / stable scatter by expert, and
//                         the tile schedules of the grouped GEMMs (one CTA);
//   permute_count/scan/scatter_kernel   the same over many CTAs (large T)
//   scatter_rows_kernel   x_perm written token-major (bf16)
//   gather_rows_kernel    rows of x by a token table (bf16; the expert-parallel send rows)
//   quant_act_kernel      1x128 e4m3 activation quantisation
//   quant_scatter_fp8_kernel  the quantisation and the copy into expert order, token-major
//   moe_gemm_kernel       tcgen05 grouped GEMM, one CTA per tile (moe_gemm.cuh)
//   moe_gemm_fp8_kernel   the same for e4m3 with block scales (moe_gemm_fp8.cuh)
//   moe_gemm2_kernel      CTA-pair grouped GEMM, cta_group::2 (moe_gemm2.cuh)
//   moe_gemm2_fp8_kernel  CTA-pair e4m3 GEMM (moe_gemm2_fp8.cuh)
//   update_bias_kernel    selection-bias controller step
//   rmsnorm_kernel        pre-norm of the sublayer (+ the 1x128 e4m3 quantisation)
//   dense_schedule_kernel the one-group tables of the dense FFN
//   finalize_kernel       fp32 combine buffer -> bf16 output (+ residual)
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>

#include "moe_device.cuh"
#include "moe_gemm.cuh"
#include "moe_gemm_fp8.cuh"
#include "moe_gemm2.cuh"
#include "moe_gemm2_fp8.cuh"
#include "moe_launch.h"

namespace moe {

// Kernels launched by this library in this process (all devices and streams).
static std::atomic<unsigned long long> g_launch_count{0};
static inline void note_launch() { g_launch_count.fetch_add(1, std::memory_order_relaxed); }
unsigned long long launch_count() { return g_launch_count.load(std::memory_order_relaxed); }

// ============================================================================ router (fp32 x)
// logits[t, e] = sum_c x[t, c] * Wr[e, c], fp32 products and fp32 sums
// ("MoE router" box: gate(x.float())).  One block per token, one warp per
// expert at a time, lanes stride over c, then a butterfly sum.
__global__ void __launch_bounds__(256) router_f32_kernel(const float* __restrict__ x,
                                                         const __nv_bfloat16* __restrict__ wr, int T, int d, int E,
                                                         float* __restrict__ logits) {
    const int t = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float* xr = x + (size_t)t * d;
    for (int e = warp; e < E; e += 8) {
        const __nv_bfloat16* w = wr + (size_t)e * d;
        float acc = 0.0f;
        for (int c = lane; c < d; c += 32) acc = fmaf(xr[c], __bfloat162float(w[c]), acc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) logits[(size_t)t * E + e] = acc;
    }
}

// ============================================================================ selection
// Field guide cutaway 02 / "MoE router" box, one warp per token:
//   s = sigmoid_spec(l); b = s + bias (selection only; -0 ranks as +0)
//   group score = b(1) + b(2), the two strongest b of the group
//   the topk_groups best groups are eligible
//   slot j = the j-th best eligible expert by b
//   w[j] = s[idx[j]] / S, S = sum of the selected s in ascending expert index
// "a ranks before b": larger value, then lower index.
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
    return va > vb || (va == vb && ia < ib);
}

__device__ __forceinline__ void warp_best(float& v, int& id) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        float ov = __shfl_xor_sync(0xffffffffu, v, o);
        int oi = __shfl_xor_sync(0xffffffffu, id, o);
        if (ranks_before(ov, oi, v, id)) {
            v = ov;
            id = oi;
        }
    }
}

constexpr int SELECT_THREADS = 256;
constexpr int MAX_ROUTER_SPLITS = 16;

// tpb tokens per CTA (1 at small T, where latency rules, else up to 8): all
// threads sum the router's K-split partials (each expert's in split order) and
// apply sigmoid and bias into shared memory; then warp w takes the decisions
// of token w.
__global__ void __launch_bounds__(SELECT_THREADS) select_kernel(float* __restrict__ logits,
                                                                const float* __restrict__ bias, int T, int E,
                                                                int G, int topk_groups, int k,
                                                                int32_t* __restrict__ idx_out,
                                                                float* __restrict__ w_out,
                                                                const float* __restrict__ parts, int n_parts,
                                                                int tpb) {
    extern __shared__ float ssm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * tpb;
    for (int i = threadIdx.x; i < tpb * E; i += SELECT_THREADS) {
        const int tl = i / E, e = i - tl * E;
        const int t = t0 + tl;
        if (t >= T) break;  // i only grows
        float* l = logits + (size_t)t * E;
        float lv;
        if (parts) {
            // split-K router: the partial logits summed in split order, stored as the logits
            float pv[MAX_ROUTER_SPLITS];
#pragma unroll
            for (int p = 0; p < MAX_ROUTER_SPLITS; ++p)
                pv[p] = p < n_parts ? parts[((size_t)p * T + t) * E + e] : 0.0f;
            lv = pv[0];
#pragma unroll
            for (int p = 1; p < MAX_ROUTER_SPLITS; ++p)
                if (p < n_parts) lv = __fadd_rn(lv, pv[p]);
            l[e] = lv;
        } else {
            lv = l[e];
        }
        float sv = sigmoid_spec(lv);
        float bv = __fadd_rn(sv, bias[e]);
        if (bv == 0.0f) bv = 0.0f;
        if (!isfinite(lv) || bv != bv) {
            // logits must be finite: flag it, and let a NaN rank last so every
            // decision below still picks valid ids
            set_dev_error(MOE_DEVERR_NONFINITE);
            if (bv != bv) bv = -INFINITY;
        }
        ssm[(size_t)tl * 2 * E + e] = sv;
        ssm[(size_t)tl * 2 * E + E + e] = bv;
    }
    __syncthreads();
    const int t = t0 + warp;
    if (warp >= tpb || t >= T) return;  // uniform per warp
    float* s = ssm + (size_t)warp * 2 * E;
    float* b = s + E;
    const int gs = E / G;
    // group scores (lane g owns group g)
    float gsc = -INFINITY;
    if (lane < G) {
        int i1 = -1, i2 = -1;
        for (int e = lane * gs; e < (lane + 1) * gs; ++e) {
            if (i1 < 0 || ranks_before(b[e], e, b[i1], i1)) {
                i2 = i1;
                i1 = e;
            } else if (i2 < 0 || ranks_before(b[e], e, b[i2], i2)) {
                i2 = e;
            }
        }
        gsc = __fadd_rn(b[i1], b[i2]);
        if (gsc == 0.0f) gsc = 0.0f;
        if (gsc != gsc) gsc = -INFINITY;
    }
    unsigned gmask = 0;
    for (int r = 0; r < topk_groups; ++r) {
        // non-candidates carry id G: any candidate, even at -inf, ranks before them
        bool cand = lane < G && !((gmask >> lane) & 1u);
        float v = cand ? gsc : -INFINITY;
        int id = cand ? lane : G;
        warp_best(v, id);
        if (id < G) gmask |= 1u << id;
    }
    // experts: lane owns e = lane + 32 i
    unsigned taken = 0;
    int my_idx = -1;
    for (int j = 0; j < k; ++j) {
        float v = -INFINITY;
        int id = 0x7fffffff;
        for (int i = 0, e = lane; e < E; ++i, e += 32) {
            if (((gmask >> (e / gs)) & 1u) && !((taken >> i) & 1u) && ranks_before(b[e], e, v, id)) {
                v = b[e];
                id = e;
            }
        }
        warp_best(v, id);
        if (id < E && (id & 31) == lane) taken |= 1u << (id >> 5);
        if (lane == j) my_idx = id < E ? id : 0;
    }
    // S over the selected experts in ascending expert index
    int rank = 0;
    for (int jj = 0; jj < k; ++jj) {
        int o = __shfl_sync(0xffffffffu, my_idx, jj);
        if (lane < k && o < my_idx) ++rank;
    }
    const float my_s = lane < k ? s[my_idx] : 0.0f;
    float S = 0.0f;
    for (int r = 0; r < k; ++r) {
        unsigned who = __ballot_sync(0xffffffffu, lane < k && rank == r);
        float sv = __shfl_sync(0xffffffffu, my_s, __ffs(who) - 1);
        S = __fadd_rn(S, sv);
    }
    if (lane < k) {
        idx_out[(size_t)t * k + lane] = my_idx;
        w_out[(size_t)t * k + lane] = __fdiv_rn(my_s, S);
    }
}

// ============================================================================ permutation
// "Routed experts" box (group all tokens per expert) as a counting sort:
// histogram -> exclusive prefix sum -> stable scatter, one CTA of 1024 threads.
// Stability (ascending t inside an expert) without a second sort: tokens are
// processed in rounds of WR warps x 32 tokens; per warp and expert a 32-bit
// mask of the lanes (tokens) that chose the expert gives the rank inside the
// warp (popc of the lower lanes) and, prefix-summed over warps in order, the
// warp's base.
constexpr int PERM_THREADS = 1024;
constexpr int PERM_SCAN_CAP = 2048;

__device__ int block_excl_scan(int* a, int n, int* wsum) {
    // in-place exclusive scan of a[0..n), n <= 2048, returns the total
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int v0 = 2 * tid < n ? a[2 * tid] : 0;
    int v1 = 2 * tid + 1 < n ? a[2 * tid + 1] : 0;
    int sum = v0 + v1;
    int inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int w = wsum[lane];
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        wsum[lane] = wi - w;  // exclusive
        if (lane == 31) wsum[32] = wi;
    }
    __syncthreads();
    int excl = wsum[warp] + inc - sum;
    if (2 * tid < n) a[2 * tid] = excl;
    if (2 * tid + 1 < n) a[2 * tid + 1] = excl + v0;
    int total = wsum[32];
    __syncthreads();
    return total;
}

// Group of global expert id `gid` when the groups are experts [lo, lo + E), else -1
// (unsigned arithmetic: any int id, however negative, maps outside).
__device__ __forceinline__ int local_expert(int gid, int lo, int E) {
    const unsigned e = (unsigned)gid - (unsigned)lo;
    return e < (unsigned)E ? (int)e : -1;
}

__global__ void __launch_bounds__(PERM_THREADS, 1) permute_kernel(PermuteArgs a, int WR) {
    extern __shared__ int psm[];
    const int E = a.E, T = a.T, k = a.k;
    int* s_scan = psm;                              // [PERM_SCAN_CAP]
    int* s_base = s_scan + PERM_SCAN_CAP;           // [E]
    int* s_wsum = s_base + E;                       // [33] (+pad)
    unsigned* s_mask = reinterpret_cast<unsigned*>(s_wsum + 64);  // [WR * E]
    int* s_wbase = reinterpret_cast<int*>(s_mask + WR * E);       // [WR * E]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool fwd = a.row_off != nullptr;
    const int total_pairs = T * k;

    for (int e = tid; e < E; e += PERM_THREADS) s_scan[e] = 0;
    __syncthreads();
    bool bad = false;
    for (int p = tid; p < total_pairs; p += PERM_THREADS) {
        int e = local_expert(a.idx[p], a.id_lo, E);
        if (e >= 0 && e < E) atomicAdd(&s_scan[e], 1);
        else bad = true;
    }
    if (bad && !a.foreign_ok) set_dev_error(MOE_DEVERR_BAD_EXPERT);
    __syncthreads();
    for (int e = tid; e < E; e += PERM_THREADS) a.counts[e] = s_scan[e];
    __syncthreads();
    int tot = block_excl_scan(s_scan, E, s_wsum);
    for (int e = tid; e < E; e += PERM_THREADS) {
        a.offsets[e] = s_scan[e];
        s_base[e] = s_scan[e];
    }
    if (tid == 0) a.offsets[E] = tot;
    __syncthreads();

    if (fwd) {
        const int NG = E + a.n_shared;
        // group extents: routed experts back to back, the shared expert after them
        for (int g = tid; g <= NG; g += PERM_THREADS)
            a.row_off[g] = g <= E ? (g < E ? s_base[g] : tot) : tot + T;
        __syncthreads();
        for (int pass = 0; pass < 2; ++pass) {
            const int bn = pass == 0 ? a.bn_gu : a.bn_dn;
            for (int g = tid; g < NG; g += PERM_THREADS) {
                int n = g < E ? a.counts[g] : T;
                int mt = pass == 0 ? (g < E ? a.mt_gu_routed : a.mt_gu_shared) : a.mt_dn;
                s_scan[g] = ((n + bn - 1) / bn) * mt;
            }
            __syncthreads();
            int items = block_excl_scan(s_scan, NG, s_wsum);
            int32_t* dst = pass == 0 ? a.item_off_gu : a.item_off_dn;
            for (int g = tid; g < NG; g += PERM_THREADS) dst[g] = s_scan[g];
            if (tid == 0) dst[NG] = items;
            __syncthreads();
        }
        for (int t = tid; t < T * a.n_shared; t += PERM_THREADS) {
            a.row_tok[tot + t] = t;
            a.row_coef[tot + t] = 1.0f;
        }
    }

    // stable scatter, rounds of WR warps x 32 tokens
    const int TPR = WR * 32;
    for (int base = 0; base < T; base += TPR) {
        for (int i = tid; i < WR * E; i += PERM_THREADS) s_mask[i] = 0u;
        __syncthreads();
        const int t = base + warp * 32 + lane;
        const bool mine = warp < WR && t < T;
        if (mine) {
            for (int j = 0; j < k; ++j) {
                int e = local_expert(a.idx[(size_t)t * k + j], a.id_lo, E);
                if (e >= 0 && e < E) atomicOr(&s_mask[warp * E + e], 1u << lane);
            }
        }
        __syncthreads();
        for (int e = tid; e < E; e += PERM_THREADS) {
            int acc = s_base[e];
            for (int w2 = 0; w2 < WR; ++w2) {
                s_wbase[w2 * E + e] = acc;
                acc += __popc(s_mask[w2 * E + e]);
            }
            s_base[e] = acc;
        }
        __syncthreads();
        if (mine) {
            const unsigned lower = (1u << lane) - 1u;
            for (int j = 0; j < k; ++j) {
                const int p = t * k + j;
                int e = local_expert(a.idx[p], a.id_lo, E);
                if (e >= 0 && e < E) {
                    int row = s_wbase[warp * E + e] + __popc(s_mask[warp * E + e] & lower);
                    a.src[row] = p;
                    a.inv[p] = row;
                    if (fwd) {
                        a.row_tok[row] = t;
                        a.row_coef[row] = a.routed_scale * a.topk_w[p];
                    }
                } else {
                    a.inv[p] = -1;
                }
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------- multi-CTA permutation
// The same counting sort over many CTAs for large T: each CTA owns
// PERM_TB consecutive tokens (8 warps x 32).
//   count:   per-CTA histogram (per-warp lane masks, as above) -> hist[b][e]
//   scan:    one CTA: hist[b][e] -> exclusive prefix over b (the CTA's base
//            inside expert e), counts, offsets, group extents, tile schedules
//   scatter: per CTA, warp bases from the masks, rows = offsets[e] + hist[b][e]
//            + warp base + rank among the lower lanes
// The rows come out identical to the single-CTA kernel's (ascending t).
constexpr int PERM_TB = 256;

__device__ __forceinline__ void build_lane_masks(const PermuteArgs& a, unsigned* s_mask, int t0, bool flag_bad) {
    const int E = a.E, k = a.k, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < (PERM_TB / 32) * E; i += PERM_TB) s_mask[i] = 0u;
    __syncthreads();
    const int t = t0 + warp * 32 + lane;
    if (t < a.T) {
        bool bad = false;
        for (int j = 0; j < k; ++j) {
            const int e = local_expert(a.idx[(size_t)t * k + j], a.id_lo, E);
            if (e >= 0 && e < E) atomicOr(&s_mask[warp * E + e], 1u << lane);
            else bad = true;
        }
        if (bad && flag_bad && !a.foreign_ok) set_dev_error(MOE_DEVERR_BAD_EXPERT);
    }
    __syncthreads();
}

__global__ void __launch_bounds__(PERM_TB) permute_count_kernel(PermuteArgs a, int32_t* __restrict__ hist) {
    extern __shared__ unsigned pcm[];
    build_lane_masks(a, pcm, blockIdx.x * PERM_TB, true);
    for (int e = threadIdx.x; e < a.E; e += PERM_TB) {
        int c = 0;
        for (int w = 0; w < PERM_TB / 32; ++w) c += __popc(pcm[w * a.E + e]);
        hist[(size_t)blockIdx.x * a.E + e] = c;
    }
}

__global__ void __launch_bounds__(PERM_THREADS, 1) permute_scan_kernel(PermuteArgs a, int32_t* __restrict__ hist,
                                                                       int nb) {
    extern __shared__ int psm2[];
    const int E = a.E, T = a.T, tid = threadIdx.x;
    int* s_scan = psm2;                      // [PERM_SCAN_CAP]
    int* s_wsum = s_scan + PERM_SCAN_CAP;    // [64]
    for (int e = tid; e < E; e += PERM_THREADS) {
        int run = 0;
        for (int b = 0; b < nb; ++b) {
            const int v = hist[(size_t)b * E + e];
            hist[(size_t)b * E + e] = run;
            run += v;
        }
        a.counts[e] = run;
        s_scan[e] = run;
    }
    __syncthreads();
    const int tot = block_excl_scan(s_scan, E, s_wsum);
    for (int e = tid; e < E; e += PERM_THREADS) a.offsets[e] = s_scan[e];
    if (tid == 0) a.offsets[E] = tot;
    const int NG = E + a.n_shared;
    for (int g = tid; g <= NG; g += PERM_THREADS) a.row_off[g] = g <= E ? (g < E ? s_scan[g] : tot) : tot + T;
    __syncthreads();
    for (int pass = 0; pass < 2; ++pass) {
        const int bn = pass == 0 ? a.bn_gu : a.bn_dn;
        for (int g = tid; g < NG; g += PERM_THREADS) {
            const int n = g < E ? a.counts[g] : T;
            const int mt = pass == 0 ? (g < E ? a.mt_gu_routed : a.mt_gu_shared) : a.mt_dn;
            s_scan[g] = ((n + bn - 1) / bn) * mt;
        }
        __syncthreads();
        const int items = block_excl_scan(s_scan, NG, s_wsum);
        int32_t* dst = pass == 0 ? a.item_off_gu : a.item_off_dn;
        for (int g = tid; g < NG; g += PERM_THREADS) dst[g] = s_scan[g];
        if (tid == 0) dst[NG] = items;
        __syncthreads();
    }
    for (int t = tid; t < T * a.n_shared; t += PERM_THREADS) {
        a.row_tok[tot + t] = t;
        a.row_coef[tot + t] = 1.0f;
    }
}

__global__ void __launch_bounds__(PERM_TB) permute_scatter_kernel(PermuteArgs a, const int32_t* __restrict__ hist) {
    extern __shared__ unsigned psc[];
    const int E = a.E, k = a.k, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    unsigned* s_mask = psc;                                       // [8][E]
    int* s_wbase = reinterpret_cast<int*>(psc + (PERM_TB / 32) * E);  // [8][E]
    const int t0 = blockIdx.x * PERM_TB;
    build_lane_masks(a, s_mask, t0, false);
    for (int e = tid; e < E; e += PERM_TB) {
        int acc = a.offsets[e] + hist[(size_t)blockIdx.x * E + e];
        for (int w = 0; w < PERM_TB / 32; ++w) {
            s_wbase[w * E + e] = acc;
            acc += __popc(s_mask[w * E + e]);
        }
    }
    __syncthreads();
    const int t = t0 + warp * 32 + lane;
    if (t < a.T) {
        const unsigned lower = (1u << lane) - 1u;
        for (int j = 0; j < k; ++j) {
            const int p = t * k + j;
            const int e = local_expert(a.idx[p], a.id_lo, E);
            if (e >= 0 && e < E) {
                const int row = s_wbase[warp * E + e] + __popc(s_mask[warp * E + e] & lower);
                a.src[row] = p;
                a.inv[p] = row;
                a.row_tok[row] = t;
                a.row_coef[row] = a.routed_scale * a.topk_w[p];
            } else {
                a.inv[p] = -1;
            }
        }
    }
}

// ============================================================================ gather
__global__ void __launch_bounds__(256) gather_rows_kernel(const void* __restrict__ x, int x_f32, int d, int n_tok,
                                                          const int32_t* __restrict__ row_tok,
                                                          const int32_t* __restrict__ n_rows_dev, int rows_cap,
                                                          __nv_bfloat16* __restrict__ xp) {
    int n_rows = *n_rows_dev;
    // checking build: the row count fits the permuted buffer, every row's token exists
    if (kDebugChecks && !dbg_ok(n_rows >= 0 && n_rows <= rows_cap)) n_rows = n_rows < 0 ? 0 : rows_cap;
    const int nvec = d / 8;  // 8 bf16 per 16-byte vector
    for (int r = blockIdx.x; r < n_rows; r += gridDim.x) {
        const int t = row_tok[r];
        if (kDebugChecks && !dbg_ok((unsigned)t < (unsigned)n_tok)) continue;  // uniform over the block
        uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)r * d);
        if (x_f32) {
            const float4* srcf = reinterpret_cast<const float4*>(static_cast<const float*>(x) + (size_t)t * d);
            for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
                float4 a = srcf[2 * v], b = srcf[2 * v + 1];
                __nv_bfloat162 p0 = __floats2bfloat162_rn(a.x, a.y), p1 = __floats2bfloat162_rn(a.z, a.w);
                __nv_bfloat162 p2 = __floats2bfloat162_rn(b.x, b.y), p3 = __floats2bfloat162_rn(b.z, b.w);
                dst[v] = make_uint4(*reinterpret_cast<uint32_t*>(&p0), *reinterpret_cast<uint32_t*>(&p1),
                                    *reinterpret_cast<uint32_t*>(&p2), *reinterpret_cast<uint32_t*>(&p3));
            }
        } else {
            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + (size_t)t * d);
            for (int v = threadIdx.x; v < nvec; v += blockDim.x) dst[v] = src[v];
        }
    }
}

// Token-major form of the same copy: a CTA reads token t's row once (converting
// fp32 to bf16 once) and writes it to the permuted rows of its (token, slot)
// pairs, inv[t*k + j] (-1: the pair has no row here), and to its shared-expert
// row shared_base + t.  Every x row is read once instead of once per row that
// holds it, which matters when x does not stay in L2 between its copies.
__global__ void __launch_bounds__(256) scatter_rows_kernel(const void* __restrict__ x, int x_f32, int d, int T, int k,
                                                           const int32_t* __restrict__ inv,
                                                           const int32_t* __restrict__ shared_base_dev, int rows_cap,
                                                           __nv_bfloat16* __restrict__ xp) {
    __shared__ int s_rows[33];  // top_k <= 32, + the shared-expert row
    const int nvec = d / 8;     // 8 bf16 per 16-byte vector
    const int shared_base = shared_base_dev ? *shared_base_dev : -1;
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        __syncthreads();  // the previous token's rows are no longer read
        if (threadIdx.x <= k) {
            int row = threadIdx.x < k ? inv[(size_t)t * k + threadIdx.x] : (shared_base >= 0 ? shared_base + t : -1);
            // checking build: a row inside the permuted buffer (else it is skipped)
            if (kDebugChecks && row >= 0 && !dbg_ok(row < rows_cap)) row = -1;
            s_rows[threadIdx.x] = row;
        }
        __syncthreads();
        for (int v0 = 0; v0 < nvec; v0 += 4 * 256) {
            uint4 buf[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int v = v0 + j * 256 + threadIdx.x;
                if (v >= nvec) break;
                if (x_f32) {
                    const float4* srcf = reinterpret_cast<const float4*>(static_cast<const float*>(x) + (size_t)t * d);
                    const float4 a = srcf[2 * v], b = srcf[2 * v + 1];
                    __nv_bfloat162 p0 = __floats2bfloat162_rn(a.x, a.y), p1 = __floats2bfloat162_rn(a.z, a.w);
                    __nv_bfloat162 p2 = __floats2bfloat162_rn(b.x, b.y), p3 = __floats2bfloat162_rn(b.z, b.w);
                    buf[j] = make_uint4(*reinterpret_cast<uint32_t*>(&p0), *reinterpret_cast<uint32_t*>(&p1),
                                        *reinterpret_cast<uint32_t*>(&p2), *reinterpret_cast<uint32_t*>(&p3));
                } else {
                    buf[j] = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + (size_t)t * d)[v];
                }
            }
            for (int jr = 0; jr <= k; ++jr) {
                const int row = s_rows[jr];
                if (row < 0) continue;  // uniform over the block
                uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)row * d);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int v = v0 + j * 256 + threadIdx.x;
                    if (v >= nvec) break;
                    dst[v] = buf[j];
                }
            }
        }
    }
}

// ============================================================================ FP8 activations
// "Teardown: DeepSeek-V3", section 10: activations scaled in 1x128 tiles.
// One warp per (token, 128-channel block), 4 channels per lane:
//   sx = amax / 448 (1 when the block is all zero), q = e4m3_rn_sat(x / sx),
// with the divides correctly rounded in fp32, so the codes are reproducible.
// One lane's four consecutive channels of a 1x128 block held by the warp:
// sx = amax / 448 over the block (1 when it is all zero), codes e4m3_rn_sat(x / sx)
// with correctly rounded divides.  Returns the four codes (channel 0 in the low
// byte) and the block's scale.
__device__ __forceinline__ uint32_t quant_block_lane4(float x0, float x1, float x2, float x3, float* scale_out) {
    float amax = fmaxf(fmaxf(fabsf(x0), fabsf(x1)), fmaxf(fabsf(x2), fabsf(x3)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float scale = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    *scale_out = scale;
    const uint32_t lo = cvt_e4m3x2(__fdiv_rn(x1, scale), __fdiv_rn(x0, scale));
    const uint32_t hi = cvt_e4m3x2(__fdiv_rn(x3, scale), __fdiv_rn(x2, scale));
    return lo | (hi << 16);
}

__global__ void __launch_bounds__(256) quant_act_kernel(const __nv_bfloat16* __restrict__ x, int T, int d,
                                                        uint8_t* __restrict__ q, float* __restrict__ sx) {
    const int nb = d / 128;
    const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (gw >= (long long)T * nb) return;  // uniform per warp
    const int t = (int)(gw / nb), b = (int)(gw % nb);
    const size_t off = (size_t)t * d + (size_t)b * 128 + lane * 4;
    const uint2 raw = *reinterpret_cast<const uint2*>(x + off);
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
    const float2 a = __bfloat1622float2(p2[0]), c = __bfloat1622float2(p2[1]);
    float scale;
    *reinterpret_cast<uint32_t*>(q + off) = quant_block_lane4(a.x, a.y, c.x, c.y, &scale);
    if (lane == 0) sx[(size_t)t * nb + b] = scale;
}

// S6 and the copy into expert order in one token-major pass: a CTA takes token t,
// its warps quantise the row's 1x128 blocks (quant_block_lane4, the arithmetic of
// quant_act_kernel) and write codes and scale to every permuted row of the token:
// inv[t*k + j] >= 0 and, when shared_base_dev is set, *shared_base_dev + t.  With
// xq_in set (codes made by the pre-norm) the codes and scales are copied instead.
// Codes [rows, d]; scales K-block major, sxT[b * rows_ld + row].
__global__ void __launch_bounds__(256) quant_scatter_fp8_kernel(
    const __nv_bfloat16* __restrict__ x, const uint8_t* __restrict__ xq_in, const float* __restrict__ sx_in, int d,
    int T, int k, const int32_t* __restrict__ inv, const int32_t* __restrict__ shared_base_dev, int rows_ld,
    uint8_t* __restrict__ xpq, float* __restrict__ sxT) {
    __shared__ int s_rows[33];  // top_k <= 32, + the shared-expert row
    const int nb = d / 128, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int shared_base = shared_base_dev ? *shared_base_dev : -1;
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        __syncthreads();  // the previous token's rows are no longer read
        if (threadIdx.x <= k) {
            int row = threadIdx.x < k ? inv[(size_t)t * k + threadIdx.x] : (shared_base >= 0 ? shared_base + t : -1);
            // checking build: a row inside the permuted buffers (else it is skipped)
            if (kDebugChecks && row >= 0 && !dbg_ok(row < rows_ld)) row = -1;
            s_rows[threadIdx.x] = row;
        }
        __syncthreads();
        for (int b = warp; b < nb; b += blockDim.x / 32) {
            const size_t off = (size_t)t * d + (size_t)b * 128 + lane * 4;
            uint32_t code;
            float scale;
            if (xq_in) {
                code = *reinterpret_cast<const uint32_t*>(xq_in + off);
                scale = sx_in[(size_t)t * nb + b];
            } else {
                const uint2 raw = *reinterpret_cast<const uint2*>(x + off);
                const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
                const float2 a = __bfloat1622float2(p2[0]), c = __bfloat1622float2(p2[1]);
                code = quant_block_lane4(a.x, a.y, c.x, c.y, &scale);
            }
            for (int jr = 0; jr <= k; ++jr) {
                const int row = s_rows[jr];
                if (row < 0) continue;  // uniform over the block
                *reinterpret_cast<uint32_t*>(xpq + (size_t)row * d + (size_t)b * 128 + lane * 4) = code;
                if (lane == 0) sxT[(size_t)b * rows_ld + row] = scale;
            }
        }
    }
}

// ============================================================================ wait self-test
// The failure path of the bounded waits, on its own: one thread waits on an
// mbarrier that nothing completes; after limit_ns the wait gives up, sets
// MOE_DEVERR_TIMEOUT and the kernel returns (no TMA, TMEM or MMA in flight).
__global__ void __launch_bounds__(32) wait_selftest_kernel(unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, &abort_flag, limit_ns);
}

// ============================================================================ dense schedule
// The tables of one group of all T rows (the dense FFN): row_tok = identity,
// row_coef = 1, group extents {0, T}, tile counts of the two GEMMs.
__global__ void __launch_bounds__(256) dense_schedule_kernel(int T, int bn, int mt_gu, int mt_dn,
                                                             int32_t* __restrict__ row_off,
                                                             int32_t* __restrict__ item_gu,
                                                             int32_t* __restrict__ item_dn,
                                                             int32_t* __restrict__ row_tok,
                                                             float* __restrict__ row_coef) {
    const int i0 = blockIdx.x * blockDim.x + threadIdx.x;
    for (int r = i0; r < T; r += gridDim.x * blockDim.x) {
        row_tok[r] = r;
        row_coef[r] = 1.0f;
    }
    if (i0 == 0) {
        const int chunks = (T + bn - 1) / bn;
        row_off[0] = 0;
        row_off[1] = T;
        item_gu[0] = 0;
        item_gu[1] = chunks * mt_gu;
        item_dn[0] = 0;
        item_dn[1] = chunks * mt_dn;
    }
}

// ============================================================================ pre-norm
// "RMSNorm" box: r = 1/sqrt(mean_c h[c]^2 + eps), the mean reduced in fp32;
// out = bf16(bf16(h * r) * g).  With q and sx the same pass also writes the
// 1x128 e4m3 codes and scales of out, in the arithmetic of quant_act_kernel.
// One CTA of 128 threads per token row; vector i of 8 features goes to thread
// i % 128, so a 128-feature block is 16 consecutive lanes of one warp.
__global__ void __launch_bounds__(NORM_THREADS) rmsnorm_kernel(const __nv_bfloat16* __restrict__ h,
                                                               const __nv_bfloat16* __restrict__ g, int d, float eps,
                                                               __nv_bfloat16* __restrict__ out,
                                                               uint8_t* __restrict__ q, float* __restrict__ sx) {
    __shared__ float s_part[NORM_THREADS / 32];
    const int t = blockIdx.x;
    const int lane = threadIdx.x & 31;
    const int nvec = d / 8;
    const uint4* hr = reinterpret_cast<const uint4*>(h + (size_t)t * d);
    uint4 v[NORM_MAX_VEC];
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < NORM_MAX_VEC; ++i) {
        const int vi = threadIdx.x + i * NORM_THREADS;
        v[i] = vi < nvec ? hr[vi] : make_uint4(0u, 0u, 0u, 0u);
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&v[i]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(p2[j]);
            ss = fmaf(f.x, f.x, ss);
            ss = fmaf(f.y, f.y, ss);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) s_part[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.0f;
#pragma unroll
    for (int w = 0; w < NORM_THREADS / 32; ++w) tot += s_part[w];
    const float r = __frsqrt_rn(__fadd_rn(__fdiv_rn(tot, (float)d), eps));
    const uint4* gv = reinterpret_cast<const uint4*>(g);
    uint4* ov = reinterpret_cast<uint4*>(out + (size_t)t * d);
#pragma unroll
    for (int i = 0; i < NORM_MAX_VEC; ++i) {
        const int vi = threadIdx.x + i * NORM_THREADS;
        if (i * NORM_THREADS >= nvec) break;  // uniform over the CTA
        const bool ok = vi < nvec;
        const uint4 gg = ok ? gv[vi] : make_uint4(0u, 0u, 0u, 0u);
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&v[i]);
        const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gg);
        float o[8];
        uint32_t pk[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(p2[j]);
            const float2 gf = __bfloat1622float2(g2[j]);
            const float a0 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(f.x, r)));
            const float a1 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(f.y, r)));
            const __nv_bfloat162 b = __floats2bfloat162_rn(__fmul_rn(a0, gf.x), __fmul_rn(a1, gf.y));
            const float2 bf = __bfloat1622float2(b);
            o[2 * j] = bf.x;
            o[2 * j + 1] = bf.y;
            pk[j] = *reinterpret_cast<const uint32_t*>(&b);
        }
        if (ok) ov[vi] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        if (q) {
            float amax = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(o[j]));
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            const float scale = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
            uint32_t c[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) c[j] = cvt_e4m3x2(__fdiv_rn(o[2 * j + 1], scale), __fdiv_rn(o[2 * j], scale));
            if (ok) {
                *reinterpret_cast<uint2*>(q + (size_t)t * d + (size_t)vi * 8) =
                    make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
                if ((vi & 15) == 0) sx[(size_t)t * (d / 128) + vi / 16] = scale;
            }
        }
    }
}

// ============================================================================ bias controller
// "MoE router" box, update_bias: mean = sum(counts) / E in fp32; experts above
// it get bias - gamma, the others bias + gamma (one correctly rounded fp32 op).
__global__ void __launch_bounds__(1024) update_bias_kernel(const int32_t* __restrict__ counts, int E,
                                                           float* __restrict__ bias, float gamma) {
    __shared__ long long s_part[32];
    long long sum = 0;
    for (int e = threadIdx.x; e < E; e += blockDim.x) sum += counts[e];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = sum;
    __syncthreads();
    if (threadIdx.x < 32) {
        long long v = threadIdx.x < (blockDim.x + 31) / 32 ? s_part[threadIdx.x] : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (threadIdx.x == 0) s_part[0] = v;
    }
    __syncthreads();
    const float mean = __fdiv_rn(__ll2float_rn(s_part[0]), __int2float_rn(E));
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        bias[e] = __int2float_rn(counts[e]) > mean ? __fsub_rn(bias[e], gamma) : __fadd_rn(bias[e], gamma);
}

// ============================================================================ finalize
// y = bf16(acc (+ residual)); residual may be y itself (an in-place update of the
// residual stream: each element is read before it is written, by the same thread).
__global__ void __launch_bounds__(256) finalize_kernel(const float* __restrict__ acc, const __nv_bfloat16* residual,
                                                       __nv_bfloat16* y, size_t n8) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
        float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
        float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
        float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint4* yp = reinterpret_cast<uint4*>(y) + i;
        if (residual) {
            uint4 old = reinterpret_cast<const uint4*>(residual)[i];
            const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&old);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float2 f = __bfloat1622float2(o2[j]);
                v[2 * j] += f.x;
                v[2 * j + 1] += f.y;
            }
        }
        uint32_t p[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
            p[j] = *reinterpret_cast<uint32_t*>(&h);
        }
        *yp = make_uint4(p[0], p[1], p[2], p[3]);
    }
}

// ============================================================================ expert parallelism
// The experts are split over R ranks in contiguous blocks of epr = E / R; with
// R = n_groups rank r holds group r (the pages' device-aligned groups).
// Dispatch: token t goes to rank r when one of its k experts lies in r's block,
// once per rank however many of its experts sit there.  Send rows are
// rank-major, ascending token inside a rank.
constexpr int EP_THREADS = 1024;

__device__ __forceinline__ uint32_t ep_rank_mask(const int32_t* __restrict__ idx, int t, int k, int E, int epr) {
    uint32_t m = 0;
    for (int j = 0; j < k; ++j) {
        const int e = idx[(size_t)t * k + j];
        if ((unsigned)e < (unsigned)E) m |= 1u << (e / epr);
    }
    return m;
}

// one CTA per rank: the number of tokens it receives from this rank
__global__ void __launch_bounds__(EP_THREADS) ep_count_kernel(const int32_t* __restrict__ idx, int T, int k, int E,
                                                              int epr, int32_t* __restrict__ counts) {
    __shared__ int wsum[EP_THREADS / 32];
    const int r = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int c = 0;
    for (int t = threadIdx.x; t < T; t += EP_THREADS) c += (ep_rank_mask(idx, t, k, E, epr) >> r) & 1u;
    for (int o = 16; o >= 1; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (lane == 0) wsum[warp] = c;
    __syncthreads();
    if (warp == 0) {
        c = wsum[lane];
        for (int o = 16; o >= 1; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        if (lane == 0) counts[r] = c;
    }
}

// one CTA per rank: its offset and its send rows' origin tokens, in token order
// capacity > 0: rank r's rows start at r * capacity (fixed-capacity layout; offsets
// is not written) and its unused slots get token -1
__global__ void __launch_bounds__(EP_THREADS) ep_place_kernel(const int32_t* __restrict__ idx, int T, int k, int E,
                                                              int epr, int R, const int32_t* __restrict__ counts,
                                                              int32_t* __restrict__ offsets,
                                                              int32_t* __restrict__ send_tok, int capacity) {
    __shared__ int wsum[EP_THREADS / 32 + 1];
    __shared__ int base_s;
    const int r = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        int o = 0;
        if (capacity > 0) {
            o = r * capacity;
        } else {
            for (int q = 0; q < r; ++q) o += counts[q];
            offsets[r] = o;
            if (r == R - 1) offsets[R] = o + counts[r];
        }
        base_s = o;
    }
    __syncthreads();
    if (capacity > 0)
        for (int j = counts[r] + threadIdx.x; j < capacity; j += EP_THREADS) send_tok[(size_t)r * capacity + j] = -1;
    int base = base_s;
    for (int t0 = 0; t0 < T; t0 += EP_THREADS) {
        const int t = t0 + threadIdx.x;
        const bool mine = t < T && ((ep_rank_mask(idx, t, k, E, epr) >> r) & 1u);
        const unsigned b = __ballot_sync(0xffffffffu, mine);
        if (lane == 0) wsum[warp] = __popc(b);
        __syncthreads();
        if (warp == 0) {  // exclusive prefix over the 32 warps; wsum[32] = the chunk's total
            const int v = wsum[lane];
            int inc = v;
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += u;
            }
            wsum[lane] = inc - v;
            if (lane == 31) wsum[32] = inc;
        }
        __syncthreads();
        if (mine) send_tok[base + wsum[warp] + __popc(b & ((1u << lane) - 1u))] = t;
        base += wsum[32];
        __syncthreads();
    }
}

// the routing of every send row: its token's k expert ids and weights
__global__ void __launch_bounds__(256) ep_rows_kernel(const int32_t* __restrict__ idx, const float* __restrict__ w,
                                                      int k, const int32_t* __restrict__ send_tok,
                                                      const int32_t* __restrict__ n_rows_dev,
                                                      int32_t* __restrict__ send_idx, float* __restrict__ send_w) {
    const int n = *n_rows_dev * k;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const int r = i / k, j = i - r * k;
        const size_t p = (size_t)send_tok[r] * k + j;
        send_idx[i] = idx[p];
        send_w[i] = w[p];
    }
}

// Packed dispatch rows (fixed-capacity layout): row r = bf16 x [d] | ids int32 [k] |
// weights fp32 [k] | padding to row_bytes.  One CTA per row; a padding slot (token
// -1) gets ids -1 (its x and weights are left as they are).  Row r (destination rank
// q = r / capacity, slot i = r % capacity) goes to packed + r * row_bytes, or, with
// dst_rank set (peer form), straight into rank q's receive buffer at slot
// dst_row0 + i: dst_rank[q] + (dst_row0 + i) * row_bytes.
__global__ void __launch_bounds__(128) ep_pack_kernel(const int32_t* __restrict__ idx, const float* __restrict__ w,
                                                      int k, const void* __restrict__ x, int x_f32, int d,
                                                      const int32_t* __restrict__ send_tok,
                                                      uint8_t* __restrict__ packed, int row_bytes,
                                                      uint8_t* const* __restrict__ dst_rank, int capacity,
                                                      int dst_row0) {
    const int r = blockIdx.x;
    const int t = send_tok[r];
    uint8_t* row;
    if (dst_rank) {
        const int q = r / capacity;
        row = dst_rank[q] + (size_t)(dst_row0 + (r - q * capacity)) * row_bytes;
    } else {
        row = packed + (size_t)r * row_bytes;
    }
    int32_t* ids = reinterpret_cast<int32_t*>(row + (size_t)d * 2);
    float* ws = reinterpret_cast<float*>(row + (size_t)d * 2 + (size_t)k * 4);
    if (t < 0) {
        for (int j = threadIdx.x; j < k; j += blockDim.x) ids[j] = -1;
        return;
    }
    for (int j = threadIdx.x; j < k; j += blockDim.x) {
        ids[j] = idx[(size_t)t * k + j];
        ws[j] = w[(size_t)t * k + j];
    }
    uint4* dst = reinterpret_cast<uint4*>(row);
    const int nvec = d / 8;  // 8 bf16 per 16 bytes
    if (x_f32) {
        const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(x) + (size_t)t * d);
        for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
            const float4 a = src[2 * v], b = src[2 * v + 1];
            __nv_bfloat162 p0 = __floats2bfloat162_rn(a.x, a.y), p1 = __floats2bfloat162_rn(a.z, a.w);
            __nv_bfloat162 p2 = __floats2bfloat162_rn(b.x, b.y), p3 = __floats2bfloat162_rn(b.z, b.w);
            dst[v] = make_uint4(*reinterpret_cast<uint32_t*>(&p0), *reinterpret_cast<uint32_t*>(&p1),
                                *reinterpret_cast<uint32_t*>(&p2), *reinterpret_cast<uint32_t*>(&p3));
        }
    } else {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + (size_t)t * d);
        for (int v = threadIdx.x; v < nvec; v += blockDim.x) dst[v] = src[v];
    }
}

// received packed rows -> the three arrays moe_experts_routed reads; one CTA per row
// (a padding row's ids stay -1, so its slots are skipped there)
__global__ void __launch_bounds__(128) ep_unpack_kernel(const uint8_t* __restrict__ packed, int row_bytes, int d,
                                                        int k, __nv_bfloat16* __restrict__ x_rows,
                                                        int32_t* __restrict__ ids_out, float* __restrict__ w_out) {
    const int r = blockIdx.x;
    const uint8_t* row = packed + (size_t)r * row_bytes;
    const int32_t* ids = reinterpret_cast<const int32_t*>(row + (size_t)d * 2);
    const float* ws = reinterpret_cast<const float*>(row + (size_t)d * 2 + (size_t)k * 4);
    bool live = false;
    for (int j = 0; j < k; ++j) live |= ids[j] >= 0;  // uniform over the block
    for (int j = threadIdx.x; j < k; j += blockDim.x) {
        ids_out[(size_t)r * k + j] = ids[j];
        w_out[(size_t)r * k + j] = live ? ws[j] : 0.0f;
    }
    if (!live) return;  // nothing reads a padding row's x
    const uint4* src = reinterpret_cast<const uint4*>(row);
    uint4* dst = reinterpret_cast<uint4*>(x_rows + (size_t)r * d);
    for (int v = threadIdx.x; v < d / 8; v += blockDim.x) dst[v] = src[v];
}

// combine: acc[send_tok[r], :] += back[r, :] (the partial sums the ranks returned),
// or, with src_rank set (peer form), the row read straight from the result buffer of
// the rank that computed it: src_rank[q] + (src_row0 + i) * d for q = r / capacity,
// i = r % capacity.
__global__ void __launch_bounds__(256) ep_combine_kernel(const float* __restrict__ back,
                                                         const int32_t* __restrict__ send_tok, int n_rows, int T,
                                                         int d, float* __restrict__ acc,
                                                         const float* const* __restrict__ src_rank, int capacity,
                                                         int src_row0) {
    const int d4 = d / 4;
    const size_t n = (size_t)n_rows * d4;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const size_t r = i / d4;
        const int c = (int)(i - r * d4) * 4;
        const int t = send_tok[r];
        if (t == -1) continue;             // a padding slot of the fixed-capacity layout
        if ((unsigned)t >= (unsigned)T) {  // not a token of this batch: flagged and skipped
            set_dev_error(MOE_DEVERR_BAD_ROWS);
            continue;
        }
        const float* src;
        if (src_rank) {
            const int q = (int)(r / capacity);
            src = src_rank[q] + (size_t)(src_row0 + (int)(r - (size_t)q * capacity)) * d;
        } else {
            src = back + r * d;
        }
        const float4 v = *reinterpret_cast<const float4*>(src + c);
        float* dst = acc + (size_t)t * d + c;
        atomicAdd(dst + 0, v.x);
        atomicAdd(dst + 1, v.y);
        atomicAdd(dst + 2, v.z);
        atomicAdd(dst + 3, v.w);
    }
}

// ============================================================================ launchers
size_t gemm_args_size() { return sizeof(GemmArgs); }

template <int MODE, int BN>
static cudaError_t launch_gemm_t(const GemmArgs* args, int grid, cudaStream_t s) {
    using C = GemmCfg<MODE, BN>;
    static std::atomic<bool> attr_set[64];  // once per device (a repeated set is harmless)
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev].load(std::memory_order_relaxed)) {
        cudaError_t e = cudaFuncSetAttribute(moe_gemm_kernel<MODE, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(true, std::memory_order_relaxed);
    }
    note_launch();
    moe_gemm_kernel<MODE, BN><<<grid, GEMM_THREADS, C::SMEM_BYTES, s>>>(*args);
    return cudaGetLastError();
}

template <int MODE>
static int smem_t(int bn) {
    switch (bn) {
        case 32: return GemmCfg<MODE, 32>::SMEM_BYTES;
        case 64: return GemmCfg<MODE, 64>::SMEM_BYTES;
        case 128: return GemmCfg<MODE, 128>::SMEM_BYTES;
        case 256: return GemmCfg<MODE, 256>::SMEM_BYTES;
    }
    return -1;
}

int gemm_smem_bytes(int mode, int bn) {
    if (mode == MODE_GATEUP) return smem_t<GEMM_GATEUP>(bn);
    if (mode == MODE_DOWN) return smem_t<GEMM_DOWN>(bn);
    return smem_t<GEMM_LOGITS>(bn);
}

template <int MODE>
static cudaError_t launch_mode(int bn, const GemmArgs* args, int grid, cudaStream_t s) {
    switch (bn) {
        case 32: return launch_gemm_t<MODE, 32>(args, grid, s);
        case 64: return launch_gemm_t<MODE, 64>(args, grid, s);
        case 128: return launch_gemm_t<MODE, 128>(args, grid, s);
        case 256: return launch_gemm_t<MODE, 256>(args, grid, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_gemm(int mode, int bn, const GemmArgs* args, int grid, cudaStream_t s) {
    if (mode == MODE_GATEUP) return launch_mode<GEMM_GATEUP>(bn, args, grid, s);
    if (mode == MODE_DOWN) return launch_mode<GEMM_DOWN>(bn, args, grid, s);
    return launch_mode<GEMM_LOGITS>(bn, args, grid, s);
}

template <int MODE, int BN>
static cudaError_t launch_gemm_fp8_t(const GemmArgs* args, int grid, cudaStream_t s) {
    using C = Fp8Cfg<MODE, BN>;
    static std::atomic<bool> attr_set[64];  // once per device (a repeated set is harmless)
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev].load(std::memory_order_relaxed)) {
        cudaError_t e = cudaFuncSetAttribute(moe_gemm_fp8_kernel<MODE, BN>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(true, std::memory_order_relaxed);
    }
    note_launch();
    moe_gemm_fp8_kernel<MODE, BN><<<grid, GEMM_THREADS, C::SMEM_BYTES, s>>>(*args);
    return cudaGetLastError();
}

int gemm_fp8_smem_bytes(int mode, int bn) {
    // token tiles of 128 rows and more run on the CTA-pair kernel
    if (mode == MODE_GATEUP)
        return bn == 32 ? Fp8Cfg<GEMM_GATEUP, 32>::SMEM_BYTES : Fp8Cfg<GEMM_GATEUP, 64>::SMEM_BYTES;
    return bn == 32 ? Fp8Cfg<GEMM_DOWN, 32>::SMEM_BYTES : Fp8Cfg<GEMM_DOWN, 64>::SMEM_BYTES;
}

cudaError_t launch_gemm_fp8(int mode, int bn, const GemmArgs* args, int grid, cudaStream_t s) {
    if (mode == MODE_GATEUP) {
        switch (bn) {
            case 32: return launch_gemm_fp8_t<GEMM_GATEUP, 32>(args, grid, s);
            case 64: return launch_gemm_fp8_t<GEMM_GATEUP, 64>(args, grid, s);
        }
    } else if (mode == MODE_DOWN) {
        switch (bn) {
            case 32: return launch_gemm_fp8_t<GEMM_DOWN, 32>(args, grid, s);
            case 64: return launch_gemm_fp8_t<GEMM_DOWN, 64>(args, grid, s);
        }
    }
    return cudaErrorInvalidValue;
}

template <int MODE>
static cudaError_t launch_gemm2_t(const GemmArgs* args, int grid, cudaStream_t s) {
    static std::atomic<bool> attr_set[64];  // once per device (a repeated set is harmless)
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev].load(std::memory_order_relaxed)) {
        cudaError_t e = cudaFuncSetAttribute(moe_gemm2_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             Gemm2Cfg::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(true, std::memory_order_relaxed);
    }
    note_launch();
    moe_gemm2_kernel<MODE><<<grid, PAIR_THREADS, Gemm2Cfg::SMEM_BYTES, s>>>(*args);
    return cudaGetLastError();
}

cudaError_t launch_gemm2(int mode, const GemmArgs* args, int grid, cudaStream_t s) {
    grid &= ~1;
    if (grid < 2) return cudaErrorInvalidValue;
    if (mode == MODE_GATEUP) return launch_gemm2_t<GEMM_GATEUP>(args, grid, s);
    if (mode == MODE_DOWN) return launch_gemm2_t<GEMM_DOWN>(args, grid, s);
    return cudaErrorInvalidValue;
}

template <int MODE>
static cudaError_t launch_gemm2_fp8_t(const GemmArgs* args, int grid, cudaStream_t s) {
    static std::atomic<bool> attr_set[64];  // once per device (a repeated set is harmless)
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev].load(std::memory_order_relaxed)) {
        cudaError_t e = cudaFuncSetAttribute(moe_gemm2_fp8_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             Gemm2Fp8Cfg::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(true, std::memory_order_relaxed);
    }
    note_launch();
    moe_gemm2_fp8_kernel<MODE><<<grid, PAIR8_THREADS, Gemm2Fp8Cfg::SMEM_BYTES, s>>>(*args);
    return cudaGetLastError();
}

cudaError_t launch_gemm2_fp8(int mode, const GemmArgs* args, int grid, cudaStream_t s) {
    grid &= ~1;
    if (grid < 2) return cudaErrorInvalidValue;
    if (mode == MODE_GATEUP) return launch_gemm2_fp8_t<GEMM_GATEUP>(args, grid, s);
    if (mode == MODE_DOWN) return launch_gemm2_fp8_t<GEMM_DOWN>(args, grid, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_quant_act(const __nv_bfloat16* x, int T, int d, uint8_t* q, float* sx, cudaStream_t s) {
    const long long warps = (long long)T * (d / 128);
    const long long blocks = (warps + 7) / 8;
    note_launch();
    quant_act_kernel<<<(unsigned)blocks, 256, 0, s>>>(x, T, d, q, sx);
    return cudaGetLastError();
}

cudaError_t launch_router_f32(const float* x, const __nv_bfloat16* wr, int T, int d, int E, float* logits,
                              cudaStream_t s) {
    note_launch();
    router_f32_kernel<<<T, 256, 0, s>>>(x, wr, T, d, E, logits);
    return cudaGetLastError();
}

cudaError_t launch_select(const float* logits, const float* bias, int T, int E, int G, int tg, int k, int32_t* idx,
                          float* w, cudaStream_t s, const float* parts, int n_parts) {
    if (n_parts > MAX_ROUTER_SPLITS) return cudaErrorInvalidValue;
    // few tokens: one per CTA (the partial sums and the decisions spread over
    // more SMs); many: eight per CTA (eight deciding warps a CTA)
    const int tpb = T >= 8 * 148 ? SELECT_THREADS / 32 : 1;
    const size_t smem = (size_t)tpb * 2 * E * sizeof(float);  // <= 64 KB (E <= 1024)
    static std::atomic<bool> attr_set[64];  // once per device (a repeated set is harmless)
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev].load(std::memory_order_relaxed)) {
        cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (SELECT_THREADS / 32) * 2 * 1024 * (int)sizeof(float));
        if (e != cudaSuccess) return e;
        attr_set[dev].store(true, std::memory_order_relaxed);
    }
    note_launch();
    // logits is written only when the partials are summed here (split-K router)
    select_kernel<<<(T + tpb - 1) / tpb, SELECT_THREADS, smem, s>>>(const_cast<float*>(logits), bias, T, E, G, tg,
                                                                    k, idx, w, n_parts > 1 ? parts : nullptr,
                                                                    n_parts, tpb);
    return cudaGetLastError();
}

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s) {
    int WR = 8192 / a.E;
    WR = WR > 32 ? 32 : (WR < 1 ? 1 : WR);
    const size_t smem = (size_t)(PERM_SCAN_CAP + a.E + 64) * 4 + (size_t)2 * WR * a.E * 4;
    static std::atomic<bool> attr_set[64];  // once per device (a repeated set is harmless)
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev].load(std::memory_order_relaxed)) {
        cudaError_t e = cudaFuncSetAttribute(permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(true, std::memory_order_relaxed);
    }
    note_launch();
    permute_kernel<<<1, PERM_THREADS, smem, s>>>(a, WR);
    return cudaGetLastError();
}

int permute_blocks(int T) { return (T + PERM_TB - 1) / PERM_TB; }

cudaError_t launch_permute_multi(const PermuteArgs& a, int32_t* hist, cudaStream_t s) {
    const int nb = permute_blocks(a.T);
    const size_t smem_c = (size_t)(PERM_TB / 32) * a.E * 4;
    static std::atomic<bool> attr_set[64];  // once per device (a repeated set is harmless)
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev].load(std::memory_order_relaxed)) {
        cudaError_t e = cudaFuncSetAttribute(permute_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             64 * 1024);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(permute_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(true, std::memory_order_relaxed);
    }
    note_launch();
    permute_count_kernel<<<nb, PERM_TB, smem_c, s>>>(a, hist);
    note_launch();
    permute_scan_kernel<<<1, PERM_THREADS, (PERM_SCAN_CAP + 64) * 4, s>>>(a, hist, nb);
    note_launch();
    permute_scatter_kernel<<<nb, PERM_TB, 2 * smem_c, s>>>(a, hist);
    return cudaGetLastError();
}

cudaError_t launch_gather(const void* x, bool x_f32, int d, int n_tok, const int32_t* row_tok, const int32_t* n_rows_dev,
                          int max_rows, __nv_bfloat16* x_perm, int n_sm, cudaStream_t s) {
    int grid = max_rows < n_sm * 8 ? max_rows : n_sm * 8;
    if (grid < 1) grid = 1;
    note_launch();
    gather_rows_kernel<<<grid, 256, 0, s>>>(x, x_f32 ? 1 : 0, d, n_tok, row_tok, n_rows_dev, max_rows, x_perm);
    return cudaGetLastError();
}

cudaError_t launch_quant_scatter_fp8(const __nv_bfloat16* x, const uint8_t* xq_in, const float* sx_in, int d, int T,
                                     int k, const int32_t* inv, const int32_t* shared_base_dev, int rows_ld,
                                     uint8_t* xpq, float* sxT, int n_sm, cudaStream_t s) {
    int grid = T < n_sm * 8 ? T : n_sm * 8;
    if (grid < 1) grid = 1;
    note_launch();
    quant_scatter_fp8_kernel<<<grid, 256, 0, s>>>(x, xq_in, sx_in, d, T, k, inv, shared_base_dev, rows_ld, xpq, sxT);
    return cudaGetLastError();
}

cudaError_t launch_scatter_rows(const void* x, bool x_f32, int d, int T, int k, const int32_t* inv,
                                const int32_t* shared_base_dev, int rows_cap, __nv_bfloat16* x_perm, int n_sm,
                                cudaStream_t s) {
    int grid = T < n_sm * 8 ? T : n_sm * 8;
    if (grid < 1) grid = 1;
    note_launch();
    scatter_rows_kernel<<<grid, 256, 0, s>>>(x, x_f32 ? 1 : 0, d, T, k, inv, shared_base_dev, rows_cap, x_perm);
    return cudaGetLastError();
}

__global__ void debug_poke_kernel(int32_t* p, int v) { *p = v; }

cudaError_t launch_debug_poke(int32_t* p, int v, cudaStream_t s) {
    note_launch();
    debug_poke_kernel<<<1, 1, 0, s>>>(p, v);
    return cudaGetLastError();
}

cudaError_t launch_finalize_bf16(const float* acc, const __nv_bfloat16* residual, __nv_bfloat16* y, size_t n,
                                 cudaStream_t s) {
    size_t n8 = n / 8;
    size_t grid = (n8 + 255) / 256;
    if (grid > 148 * 16) grid = 148 * 16;
    if (grid < 1) grid = 1;
    note_launch();
    finalize_kernel<<<(unsigned)grid, 256, 0, s>>>(acc, residual, y, n8);
    return cudaGetLastError();
}

cudaError_t launch_dense_schedule(int T, int bn, int mt_gu, int mt_dn, int32_t* row_off, int32_t* item_gu,
                                  int32_t* item_dn, int32_t* row_tok, float* row_coef, cudaStream_t s) {
    int grid = (T + 255) / 256;
    if (grid > 148) grid = 148;
    if (grid < 1) grid = 1;
    note_launch();
    dense_schedule_kernel<<<grid, 256, 0, s>>>(T, bn, mt_gu, mt_dn, row_off, item_gu, item_dn, row_tok, row_coef);
    return cudaGetLastError();
}

cudaError_t launch_wait_selftest(unsigned long long limit_ns, cudaStream_t s) {
    note_launch();
    wait_selftest_kernel<<<1, 32, 0, s>>>(limit_ns);
    return cudaGetLastError();
}

cudaError_t launch_rmsnorm(const __nv_bfloat16* h, const __nv_bfloat16* g, int T, int d, float eps,
                           __nv_bfloat16* out, uint8_t* q, float* sx, cudaStream_t s) {
    note_launch();
    rmsnorm_kernel<<<T, NORM_THREADS, 0, s>>>(h, g, d, eps, out, q, sx);
    return cudaGetLastError();
}

cudaError_t launch_update_bias(const int32_t* counts, int E, float* bias, float gamma, cudaStream_t s) {
    note_launch();
    update_bias_kernel<<<1, 1024, 0, s>>>(counts, E, bias, gamma);
    return cudaGetLastError();
}

cudaError_t read_clear_dev_error(unsigned int* flags, cudaStream_t s) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(flags, g_dev_error, sizeof(unsigned int), 0,
                                              cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return e;
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbolAsync(g_dev_error, &zero, sizeof(unsigned int), 0, cudaMemcpyHostToDevice, s) ==
                   cudaSuccess
               ? cudaStreamSynchronize(s)
               : cudaGetLastError();
}

cudaError_t launch_ep_dispatch(const int32_t* idx, const float* w, int T, int k, int E, int R, const void* x,
                               bool x_f32, int d, int32_t* counts, int32_t* offsets, int32_t* send_tok,
                               __nv_bfloat16* send_x, int32_t* send_idx, float* send_w, int n_sm, cudaStream_t s) {
    const int epr = E / R;
    note_launch();
    ep_count_kernel<<<R, EP_THREADS, 0, s>>>(idx, T, k, E, epr, counts);
    note_launch();
    ep_place_kernel<<<R, EP_THREADS, 0, s>>>(idx, T, k, E, epr, R, counts, offsets, send_tok, 0);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || T == 0) return e;
    const int max_rows = T * (k < R ? k : R);
    if ((e = launch_gather(x, x_f32, d, T, send_tok, offsets + R, max_rows, send_x, n_sm, s)) != cudaSuccess) return e;
    int grid = (max_rows * k + 255) / 256;
    grid = grid < n_sm * 4 ? grid : n_sm * 4;
    note_launch();
    ep_rows_kernel<<<grid, 256, 0, s>>>(idx, w, k, send_tok, offsets + R, send_idx, send_w);
    return cudaGetLastError();
}

cudaError_t launch_ep_dispatch_packed(const int32_t* idx, const float* w, int T, int k, int E, int R, int capacity,
                                      const void* x, bool x_f32, int d, int32_t* counts, int32_t* send_tok,
                                      uint8_t* packed, int row_bytes, cudaStream_t s, uint8_t* const* dst_rank,
                                      int dst_row0) {
    const int epr = E / R;
    note_launch();
    ep_count_kernel<<<R, EP_THREADS, 0, s>>>(idx, T, k, E, epr, counts);
    note_launch();
    ep_place_kernel<<<R, EP_THREADS, 0, s>>>(idx, T, k, E, epr, R, counts, nullptr, send_tok, capacity);
    note_launch();
    ep_pack_kernel<<<R * capacity, 128, 0, s>>>(idx, w, k, x, x_f32 ? 1 : 0, d, send_tok, packed, row_bytes, dst_rank,
                                                capacity, dst_row0);
    return cudaGetLastError();
}

cudaError_t launch_ep_unpack(const uint8_t* packed, int n_rows, int row_bytes, int d, int k, __nv_bfloat16* x_rows,
                             int32_t* ids, float* w, cudaStream_t s) {
    note_launch();
    ep_unpack_kernel<<<n_rows, 128, 0, s>>>(packed, row_bytes, d, k, x_rows, ids, w);
    return cudaGetLastError();
}

cudaError_t launch_ep_combine(const float* back, const int32_t* send_tok, int n_rows, int T, int d, float* acc,
                              int n_sm, cudaStream_t s, const float* const* src_rank, int capacity, int src_row0) {
    if (n_rows == 0) return cudaSuccess;
    const size_t n = (size_t)n_rows * (d / 4);
    size_t grid = (n + 255) / 256;
    if (grid > (size_t)n_sm * 16) grid = (size_t)n_sm * 16;
    note_launch();
    ep_combine_kernel<<<(unsigned)grid, 256, 0, s>>>(back, send_tok, n_rows, T, d, acc, src_rank, capacity, src_row0);
    return cudaGetLastError();
}

}  // namespace moe
