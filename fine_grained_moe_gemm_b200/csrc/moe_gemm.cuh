// Grouped GEMM on tcgen05 / TMEM, fed by TMA, for the MoE expert projections
// ("Routed experts" box: every expert runs one GEMM over the tokens routed to
// it; "SwiGLU MLP" box for the gate/up/down structure).
//
// Formulation (weights as the M operand, tokens as N):
//   D[f, r] = sum_k A[f, k] * B[r, k]
// with A the expert weight rows (nn.Linear [out, in], K contiguous) and B the
// permuted token rows (K contiguous).  One work item is one 128-row weight
// tile of one expert times up to BN token rows of that expert, over the full K.
// A persistent CTA per SM walks items i = blockIdx.x, blockIdx.x + gridDim.x, ...
// Item order inside an expert is weight-tile major and token-chunk minor, so
// the chunks that share a weight tile run at the same time and hit in L2.
//
// Roles (192 threads, one CTA per SM):
//   warp 0      TMA producer (one lane): A and B k-blocks into a STAGES-deep
//               ring of 128B-swizzled shared-memory tiles.
//   warp 1      TMEM allocator; one lane issues tcgen05.mma (M = 128, N = the
//               item's token count rounded up to 16, K = 16 per instruction)
//               into one of two TMEM accumulators.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (each warp its lane
//               quarter), then one of
//     GATEUP  A = 64 gate rows over 64 up rows of the same features; writes
//             h = SiLU(gate) * up as bf16 [rows, ldh];
//     DOWN    scales column r by row_coef[r] (routed_scale * w, or 1 for the
//             shared expert) and adds it into y[row_tok[r], :] (fp32 red.add),
//             which is the un-permute scatter of the combine;
//     LOGITS  stores fp32 router logits [T, E].
// Every mbarrier wait is bounded (2 s); on expiry the kernel records
// MOE_DEVERR_TIMEOUT, drains and returns.
#pragma once

#include "moe_device.cuh"
#include "moe_launch.h"

namespace moe {

enum GemmMode { GEMM_GATEUP = 0, GEMM_DOWN = 1, GEMM_LOGITS = 2 };


template <int MODE, int BN>
struct GemmCfg {
    static constexpr int A_BYTES = 128 * 128;  // 128 rows x 64 bf16
    static constexpr int B_BYTES = BN * 128;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int EPI_STRIDE = 33;  // padded fp32 row of the GATEUP staging tile
    static constexpr int EPI_BYTES = MODE == GEMM_GATEUP ? 128 * EPI_STRIDE * 4 : 0;
    static constexpr int SMEM_LIMIT = 227 * 1024;
    static constexpr int MISC_BYTES = 1024;  // barriers, TMEM slot, flags
    static constexpr int STAGES_FIT = (SMEM_LIMIT - 1024 - EPI_BYTES - MISC_BYTES) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
    static constexpr int TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + MISC_BYTES;
    static_assert(STAGES >= 2, "pipeline needs two stages");
    static_assert(BN % 32 == 0 && BN <= 256, "BN");
};

struct Item {
    int g, m, row0, nvalid, K;
    bool shared;
};

template <int BN>
__device__ __forceinline__ Item decode_item(const GemmArgs& P, int i) {
    Item it;
    if (P.item_off == nullptr) {
        int nch = (P.n_rows_single + BN - 1) / BN;
        it.g = 0;
        it.m = i / nch;
        int c = i - it.m * nch;
        it.row0 = c * BN;
        it.nvalid = min(BN, P.n_rows_single - c * BN);
        it.shared = false;
        it.K = P.K_routed;
        return it;
    }
    int lo = 0, hi = P.n_groups - 1;  // largest g with item_off[g] <= i
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (__ldg(&P.item_off[mid]) <= i) lo = mid;
        else hi = mid - 1;
    }
    it.g = lo;
    int local = i - __ldg(&P.item_off[lo]);
    int r0 = __ldg(&P.row_off[lo]);
    int ng = __ldg(&P.row_off[lo + 1]) - r0;
    int nch = (ng + BN - 1) / BN;
    it.m = local / nch;
    int c = local - it.m * nch;
    it.row0 = r0 + c * BN;
    it.nvalid = min(BN, ng - c * BN);
    it.shared = lo >= P.n_routed;
    it.K = it.shared ? P.K_shared : P.K_routed;
    return it;
}

template <int MODE, int BN>
__global__ void __launch_bounds__(192, 1) moe_gemm_kernel(const __grid_constant__ GemmArgs P) {
    using C = GemmCfg<MODE, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    float* epi = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES + C::EPI_BYTES);
    uint64_t* full = bars;
    uint64_t* empty = bars + C::STAGES;
    uint64_t* tfull = bars + 2 * C::STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* epi_ok = reinterpret_cast<volatile int*>(tmem_slot + 2);  // [2], epilogue wait result

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&P.a0);
        tma_prefetch_desc(&P.b);
        if (MODE != GEMM_LOGITS) tma_prefetch_desc(&P.s0);
        if (MODE == GEMM_GATEUP) {
            tma_prefetch_desc(&P.a1);
            tma_prefetch_desc(&P.s1);
        }
    }
    if (warp == 1) tmem_alloc<C::TMEM_COLS>(tmem_slot);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    int total;
    if (P.item_off == nullptr) total = P.mt_routed * ((P.n_rows_single + BN - 1) / BN);
    else total = __ldg(&P.item_off[P.n_groups]);

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            const uint64_t pol_w = l2_policy_evict_first();
            const uint64_t pol_x = l2_policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            for (int i = blockIdx.x; i < total; i += gridDim.x) {
                const Item it = decode_item<BN>(P, i);
                const int KB = it.K / 64;
                int arow;
                if (MODE == GEMM_GATEUP) arow = (it.shared ? 0 : it.g * P.rows_per_expert) + it.m * 64;
                else arow = (it.shared ? 0 : it.g * P.rows_per_expert) + it.m * 128;
                const CUtensorMap* ma = it.shared ? &P.s0 : &P.a0;
                const CUtensorMap* mu = it.shared ? &P.s1 : &P.a1;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
                    uint8_t* sa = ring + stage * C::STAGE_BYTES;
                    uint8_t* sb = sa + C::A_BYTES;
                    mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
                    if (MODE == GEMM_GATEUP) {
                        tma_load_2d(sa, ma, kb * 64, arow, &full[stage], pol_w);
                        tma_load_2d(sa + 64 * 128, mu, kb * 64, arow, &full[stage], pol_w);
                    } else {
                        tma_load_2d(sa, ma, kb * 64, arow, &full[stage], pol_w);
                    }
                    tma_load_2d(sb, &P.b, kb * 64, it.row0, &full[stage], pol_x);
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool issued = false;
            for (int i = blockIdx.x; i < total; i += gridDim.x) {
                const Item it = decode_item<BN>(P, i);
                const int KB = it.K / 64;
                uint32_t n_mma = (uint32_t)((it.nvalid + 15) & ~15);
                n_mma = n_mma < 16u ? 16u : n_mma;
                const uint32_t idesc = idesc_bf16_f32(128, n_mma);
                if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(ring + stage * C::STAGE_BYTES);
                    const uint64_t adesc = smem_desc_sw128(a_addr);
                    const uint64_t bdesc = smem_desc_sw128(a_addr + C::A_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16(d_tmem, adesc + 2ull * k, bdesc + 2ull * k, idesc, (kb | k) != 0 ? 1u : 0u);
                    mma_commit(&empty[stage]);
                    issued = true;
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (*abort_flag && issued) {
                // let every MMA already issued finish before TMEM is released
                mma_commit(drain);
                volatile int dummy = 0;
                mbar_wait_bounded(drain, 0, &dummy, 100000000ull);
            }
        }
    } else {
        // ---------------------------------------------------- epilogue
        const int q = warp & 3;          // TMEM lane quarter this warp may read
        const int et = threadIdx.x - 64; // 0..127
        int acc = 0;
        uint32_t acc_phase = 0;
        int n_done = 0;
        for (int i = blockIdx.x; i < total; i += gridDim.x, ++n_done) {
            const Item it = decode_item<BN>(P, i);
            // one thread waits, all four warps take the same decision (the
            // GATEUP epilogue synchronises the four warps by named barrier)
            if (et == 0) epi_ok[n_done & 1] = mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag) ? 1 : 0;
            named_bar_sync(1, 128);
            if (!epi_ok[n_done & 1]) break;
            tc_fence_after();
            const uint32_t tacc = tmem_base + (uint32_t)(acc * BN) + ((uint32_t)(q * 32) << 16);
            for (int c0 = 0; c0 < it.nvalid; c0 += 32) {
                float v[32];
                tmem_ld32(tacc + (uint32_t)c0, v);
                if (MODE == GEMM_GATEUP) {
                    // stage [128 lanes][32 cols]: lanes 0-63 gate, 64-127 up
                    float* row = epi + (q * 32 + lane) * C::EPI_STRIDE;
#pragma unroll
                    for (int j = 0; j < 32; ++j) row[j] = v[j];
                    named_bar_sync(1, 128);
                    const int jj = et >> 2;          // token column within the chunk
                    const int f0 = (et & 3) * 16;    // 16 features
                    const int j = c0 + jj;
                    if (j < it.nvalid) {
                        uint32_t packed[8];
#pragma unroll
                        for (int ff = 0; ff < 16; ff += 2) {
                            float g0 = epi[(f0 + ff) * C::EPI_STRIDE + jj];
                            float g1 = epi[(f0 + ff + 1) * C::EPI_STRIDE + jj];
                            float u0 = epi[(64 + f0 + ff) * C::EPI_STRIDE + jj];
                            float u1 = epi[(64 + f0 + ff + 1) * C::EPI_STRIDE + jj];
                            float h0 = g0 / (1.0f + __expf(-g0)) * u0;
                            float h1 = g1 / (1.0f + __expf(-g1)) * u1;
                            __nv_bfloat162 p2 = __floats2bfloat162_rn(h0, h1);
                            packed[ff >> 1] = *reinterpret_cast<uint32_t*>(&p2);
                        }
                        __nv_bfloat16* dst = P.h + (size_t)(it.row0 + j) * P.ldh + it.m * 64 + f0;
                        uint4* d4 = reinterpret_cast<uint4*>(dst);
                        d4[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                        d4[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
                    }
                    named_bar_sync(1, 128);
                } else if (MODE == GEMM_DOWN) {
                    const int f = it.m * 128 + q * 32 + lane;
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const int j = c0 + jj;
                        if (j < it.nvalid) {
                            const int r = it.row0 + j;
                            const float cf = __ldg(&P.row_coef[r]);
                            const int t = __ldg(&P.row_tok[r]);
                            atomicAdd(&P.y[(size_t)t * P.ldy + f], v[jj] * cf);
                        }
                    }
                } else {
                    const int e = it.m * 128 + q * 32 + lane;
                    if (e < P.n_logit_cols) {
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            const int j = c0 + jj;
                            if (j < it.nvalid) P.logits[(size_t)(it.row0 + j) * P.n_logit_cols + e] = v[jj];
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc<C::TMEM_COLS>(tmem_base);
    }
}

}  // namespace moe
