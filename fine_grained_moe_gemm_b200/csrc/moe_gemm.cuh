// Grouped GEMM on tcgen05 / TMEM, fed by TMA, for the MoE expert projections
// ("Routed experts" box: every expert runs one GEMM over the tokens routed to
// it; "SwiGLU MLP" box for the gate/up/down structure).
//
// Formulation (weights as the M operand, tokens as N):
//   D[f, r] = sum_k A[f, k] * B[r, k]
// with A the expert weight rows (nn.Linear [out, in], K contiguous) and B the
// permuted token rows (K contiguous).  One work item is 256 weight rows (two
// 128-row tiles, two accumulators) of one expert times up to BN token rows of
// that expert, over the full K.  Two tiles against one token tile halve the
// L2 -> SM traffic of the token rows, which every weight tile of the expert
// re-reads.  The token rows of an item are loaded in 32-row boxes, only as
// many as the item has, so BN can cover a whole expert at prefill sizes.
// A persistent CTA per SM walks items i = blockIdx.x, blockIdx.x + gridDim.x, ...
// Item order inside an expert is weight-block major and token-chunk minor, so
// chunks that share weights run at the same time and hit in L2.
//
// Roles (320 threads, one CTA per SM):
//   warp 0      TMA producer (one lane): A and B k-blocks into a STAGES-deep
//               ring of 128B-swizzled shared-memory tiles.
//   warp 1      TMEM allocator; one lane issues tcgen05.mma (M = 128 twice,
//               N = the item's row count rounded up to 16, K = 16 per
//               instruction) into the item's accumulator pair.
//   warps 2-9   epilogue, two groups of four (a warp reads the TMEM lane
//               quarter warp % 4; the groups split the columns):
//     GATEUP  tile 0 = gate rows, tile 1 = up rows of the same 128 features:
//             h = SiLU(gate) * up, written as bf16 [rows, ldh];
//     DOWN    tiles 0/1 = 256 output features; column r is scaled by
//             row_coef[r] (routed_scale * w, or 1 for the shared expert) and
//             added into y[row_tok[r], :] (fp32 red.add): the combine's
//             un-permute scatter;
//     LOGITS  tiles 0/1 = experts 0-255; stores fp32 router logits [T, E], or,
//             with K split over several items, one partial per split (summed
//             in a fixed order by the selection kernel).
// Every mbarrier wait is bounded (2 s); on expiry the kernel records
// MOE_DEVERR_TIMEOUT, drains and returns.
#pragma once

#include "moe_device.cuh"
#include "moe_launch.h"

namespace moe {

enum GemmMode { GEMM_GATEUP = 0, GEMM_DOWN = 1, GEMM_LOGITS = 2 };

constexpr int GEMM_THREADS = 320;
constexpr int GEMM_EPI_THREADS = 256;
constexpr int B_BOX_ROWS = 32;

template <int MODE, int BN>
struct GemmCfg {
    static constexpr int A_TILE = 128 * 128;        // 128 rows x 64 bf16
    static constexpr int A_BYTES = 2 * A_TILE;      // two tiles
    static constexpr int B_BYTES = BN * 128;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int SMEM_LIMIT = 227 * 1024;
    static constexpr int MISC_BYTES = 1024;         // barriers, TMEM slot, flags
    static constexpr int STAGES_FIT = (SMEM_LIMIT - 1024 - MISC_BYTES) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
    static constexpr int ACC_COLS = 2 * BN;         // [tile 0: BN cols][tile 1: BN cols]
    static constexpr int NUM_ACC = 2 * ACC_COLS <= 512 ? 2 : 1;
    static constexpr int TMEM_NEED = NUM_ACC * ACC_COLS;
    static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                     : TMEM_NEED <= 256 ? 256 : 512;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + MISC_BYTES;
    static_assert(STAGES >= 2, "pipeline needs two stages");
    static_assert(BN % 32 == 0 && BN <= 256, "BN");
    static_assert(TMEM_NEED <= 512, "TMEM");
};

struct Item {
    int g, m, row0, nvalid, K;
    int split, n_splits;  // K range of the item: blocks [split, split+1) * KB / n_splits
    int nch;              // token chunks of the item's group: > 1, its weight tiles are read again
    bool shared;
};

// First and one-past-last K block of an item with KB blocks in all.
__device__ __forceinline__ int item_kb0(const Item& it, int KB) { return it.split * KB / it.n_splits; }
__device__ __forceinline__ int item_kb1(const Item& it, int KB) { return (it.split + 1) * KB / it.n_splits; }

template <int BN>
__device__ __forceinline__ Item decode_item(const GemmArgs& P, int i) {
    Item it;
    if (P.item_off == nullptr) {
        int nch = (P.n_rows_single + BN - 1) / BN;
        it.n_splits = P.k_splits > 1 ? P.k_splits : 1;
        it.split = i % it.n_splits;
        i /= it.n_splits;
        it.g = 0;
        it.m = i / nch;
        int c = i - it.m * nch;
        it.row0 = c * BN;
        it.nvalid = min(BN, P.n_rows_single - c * BN);
        it.nch = nch;
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
    it.shared = lo >= P.n_routed;
    // k_splits > 1 (DOWN of a schedule with few tiles): each (tile, split) pair is one
    // item; the splits of a tile add their partial sums into y by the same atomics
    it.n_splits = P.k_splits > 1 ? P.k_splits : 1;
    int local = i - __ldg(&P.item_off[lo]);
    int r0 = __ldg(&P.row_off[lo]);
    int ng = __ldg(&P.row_off[lo + 1]) - r0;
    // checking build: a group that owns items has rows (else the chunk count below is 0)
    if (kDebugChecks && P.rows_cap > 0 && !dbg_ok(ng > 0)) ng = 1;
    int nch = (ng + BN - 1) / BN;
    it.nch = nch;
    // item order inside the group: weight tile, split, then token chunk (the chunks of a
    // weight slice run together), or, chunk-major, token chunk first (a chunk's tiles run
    // together and the token rows stay in L2 while the weight tiles come around again)
    int c, ms;
    if (P.chunk_major) {
        const int nms = (it.shared ? P.mt_shared : P.mt_routed) * it.n_splits;
        c = local / nms;
        ms = local - c * nms;
    } else {
        ms = local / nch;
        c = local - ms * nch;
    }
    it.m = ms / it.n_splits;
    it.split = ms - it.m * it.n_splits;
    it.row0 = r0 + c * BN;
    it.nvalid = min(BN, ng - c * BN);
    it.K = it.shared ? P.K_shared : P.K_routed;
    if (kDebugChecks && P.rows_cap > 0) {
        // checking build: the group's rows agree with its item count, the item's rows
        // lie inside the permuted buffers and its weight tile inside the expert
        // (every role decodes the same replacement)
        const int mt = it.shared ? P.mt_shared : P.mt_routed;
        const int n_items = __ldg(&P.item_off[lo + 1]) - __ldg(&P.item_off[lo]);
        dbg_ok(n_items == nch * mt * it.n_splits);
        if (!dbg_ok(it.row0 >= 0 && it.nvalid >= 1 && it.row0 + it.nvalid <= P.rows_cap && it.m >= 0 && it.m < mt)) {
            it.row0 = 0;
            it.nvalid = min(BN, P.rows_cap);
            it.m = 0;
        }
    }
    return it;
}

__device__ __forceinline__ float silu_mul(float g, float u) {
    // SiLU(g) * u with SiLU(z) = z * sigmoid(z) ("SwiGLU MLP" box)
    return g < -80.0f ? 0.0f : __fdividef(g, 1.0f + __expf(-g)) * u;
}

template <int MODE, int BN>
__global__ void __launch_bounds__(GEMM_THREADS, 1) moe_gemm_kernel(const __grid_constant__ GemmArgs P) {
    using C = GemmCfg<MODE, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
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
            mbar_init(&tempty[a], GEMM_EPI_THREADS / 32);
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
    if (P.item_off == nullptr)
        total = P.mt_routed * ((P.n_rows_single + BN - 1) / BN) * (P.k_splits > 1 ? P.k_splits : 1);
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
                const int kb0 = item_kb0(it, it.K / 64), kb1 = item_kb1(it, it.K / 64);
                const int nbox = (it.nvalid + B_BOX_ROWS - 1) / B_BOX_ROWS;
                const uint32_t bytes = C::A_BYTES + nbox * B_BOX_ROWS * 128;
                // A rows of the two tiles
                const CUtensorMap* m0;
                const CUtensorMap* m1;
                int r0, r1;
                const int base = it.shared ? 0 : it.g * P.rows_per_expert;
                if (MODE == GEMM_GATEUP) {  // gate and up rows of the same 128 features
                    m0 = it.shared ? &P.s0 : &P.a0;
                    m1 = it.shared ? &P.s1 : &P.a1;
                    r0 = r1 = base + it.m * 128;
                } else {                    // 256 consecutive rows
                    m0 = m1 = it.shared ? &P.s0 : &P.a0;
                    r0 = base + it.m * 256;
                    r1 = r0 + 128;
                }
                bool ok = true;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
                    uint8_t* sa = ring + stage * C::STAGE_BYTES;
                    uint8_t* sb = sa + C::A_BYTES;
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    tma_load_2d(sa, m0, kb * 64, r0, &full[stage], pol_w);
                    tma_load_2d(sa + C::A_TILE, m1, kb * 64, r1, &full[stage], pol_w);
                    for (int bx = 0; bx < nbox; ++bx)
                        tma_load_2d(sb + bx * B_BOX_ROWS * 128, &P.b, kb * 64, it.row0 + bx * B_BOX_ROWS,
                                    &full[stage], pol_x);
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
                const int kb0 = item_kb0(it, it.K / 64), kb1 = item_kb1(it, it.K / 64);
                uint32_t n_mma = (uint32_t)((it.nvalid + 15) & ~15);
                n_mma = n_mma < 16u ? 16u : n_mma;
                const uint32_t idesc = idesc_bf16_f32(128, n_mma);
                if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag)) break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + (uint32_t)(acc * C::ACC_COLS);
                const uint32_t d1 = d0 + BN;
                bool ok = true;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(ring + stage * C::STAGE_BYTES);
                    const uint64_t adesc0 = smem_desc_sw128(a_addr);
                    const uint64_t adesc1 = smem_desc_sw128(a_addr + C::A_TILE);
                    const uint64_t bdesc = smem_desc_sw128(a_addr + C::A_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t accum = (kb > kb0 || k != 0) ? 1u : 0u;
                        mma_bf16(d0, adesc0 + 2ull * k, bdesc + 2ull * k, idesc, accum);
                        mma_bf16(d1, adesc1 + 2ull * k, bdesc + 2ull * k, idesc, accum);
                    }
                    mma_commit(&empty[stage]);
                    issued = true;
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);
                if (C::NUM_ACC == 2) {
                    acc ^= 1;
                    if (acc == 0) acc_phase ^= 1u;
                } else {
                    acc_phase ^= 1u;
                }
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
        const int q = warp & 3;                  // TMEM lane quarter this warp may read
        const int grp = (warp - 2) >> 2;         // column group: chunks c0 = 32 * (2 i + grp)
        const int et = threadIdx.x - 64;         // 0..255
        int acc = 0;
        uint32_t acc_phase = 0;
        int n_done = 0;
        for (int i = blockIdx.x; i < total; i += gridDim.x, ++n_done) {
            const Item it = decode_item<BN>(P, i);
            // one thread waits, all eight warps take the same decision
            if (et == 0) epi_ok[n_done & 1] = mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag) ? 1 : 0;
            named_bar_sync(1, GEMM_EPI_THREADS);
            if (!epi_ok[n_done & 1]) break;
            tc_fence_after();
            const uint32_t t0 = tmem_base + (uint32_t)(acc * C::ACC_COLS) + ((uint32_t)(q * 32) << 16);
            const uint32_t t1 = t0 + BN;
            for (int c0 = 32 * grp; c0 < it.nvalid; c0 += 64) {
                float v0[32], v1[32];
                // DOWN: this lane's permuted row (routing coefficient and token), handed
                // to the other lanes by shuffles: one load a lane instead of one a column
                float cf_l = 0.0f;
                int tok_l = 0;
                if (MODE == GEMM_DOWN && c0 + lane < it.nvalid) {
                    cf_l = __ldg(&P.row_coef[it.row0 + c0 + lane]);
                    tok_l = __ldg(&P.row_tok[it.row0 + c0 + lane]);
                    // checking build: the token's y row exists (else the row is skipped)
                    if (kDebugChecks && !dbg_ok((unsigned)tok_l < (unsigned)P.y_rows)) tok_l = -1;
                }
                tmem_ld32x2(t0 + (uint32_t)c0, t1 + (uint32_t)c0, v0, v1);
                if (MODE == GEMM_GATEUP) {
                    const int f = it.m * 128 + q * 32 + lane;
                    __nv_bfloat16* dst = P.h + (size_t)(it.row0 + c0) * P.ldh + f;
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj)
                        if (c0 + jj < it.nvalid) dst[(size_t)jj * P.ldh] = __float2bfloat16_rn(silu_mul(v0[jj], v1[jj]));
                } else if (MODE == GEMM_DOWN) {
                    const int f0 = it.m * 256 + q * 32 + lane;
                    const int f1 = f0 + 128;
                    const bool ok0 = f0 < P.ldy, ok1 = f1 < P.ldy;
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const float cf = __shfl_sync(0xffffffffu, cf_l, jj);
                        const int tok = __shfl_sync(0xffffffffu, tok_l, jj);
                        if (c0 + jj < it.nvalid && (!kDebugChecks || tok >= 0)) {
                            float* yr = P.y + (size_t)tok * P.ldy;
                            if (ok0) atomicAdd(yr + f0, v0[jj] * cf);
                            if (ok1) atomicAdd(yr + f1, v1[jj] * cf);
                        }
                    }
                } else {
                    const int e0 = it.m * 256 + q * 32 + lane;
                    const int e1 = e0 + 128;
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        if (c0 + jj < it.nvalid) {
                            float* out = it.n_splits > 1
                                             ? P.part + (size_t)it.split * P.n_rows_single * P.n_logit_cols
                                             : P.logits;
                            float* lr = out + (size_t)(it.row0 + c0 + jj) * P.n_logit_cols;
                            if (e0 < P.n_logit_cols) lr[e0] = v0[jj];
                            if (e1 < P.n_logit_cols) lr[e1] = v1[jj];
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
            if (C::NUM_ACC == 2) {
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            } else {
                acc_phase ^= 1u;
            }
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
