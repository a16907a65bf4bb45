// FP8 grouped GEMM on CTA pairs: the e4m3 expert projections with the pages'
// fp32 promotion every 128 K elements ("Teardown: DeepSeek-V3", section 10),
// for wide token tiles.
//
// Each CTA of a pair holds 128 weight rows, the 2-SM MMA (M = 256, N <= 128,
// kind::f8f6f4, K = 32 per instruction) reads both CTAs' rows and both halves
// of the token rows, and each 128-element K block lands as a fresh fp32
// partial in one of four TMEM buffers of both CTAs.  The epilogue warps of
// each CTA promote it into register accumulators with the weight block scale
// and the token rows' activation scales (64 accumulators per thread: no
// spills at 128 token rows per item).
//   GATEUP  rows 0-63 = gate, 64-127 = up of this CTA's 64 features (the pair
//           covers 128 features = one h scale block).  After the last K block:
//           h = SiLU(gate) * up, the per-token amax over the block's 128
//           features (64 here, 64 in the peer CTA, exchanged through
//           distributed shared memory with a remote mbarrier arrive), scale
//           = amax / 448, e4m3 codes [rows, ldh] and scales [ldh/128][rows].
//   DOWN    128 output rows per CTA (256 per item); y[row_tok[r]] +=
//           row_coef[r] * D (fp32 red.add).
// Waits are bounded; the peer exchange wait too.
#pragma once

#include "moe_gemm2.cuh"
#include "moe_gemm_fp8.cuh"

namespace moe {

constexpr int PAIR8_BN = 128;  // token rows per item (whole pair)
// Warps 0, 2, 3: TMA producers; warp 1: TMEM allocator and MMA issuer; warps 4-11:
// eight promotion warps, two per TMEM lane quarter, each promoting 64 of the 128
// token columns.  (Sixteen warps of 32 columns read TMEM faster but ran the layer
// 15-25 % slower: per-block overheads doubled and registers dropped to 96.)
constexpr int PAIR8_EPI_WARPS = 8;
constexpr int PAIR8_NGRP = PAIR8_EPI_WARPS / 4;            // column groups
constexpr int PAIR8_NCH = PAIR8_BN / (32 * PAIR8_NGRP);    // 32-column chunks per warp
constexpr int PAIR8_EPI_BEGIN = 4;
constexpr int PAIR8_THREADS = 32 * (PAIR8_EPI_BEGIN + PAIR8_EPI_WARPS);
static_assert((PAIR8_NCH == 1 || PAIR8_NCH == 2) && PAIR8_NGRP * PAIR8_NCH * 32 == PAIR8_BN, "column split");

struct Gemm2Fp8Cfg {
    static constexpr int A_BYTES = 128 * 128;                 // 128 rows x 128 e4m3
    static constexpr int B_BYTES = PAIR8_BN / 2 * 128;        // this CTA's 64 token rows
    static_assert(B_BYTES % (PAIR_BOX_ROWS * 128) == 0, "B tile holds whole boxes");
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;     // 24 KB
    static constexpr int STAGES = 7;
    static constexpr int XUP_STRIDE = PAIR8_NCH * 32 + 1;     // padded [feature][column] fp32
    static constexpr int XUP_BYTES = PAIR8_NGRP * 64 * XUP_STRIDE * 4;  // up sums handed to the gate warps
    static constexpr int MISC_BYTES = 6144;
    static constexpr int NUM_P = 4;                           // TMEM partial buffers
    static constexpr int P_COLS = PAIR8_BN;
    static constexpr int TMEM_COLS = 512;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + XUP_BYTES + MISC_BYTES;
    static_assert(NUM_P * P_COLS <= TMEM_COLS, "TMEM");
    static_assert(SMEM_BYTES <= 227 * 1024, "smem");
};

__device__ __forceinline__ void mma2_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void st_cluster_f32(uint32_t addr_cluster, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr_cluster), "f"(v) : "memory");
}

// Wait (bounded) on a local mbarrier whose arrivals come from the peer CTA:
// acquire at cluster scope so the peer's stores before its arrive are visible.
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                          uint64_t limit_ns = 2000000000ull) {
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        if (ok) return true;
        if (it == 0) t0 = global_timer_ns();
        if ((it & 63u) == 63u) {
            if (*abort) return false;
            if (global_timer_ns() - t0 > limit_ns) {
                set_dev_error(MOE_DEVERR_TIMEOUT);
                *abort = 1;
                return false;
            }
        }
    }
}

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PAIR8_THREADS, 1)
    moe_gemm2_fp8_kernel(const __grid_constant__ GemmArgs P) {
    using C = Gemm2Fp8Cfg;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    float* xup = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES);  // [2 groups][64][65]
    uint8_t* misc = smem + C::STAGES * C::STAGE_BYTES + C::XUP_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(misc);
    uint64_t* full = bars;                       // leader: stage loaded (both CTAs' bytes)
    uint64_t* empty = full + C::STAGES;          // both: stage consumed
    uint64_t* pfull = empty + C::STAGES;         // both: partial written
    uint64_t* pempty = pfull + C::NUM_P;         // leader: partial promoted by both CTAs
    uint64_t* xbar = pempty + C::NUM_P;          // both: [2 parity][groups] peer's column maxima arrived
    uint64_t* drain = xbar + 2 * PAIR8_NGRP;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* warp_ok = reinterpret_cast<volatile int*>(tmem_slot + 2);  // [epilogue warps]
    constexpr int GCOLS = PAIR8_NCH * 32;                     // columns of one warp
    float* sc_rows = reinterpret_cast<float*>(misc + 512);    // [epilogue warps][GCOLS] scales of a K block
    float* cmax = reinterpret_cast<float*>(misc + 2560);      // [groups][chunks][2 gate warps][32] column maxima
    float* xmax = reinterpret_cast<float*>(misc + 3584);      // [2 parity][groups][GCOLS] peer's column maxima
    float* sinv = reinterpret_cast<float*>(misc + 4608);      // [groups][GCOLS] inverse scales
    static_assert(PAIR8_EPI_WARPS * GCOLS * 4 <= 2048 && PAIR8_NGRP * GCOLS * 2 * 4 <= 1024 &&
                      2 * PAIR8_NGRP * GCOLS * 4 <= 1024 && PAIR8_NGRP * GCOLS * 4 <= 1024,
                  "misc layout");
    static_assert((2 * C::STAGES + 2 * C::NUM_P + 2 * PAIR8_NGRP + 1) * 8 + 8 + 4 * PAIR8_EPI_WARPS <= 512,
                  "barriers and flags");

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], MODE == GEMM_GATEUP ? 3 : 2);  // the leader's producers of the stage
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < C::NUM_P; ++a) {
            mbar_init(&pfull[a], 1);
            mbar_init(&pempty[a], 2 * PAIR8_EPI_WARPS);
        }
        for (int a = 0; a < 2 * PAIR8_NGRP; ++a) mbar_init(&xbar[a], 1);  // the peer's q0 warp of the group arrives
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&P.a0);
        tma_prefetch_desc(&P.b);
        tma_prefetch_desc(&P.s0);
        if (MODE == GEMM_GATEUP) {
            tma_prefetch_desc(&P.a1);
            tma_prefetch_desc(&P.s1);
        }
    }
    if (warp == 1) tmem_alloc_pair(tmem_slot);
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int total = __ldg(&P.item_off[P.n_groups]);
    const int cluster_id = blockIdx.x >> 1;
    const int n_clusters = gridDim.x >> 1;

    if (warp == 0 || warp == 2 || warp == 3) {
        // ------------------------------------------------ TMA producers (both CTAs)
        // Three issuing warps, each with its own share of every stage: warp 0 the
        // gate rows (GATEUP) or the whole weight tile (DOWN), warp 2 the up rows
        // (GATEUP), warp 3 the token rows.  One thread issues a TMA instruction
        // every few hundred cycles whatever its size, so one thread per operand.
        const int role = warp == 0 ? 0 : warp - 1;  // 0 A/gate, 1 up, 2 B
        if (lane == 0 && !(MODE == GEMM_DOWN && role == 1)) {
            const uint64_t pol_w = l2_policy_evict_first();
            const uint64_t pol_keep = l2_policy_evict_normal();
            const uint64_t pol_x = l2_policy_evict_last();
            const uint32_t full0 = mapa_shared(smem_u32(&full[0]), 0);
            int stage = 0;
            uint32_t phase = 0;
            for (int i = cluster_id; i < total; i += n_clusters) {
                const Item it = decode_item<PAIR8_BN>(P, i);
                // weights read by several items stay in L2 for the others; the rest stream
                const uint64_t pw = it.nch > 1 ? pol_keep : pol_w;
                const int KB = it.K / 128;
                const int nh = ((it.nvalid + 31) & ~31) / 2;
                const int nbox = (nh + PAIR_BOX_ROWS - 1) / PAIR_BOX_ROWS;
                // bytes this role brings into the stage, both CTAs together
                const uint32_t bytes = role == 2 ? 2u * (uint32_t)(nbox * PAIR_BOX_ROWS * 128)
                                       : MODE == GEMM_GATEUP ? 2u * 64u * 128u : 2u * (uint32_t)C::A_BYTES;
                const int base = it.shared ? 0 : it.g * P.rows_per_expert;
                const int brow = it.row0 + (int)rank * nh;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
                    uint8_t* sa = ring + stage * C::STAGE_BYTES;
                    uint8_t* sb = sa + C::A_BYTES;
                    const uint32_t fb = full0 + (uint32_t)(stage * 8);
                    if (leader) mbar_arrive_expect_tx(&full[stage], bytes);
                    if (role == 2) {
                        for (int bx = 0; bx < nbox; ++bx)
                            tma_load_2d_pair(sb + bx * PAIR_BOX_ROWS * 128, &P.b, kb * 128, brow + bx * PAIR_BOX_ROWS,
                                             fb, pol_x);
                    } else if (MODE == GEMM_GATEUP) {
                        // 64 gate rows over 64 up rows of this CTA's 64 features
                        const int r = base + it.m * 128 + (int)rank * 64;
                        if (role == 0) tma_load_2d_pair(sa, it.shared ? &P.s0 : &P.a0, kb * 128, r, fb, pw);
                        else tma_load_2d_pair(sa + 64 * 128, it.shared ? &P.s1 : &P.a1, kb * 128, r, fb, pw);
                    } else {
                        tma_load_2d_pair(sa, it.shared ? &P.s0 : &P.a0, kb * 128, base + it.m * 256 + (int)rank * 128,
                                         fb, pw);
                    }
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------------------------ 2-SM MMA issuer: one partial per K block
            int stage = 0;
            uint32_t phase = 0;
            int pb = 0;
            uint32_t pb_phase = 0;
            bool issued = false, ok = true;
            for (int i = cluster_id; i < total && ok; i += n_clusters) {
                const Item it = decode_item<PAIR8_BN>(P, i);
                const int KB = it.K / 128;
                const uint32_t n_mma = (uint32_t)((it.nvalid + 31) & ~31);
                const uint32_t idesc = idesc_e4m3_f32(256, n_mma);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(&pempty[pb], pb_phase ^ 1u, abort_flag)) { ok = false; break; }
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d = tmem_base + (uint32_t)(pb * C::P_COLS);
                    const uint32_t a_addr = smem_u32(ring + stage * C::STAGE_BYTES);
                    const uint64_t adesc = smem_desc_sw128(a_addr);
                    const uint64_t bdesc = smem_desc_sw128(a_addr + C::A_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k) mma2_e4m3(d, adesc + 2ull * k, bdesc + 2ull * k, idesc, k != 0 ? 1u : 0u);
                    mma2_commit_pair(&empty[stage], 0x3);
                    mma2_commit_pair(&pfull[pb], 0x3);
                    issued = true;
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
                    if (++pb == C::NUM_P) { pb = 0; pb_phase ^= 1u; }
                }
            }
            if (*abort_flag && issued) {
                mma2_commit_local(drain);
                volatile int dummy = 0;
                mbar_wait_bounded(drain, 0, &dummy, 100000000ull);
            }
        }
    } else if (warp >= PAIR8_EPI_BEGIN) {
        // ---------------------------------------------------- epilogue: promotion + final (both CTAs)
        constexpr int NCH = PAIR8_NCH, NGRP = PAIR8_NGRP;
        const int wi = warp - PAIR8_EPI_BEGIN;
        const int q = wi & 3;                   // TMEM lane quarter (warp % 4): rows q*32 .. q*32+31
        const int grp = wi >> 2;                // column group: chunks c0 = 32*grp + 32*NGRP*c
        float* my_sc = sc_rows + wi * GCOLS;
        const uint32_t pempty0 = mapa_shared(smem_u32(&pempty[0]), 0);
        const uint32_t xmax_peer = mapa_shared(smem_u32(xmax), rank ^ 1u);
        const uint32_t xbar_peer = mapa_shared(smem_u32(&xbar[0]), rank ^ 1u);
        int pb = 0;
        uint32_t pb_phase = 0;
        uint32_t x_phase[2] = {0u, 0u};
        int n_item = 0;
        bool alive = true;
        for (int i = cluster_id; i < total && alive; i += n_clusters, ++n_item) {
            const Item it = decode_item<PAIR8_BN>(P, i);
            const int KB = it.K / 128;
            const int a_rb = it.shared ? P.a_rb_shared : P.a_rb_routed;
            // this thread's weight-scale matrix and 128-row block
            const float* sa;
            int rb;
            if (MODE == GEMM_GATEUP) {
                sa = q < 2 ? (it.shared ? P.ss0 : P.sa0) : (it.shared ? P.ss1 : P.sa1);
                rb = it.m;  // the pair's 128 features are one 128-row block of W_gate / W_up
            } else {
                sa = it.shared ? P.ss0 : P.sa0;
                rb = 2 * it.m + (int)rank;
            }
            const size_t sbase = it.shared ? 0 : (size_t)it.g * a_rb;
            const bool any = 32 * grp < it.nvalid;  // warp-uniform: this warp has columns
            float acc[NCH][32];
#pragma unroll
            for (int c = 0; c < NCH; ++c)
#pragma unroll
                for (int j = 0; j < 32; ++j) acc[c][j] = 0.0f;
            auto load_scales = [&](int kb, float& w, float (&xs)[NCH]) {
                w = rb < a_rb ? __ldg(&sa[(sbase + rb) * KB + kb]) : 0.0f;
#pragma unroll
                for (int c = 0; c < NCH; ++c) {
                    const int col = 32 * grp + 32 * NGRP * c + lane;
                    xs[c] = col < it.nvalid ? __ldg(&P.sbT[(size_t)kb * P.sb_ld + it.row0 + col]) : 0.0f;
                }
            };
            float nw, nxs[NCH];
            load_scales(0, nw, nxs);
            for (int kb = 0; kb < KB; ++kb) {
                // this block's scales were loaded one block ahead; the next block's go out now
                const float sw = nw;
                float xs[NCH];
#pragma unroll
                for (int c = 0; c < NCH; ++c) xs[c] = nxs[c];
                if (kb + 1 < KB) load_scales(kb + 1, nw, nxs);
                if (!mbar_wait_bounded(&pfull[pb], pb_phase, abort_flag)) { alive = false; break; }
                tc_fence_after();
                const uint32_t t0 = tmem_base + (uint32_t)(pb * C::P_COLS) + ((uint32_t)(q * 32) << 16);
                if (any) {
#pragma unroll
                    for (int c = 0; c < NCH; ++c) my_sc[c * 32 + lane] = sw * xs[c];
                    __syncwarp();
                    // every chunk of the warp's columns in one go (columns past the item's
                    // rows hold stale sums of this buffer and are not used)
                    float p[NCH][32];
                    if constexpr (NCH == 2) tmem_ld32x2(t0 + (uint32_t)(32 * grp), t0 + (uint32_t)(32 * grp + 32 * NGRP), p[0], p[1]);
                    else tmem_ld32(t0 + (uint32_t)(32 * grp), p[0]);
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
#pragma unroll
                        for (int c = 0; c < NCH; ++c) {
                            if (c == 0 || 32 * grp + 32 * NGRP * c < it.nvalid) {
                                const float4 sv = *reinterpret_cast<const float4*>(my_sc + c * 32 + j);
                                fma2(acc[c][j + 0], acc[c][j + 1], p[c][j + 0], p[c][j + 1], sv.x, sv.y);
                                fma2(acc[c][j + 2], acc[c][j + 3], p[c][j + 2], p[c][j + 3], sv.z, sv.w);
                            }
                        }
                    }
                    __syncwarp();  // my_sc is rewritten for the next block
                }
                // the partial is promoted: hand the buffer back to the MMA issuer (handing it
                // back right after the TMEM load, before the FMAs, measured the same)
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(pempty0 + (uint32_t)(pb * 8));
                if (++pb == C::NUM_P) { pb = 0; pb_phase ^= 1u; }
            }

            if (MODE == GEMM_GATEUP) {
                // the rest synchronises the group's four warps: agree that none gave up
                if (lane == 0) warp_ok[wi] = alive ? 1 : 0;
                named_bar_sync(2 + grp, 128);
                alive = warp_ok[4 * grp] && warp_ok[4 * grp + 1] && warp_ok[4 * grp + 2] && warp_ok[4 * grp + 3];
                if (!alive) break;
                const int par = n_item & 1;
                // (1) up sums (TMEM quarters 2, 3) -> the gate warps (quarters 0, 1) of the same features
                float* xg = xup + grp * 64 * C::XUP_STRIDE;
                if (q >= 2) {
                    const int fl = (q - 2) * 32 + lane;
#pragma unroll
                    for (int c = 0; c < NCH; ++c)
#pragma unroll
                        for (int j = 0; j < 32; ++j) xg[fl * C::XUP_STRIDE + c * 32 + j] = acc[c][j];
                }
                named_bar_sync(2 + grp, 128);
                // (2) h = SiLU(gate) * up; per-warp column maxima over its 32 features
                float* cm = cmax + grp * (NCH * 2 * 32);  // [chunks][2 gate warps][32 columns]
                if (q < 2) {
                    const int fl = q * 32 + lane;
#pragma unroll
                    for (int c = 0; c < NCH; ++c) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) acc[c][j] = silu_mul(acc[c][j], xg[fl * C::XUP_STRIDE + c * 32 + j]);
                        float m[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) m[j] = fabsf(acc[c][j]);
#pragma unroll
                        for (int off = 16; off >= 1; off >>= 1) {  // lane l ends with column l
                            const bool upper = (lane & off) != 0;
#pragma unroll
                            for (int j = 0; j < off; ++j) {
                                const float send = upper ? m[j] : m[j + off];
                                const float keep = upper ? m[j + off] : m[j];
                                m[j] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, off));
                            }
                        }
                        cm[(c * 2 + q) * 32 + lane] = m[0];
                    }
                }
                named_bar_sync(2 + grp, 128);
                // (3) the block's 128 features span both CTAs: exchange the 64-feature
                //     maxima with the peer, then scale = amax / 448 per token row
                if (q == 0) {
                    float lm[NCH];
#pragma unroll
                    for (int c = 0; c < NCH; ++c) {
                        lm[c] = fmaxf(cm[(c * 2) * 32 + lane], cm[(c * 2 + 1) * 32 + lane]);
                        st_cluster_f32(xmax_peer + (uint32_t)(((par * NGRP + grp) * GCOLS + c * 32 + lane) * 4), lm[c]);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster_release(xbar_peer + (uint32_t)((par * NGRP + grp) * 8));
                    const bool got = mbar_wait_cluster_bounded(&xbar[par * NGRP + grp], x_phase[par], abort_flag);
                    float* si = sinv + grp * GCOLS;
#pragma unroll
                    for (int c = 0; c < NCH; ++c) {
                        const float amax = got ? fmaxf(lm[c], xmax[(par * NGRP + grp) * GCOLS + c * 32 + lane]) : 0.0f;
                        const float scale = amax > 0.0f ? amax / 448.0f : 1.0f;
                        si[c * 32 + lane] = 1.0f / scale;
                        const int col = 32 * grp + 32 * NGRP * c + lane;
                        if (leader && col < it.nvalid) P.hsT[(size_t)it.m * P.hs_ld + it.row0 + col] = scale;
                    }
                    if (lane == 0) warp_ok[wi] = got ? 1 : 0;
                }
                x_phase[par] ^= 1u;
                named_bar_sync(2 + grp, 128);
                if (!warp_ok[4 * grp]) { alive = false; break; }  // the group's q0 warp
                // (4) e4m3 codes of h, one byte per (token row, feature)
                if (q < 2) {
                    const int f = it.m * 128 + (int)rank * 64 + q * 32 + lane;
                    const float* si = sinv + grp * GCOLS;
#pragma unroll
                    for (int c = 0; c < NCH; ++c) {
                        const int c0 = 32 * grp + 32 * NGRP * c;
                        if (c0 < it.nvalid) {
                            uint8_t* dst = P.hq + (size_t)(it.row0 + c0) * P.ldh + f;
#pragma unroll
                            for (int j = 0; j < 32; j += 2) {
                                const uint32_t pk = cvt_e4m3x2(acc[c][j + 1] * si[c * 32 + j + 1], acc[c][j] * si[c * 32 + j]);
                                if (c0 + j < it.nvalid) dst[(size_t)j * P.ldh] = (uint8_t)(pk & 0xff);
                                if (c0 + j + 1 < it.nvalid) dst[(size_t)(j + 1) * P.ldh] = (uint8_t)(pk >> 8);
                            }
                        }
                    }
                }
                named_bar_sync(2 + grp, 128);   // cm / sinv / xup are reused by the next item
            }
            if (!alive) break;

            if (MODE == GEMM_DOWN) {
                const int f = it.m * 256 + (int)rank * 128 + q * 32 + lane;
                const bool okf = f < P.ldy;
#pragma unroll
                for (int c = 0; c < NCH; ++c) {
                    const int c0 = 32 * grp + 32 * NGRP * c;
                    if (c0 < it.nvalid) {
                        // this lane's permuted row, handed to the other lanes by shuffles
                        const bool okr = c0 + lane < it.nvalid;
                        const float cf_l = okr ? __ldg(&P.row_coef[it.row0 + c0 + lane]) : 0.0f;
                        int tok_l = okr ? __ldg(&P.row_tok[it.row0 + c0 + lane]) : 0;
                        // checking build: the token's y row exists (else the row is skipped)
                        if (kDebugChecks && okr && !dbg_ok((unsigned)tok_l < (unsigned)P.y_rows)) tok_l = -1;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float cf = __shfl_sync(0xffffffffu, cf_l, j);
                            const int tok = __shfl_sync(0xffffffffu, tok_l, j);
                            if (c0 + j < it.nvalid && (!kDebugChecks || tok >= 0)) {
                                float* yr = P.y + (size_t)tok * P.ldy;
                                if (okf) atomicAdd(yr + f, acc[c][j] * cf);
                            }
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base);
    }
}

}  // namespace moe
