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

struct Gemm2Fp8Cfg {
    static constexpr int A_BYTES = 128 * 128;                 // 128 rows x 128 e4m3
    static constexpr int B_BYTES = PAIR8_BN / 2 * 128;        // this CTA's 64 token rows
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;     // 24 KB
    static constexpr int STAGES = 7;
    static constexpr int XUP_STRIDE = 65;                     // padded [feature][column] fp32
    static constexpr int XUP_BYTES = 2 * 64 * XUP_STRIDE * 4; // up sums handed to the gate warps
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
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GEMM_THREADS, 1)
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
    uint64_t* xbar = pempty + C::NUM_P;          // both: [2 parity][2 groups] peer's column maxima arrived
    uint64_t* drain = xbar + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* warp_ok = reinterpret_cast<volatile int*>(tmem_slot + 2);  // [8]
    float* sc_rows = reinterpret_cast<float*>(misc + 512);    // [8 warps][64]   scales of a K block
    float* cmax = reinterpret_cast<float*>(misc + 2560);      // [2 groups][2 chunks][2 warps][32] column maxima
    float* xmax = reinterpret_cast<float*>(misc + 3584);      // [2 parity][2 groups][64] peer's column maxima
    float* sinv = reinterpret_cast<float*>(misc + 4608);      // [2 groups][64] inverse scales

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < C::NUM_P; ++a) {
            mbar_init(&pfull[a], 1);
            mbar_init(&pempty[a], 2 * GEMM_EPI_THREADS / 32);
        }
        for (int a = 0; a < 4; ++a) mbar_init(&xbar[a], 1);  // the peer's q0 warp of the group arrives
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

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer (both CTAs)
            const uint64_t pol_w = l2_policy_evict_first();
            const uint64_t pol_x = l2_policy_evict_last();
            const uint32_t full0 = mapa_shared(smem_u32(&full[0]), 0);
            int stage = 0;
            uint32_t phase = 0;
            for (int i = cluster_id; i < total; i += n_clusters) {
                const Item it = decode_item<PAIR8_BN>(P, i);
                const int KB = it.K / 128;
                const int nh = ((it.nvalid + 31) & ~31) / 2;
                const int nbox = nh / PAIR_BOX_ROWS;
                const uint32_t bytes = 2u * (uint32_t)(C::A_BYTES + nh * 128);
                const int base = it.shared ? 0 : it.g * P.rows_per_expert;
                const int brow = it.row0 + (int)rank * nh;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
                    uint8_t* sa = ring + stage * C::STAGE_BYTES;
                    uint8_t* sb = sa + C::A_BYTES;
                    const uint32_t fb = full0 + (uint32_t)(stage * 8);
                    if (leader) mbar_arrive_expect_tx(&full[stage], bytes);
                    if (MODE == GEMM_GATEUP) {
                        // 64 gate rows over 64 up rows of this CTA's 64 features
                        const int r = base + it.m * 128 + (int)rank * 64;
                        tma_load_2d_pair(sa, it.shared ? &P.s0 : &P.a0, kb * 128, r, fb, pol_w);
                        tma_load_2d_pair(sa + 64 * 128, it.shared ? &P.s1 : &P.a1, kb * 128, r, fb, pol_w);
                    } else {
                        tma_load_2d_pair(sa, it.shared ? &P.s0 : &P.a0, kb * 128, base + it.m * 256 + (int)rank * 128,
                                         fb, pol_w);
                    }
                    for (int bx = 0; bx < nbox; ++bx)
                        tma_load_2d_pair(sb + bx * PAIR_BOX_ROWS * 128, &P.b, kb * 128, brow + bx * PAIR_BOX_ROWS, fb,
                                         pol_x);
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
    } else {
        // ---------------------------------------------------- epilogue: promotion + final (both CTAs)
        const int q = warp & 3;                 // TMEM lane quarter: rows q*32 .. q*32+31
        const int grp = (warp - 2) >> 2;        // column group: chunks c0 = 32*grp + 64*c
        const int wi = warp - 2;
        float* my_sc = sc_rows + wi * 64;
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
            float acc[2][32];
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int j = 0; j < 32; ++j) acc[c][j] = 0.0f;
            auto load_scales = [&](int kb, float& w, float (&xs)[2]) {
                w = rb < a_rb ? __ldg(&sa[(sbase + rb) * KB + kb]) : 0.0f;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int col = 32 * grp + 64 * c + lane;
                    xs[c] = col < it.nvalid ? __ldg(&P.sbT[(size_t)kb * P.sb_ld + it.row0 + col]) : 0.0f;
                }
            };
            float nw, nxs[2];
            load_scales(0, nw, nxs);
            for (int kb = 0; kb < KB; ++kb) {
                const float sw = nw;
                const float xs0 = nxs[0], xs1 = nxs[1];
                if (kb + 1 < KB) load_scales(kb + 1, nw, nxs);
                if (!mbar_wait_bounded(&pfull[pb], pb_phase, abort_flag)) { alive = false; break; }
                tc_fence_after();
                const uint32_t t0 = tmem_base + (uint32_t)(pb * C::P_COLS) + ((uint32_t)(q * 32) << 16);
                const int c0a = 32 * grp, c0b = 32 * grp + 64;
                if (c0a < it.nvalid) {
                    my_sc[lane] = sw * xs0;
                    my_sc[32 + lane] = sw * xs1;
                    __syncwarp();
                    float p0[32], p1[32];
                    tmem_ld32x2(t0 + (uint32_t)c0a, t0 + (uint32_t)c0b, p0, p1);
                    const bool two = c0b < it.nvalid;
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const float4 s0 = *reinterpret_cast<const float4*>(my_sc + j);
                        fma2(acc[0][j + 0], acc[0][j + 1], p0[j + 0], p0[j + 1], s0.x, s0.y);
                        fma2(acc[0][j + 2], acc[0][j + 3], p0[j + 2], p0[j + 3], s0.z, s0.w);
                        if (two) {
                            const float4 s1 = *reinterpret_cast<const float4*>(my_sc + 32 + j);
                            fma2(acc[1][j + 0], acc[1][j + 1], p1[j + 0], p1[j + 1], s1.x, s1.y);
                            fma2(acc[1][j + 2], acc[1][j + 3], p1[j + 2], p1[j + 3], s1.z, s1.w);
                        }
                    }
                    __syncwarp();
                }
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
                    for (int c = 0; c < 2; ++c)
#pragma unroll
                        for (int j = 0; j < 32; ++j) xg[fl * C::XUP_STRIDE + c * 32 + j] = acc[c][j];
                }
                named_bar_sync(2 + grp, 128);
                // (2) h = SiLU(gate) * up; per-warp column maxima over its 32 features
                float* cm = cmax + grp * 128;  // [2 chunks][2 gate warps][32 columns]
                if (q < 2) {
                    const int fl = q * 32 + lane;
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
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
                    float lm[2];
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        lm[c] = fmaxf(cm[(c * 2) * 32 + lane], cm[(c * 2 + 1) * 32 + lane]);
                        st_cluster_f32(xmax_peer + (uint32_t)((par * 128 + grp * 64 + c * 32 + lane) * 4), lm[c]);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster_release(xbar_peer + (uint32_t)((par * 2 + grp) * 8));
                    const bool got = mbar_wait_cluster_bounded(&xbar[par * 2 + grp], x_phase[par], abort_flag);
                    float* si = sinv + grp * 64;
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const float amax = got ? fmaxf(lm[c], xmax[par * 128 + grp * 64 + c * 32 + lane]) : 0.0f;
                        const float scale = amax > 0.0f ? amax / 448.0f : 1.0f;
                        si[c * 32 + lane] = 1.0f / scale;
                        const int col = 32 * grp + 64 * c + lane;
                        if (leader && col < it.nvalid) P.hsT[(size_t)it.m * P.hs_ld + it.row0 + col] = scale;
                    }
                    if (lane == 0) warp_ok[wi] = got ? 1 : 0;
                }
                x_phase[par] ^= 1u;
                named_bar_sync(2 + grp, 128);
                if (!warp_ok[4 * grp + 2]) { alive = false; break; }  // the q0 warp is warp 4 + 4 * grp
                // (4) e4m3 codes of h, one byte per (token row, feature)
                if (q < 2) {
                    const int f = it.m * 128 + (int)rank * 64 + q * 32 + lane;
                    const float* si = sinv + grp * 64;
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const int c0 = 32 * grp + 64 * c;
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
                for (int c = 0; c < 2; ++c) {
                    const int c0 = 32 * grp + 64 * c;
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
