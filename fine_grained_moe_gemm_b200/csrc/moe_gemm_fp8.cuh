// FP8 grouped GEMM for the MoE expert projections ("Teardown: DeepSeek-V3",
// section 10: E4M3 operands, activations scaled per 1x128 tile, weights per
// 128x128 block, partial sums promoted to fp32 every 128 elements).
//
// Same item structure as the bf16 kernel (moe_gemm.cuh): 256 weight rows (two
// 128-row tiles) of one expert against up to BN token rows, persistent CTAs,
// TMA producer warp, single-thread MMA issuer, eight epilogue warps.  What
// changes is the accumulation:
//   D[f, r] = sum_kb  sw[f, kb] * sx[r, kb] * P_kb[f, r],
//   P_kb[f, r] = sum_{k in block kb} qw[f, k] * qx[r, k]     (e4m3 x e4m3)
// Each 128-element K block is one stage: four tcgen05.mma kind::f8f6f4
// (K = 32 each) write a fresh partial P_kb into one of two TMEM buffers; the
// epilogue warps read it, multiply by the two scales and add it into fp32
// accumulators held in registers (the promotion), then free the buffer.
// Epilogues after the last block:
//   GATEUP  h = SiLU(gate) * up for 128 features, quantised to e4m3 per row
//           and 128-feature block (scale = amax / 448), codes [rows, ldh] and
//           scales transposed [ldh/128][rows] (the down GEMM's B operand);
//   DOWN    y[row_tok[r], f] += row_coef[r] * D[f, r] (fp32 red.add).
// BN <= 128: up to four partial buffers of 2 x BN TMEM columns, so that the
// MMAs run ahead of the promotion; each epilogue warp waits for a partial by
// itself and the scales of the next K block are loaded while it waits.  Each
// epilogue thread holds 2 x BN/2 fp32 accumulators.
#pragma once

#include "moe_gemm.cuh"

namespace moe {

template <int MODE, int BN>
struct Fp8Cfg {
    static constexpr int A_TILE = 128 * 128;   // 128 rows x 128 e4m3
    static constexpr int A_BYTES = 2 * A_TILE;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int SMEM_LIMIT = 227 * 1024;
    static constexpr int MISC_BYTES = 4096;    // barriers, flags, per-warp scale rows, amax exchange
    static constexpr int STAGES_FIT = (SMEM_LIMIT - 1024 - MISC_BYTES) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
    static constexpr int ACC_COLS = 2 * BN;    // one partial buffer: [tile 0: BN][tile 1: BN]
    static constexpr int NUM_P = 512 / ACC_COLS >= 4 ? 4 : 512 / ACC_COLS;  // partial buffers in TMEM
    static constexpr int TMEM_NEED = NUM_P * ACC_COLS;
    static constexpr int TMEM_COLS = TMEM_NEED <= 128 ? 128 : TMEM_NEED <= 256 ? 256 : 512;
    static constexpr int CH = BN >= 64 ? BN / 64 : 1;  // column chunks per epilogue thread
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + MISC_BYTES;
    static_assert(BN == 32 || BN == 64 || BN == 128, "BN");
    static_assert(STAGES >= 2, "stages");
};

__device__ __forceinline__ uint32_t cvt_e4m3x2(float hi, float lo) {
    // two fp32 -> two e4m3 (round to nearest even, saturating to +-448):
    // `hi` in bits 15..8, `lo` in bits 7..0
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

template <int MODE, int BN>
__global__ void __launch_bounds__(GEMM_THREADS, 1) moe_gemm_fp8_kernel(const __grid_constant__ GemmArgs P) {
    using C = Fp8Cfg<MODE, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    uint8_t* misc = smem + C::STAGES * C::STAGE_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(misc);
    uint64_t* full = bars;
    uint64_t* empty = bars + C::STAGES;
    uint64_t* pfull = bars + 2 * C::STAGES;   // partial buffer written
    uint64_t* pempty = pfull + C::NUM_P;      // partial buffer consumed
    uint64_t* drain = pempty + C::NUM_P;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* warp_ok = reinterpret_cast<volatile int*>(tmem_slot + 2);  // [8] epilogue warps
    float* sc_rows = reinterpret_cast<float*>(misc + 512);   // [8 warps][2 tiles][32]
    float* amax_x = reinterpret_cast<float*>(misc + 2560);   // [2 groups][4 quarters][32]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < C::NUM_P; ++a) {
            mbar_init(&pfull[a], 1);
            mbar_init(&pempty[a], GEMM_EPI_THREADS / 32);
        }
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
    if (warp == 1) tmem_alloc<C::TMEM_COLS>(tmem_slot);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = __ldg(&P.item_off[P.n_groups]);

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            const uint64_t pol_w = l2_policy_evict_first();
            const uint64_t pol_x = l2_policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            for (int i = blockIdx.x; i < total; i += gridDim.x) {
                const Item it = decode_item<BN>(P, i);
                const int KB = it.K / 128;
                const int nbox = (it.nvalid + B_BOX_ROWS - 1) / B_BOX_ROWS;
                const uint32_t bytes = C::A_BYTES + nbox * B_BOX_ROWS * 128;
                const CUtensorMap* m0;
                const CUtensorMap* m1;
                int r0, r1;
                const int base = it.shared ? 0 : it.g * P.rows_per_expert;
                if (MODE == GEMM_GATEUP) {
                    m0 = it.shared ? &P.s0 : &P.a0;
                    m1 = it.shared ? &P.s1 : &P.a1;
                    r0 = r1 = base + it.m * 128;
                } else {
                    m0 = m1 = it.shared ? &P.s0 : &P.a0;
                    r0 = base + it.m * 256;
                    r1 = r0 + 128;
                }
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
                    uint8_t* sa = ring + stage * C::STAGE_BYTES;
                    uint8_t* sb = sa + C::A_BYTES;
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    tma_load_2d(sa, m0, kb * 128, r0, &full[stage], pol_w);
                    tma_load_2d(sa + C::A_TILE, m1, kb * 128, r1, &full[stage], pol_w);
                    for (int bx = 0; bx < nbox; ++bx)
                        tma_load_2d(sb + bx * B_BOX_ROWS * 128, &P.b, kb * 128, it.row0 + bx * B_BOX_ROWS,
                                    &full[stage], pol_x);
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer: one partial per K block
            int stage = 0;
            uint32_t phase = 0;
            int pb = 0;
            uint32_t pb_phase = 0;
            bool issued = false, ok = true;
            for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
                const Item it = decode_item<BN>(P, i);
                const int KB = it.K / 128;
                uint32_t n_mma = (uint32_t)((it.nvalid + 15) & ~15);
                n_mma = n_mma < 16u ? 16u : n_mma;
                const uint32_t idesc = idesc_e4m3_f32(128, n_mma);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(&pempty[pb], pb_phase ^ 1u, abort_flag)) { ok = false; break; }
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d0 = tmem_base + (uint32_t)(pb * C::ACC_COLS);
                    const uint32_t d1 = d0 + BN;
                    const uint32_t a_addr = smem_u32(ring + stage * C::STAGE_BYTES);
                    const uint64_t adesc0 = smem_desc_sw128(a_addr);
                    const uint64_t adesc1 = smem_desc_sw128(a_addr + C::A_TILE);
                    const uint64_t bdesc = smem_desc_sw128(a_addr + C::A_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t accum = k != 0 ? 1u : 0u;
                        mma_e4m3(d0, adesc0 + 2ull * k, bdesc + 2ull * k, idesc, accum);
                        mma_e4m3(d1, adesc1 + 2ull * k, bdesc + 2ull * k, idesc, accum);
                    }
                    mma_commit(&empty[stage]);
                    mma_commit(&pfull[pb]);
                    issued = true;
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
                    if (++pb == C::NUM_P) { pb = 0; pb_phase ^= 1u; }
                }
            }
            if (*abort_flag && issued) {
                mma_commit(drain);
                volatile int dummy = 0;
                mbar_wait_bounded(drain, 0, &dummy, 100000000ull);
            }
        }
    } else {
        // ---------------------------------------------------- epilogue: promotion + final
        const int q = warp & 3;
        const int grp = (warp - 2) >> 2;
        const int wi = warp - 2;
        float* my_sc = sc_rows + wi * 64;   // [2 tiles][32 columns]
        int pb = 0;
        uint32_t pb_phase = 0;
        bool alive = true;
        for (int i = blockIdx.x; i < total && alive; i += gridDim.x) {
            const Item it = decode_item<BN>(P, i);
            const int KB = it.K / 128;
            const int a_rb = it.shared ? P.a_rb_shared : P.a_rb_routed;
            const float* sa_t0 = it.shared ? P.ss0 : P.sa0;
            const float* sa_t1 = it.shared ? P.ss1 : P.sa1;
            int rb0, rb1;
            if (MODE == GEMM_GATEUP) rb0 = rb1 = it.m;
            else { rb0 = 2 * it.m; rb1 = 2 * it.m + 1; }
            const size_t sbase = it.shared ? 0 : (size_t)it.g * a_rb;
            float acc0[C::CH][32], acc1[C::CH][32];
#pragma unroll
            for (int c = 0; c < C::CH; ++c)
#pragma unroll
                for (int j = 0; j < 32; ++j) acc0[c][j] = acc1[c][j] = 0.0f;

            // scales of K block kb: weight blocks of the two tiles, B row of this lane's column
            auto load_scales = [&](int kb, float& w0, float& w1, float (&xs)[C::CH]) {
                w0 = rb0 < a_rb ? __ldg(&sa_t0[(sbase + rb0) * KB + kb]) : 0.0f;
                w1 = rb1 < a_rb ? __ldg(&sa_t1[(sbase + rb1) * KB + kb]) : 0.0f;
#pragma unroll
                for (int c = 0; c < C::CH; ++c) {
                    const int col = 32 * grp + 64 * c + lane;
                    xs[c] = col < it.nvalid ? __ldg(&P.sbT[(size_t)kb * P.sb_ld + it.row0 + col]) : 0.0f;
                }
            };
            float nw0, nw1, nxs[C::CH];
            load_scales(0, nw0, nw1, nxs);
            for (int kb = 0; kb < KB; ++kb) {
                const float sw0 = nw0, sw1 = nw1;
                float xs[C::CH];
#pragma unroll
                for (int c = 0; c < C::CH; ++c) xs[c] = nxs[c];
                if (kb + 1 < KB) load_scales(kb + 1, nw0, nw1, nxs);
                if (!mbar_wait_bounded(&pfull[pb], pb_phase, abort_flag)) { alive = false; break; }
                tc_fence_after();
                const uint32_t t0 = tmem_base + (uint32_t)(pb * C::ACC_COLS) + ((uint32_t)(q * 32) << 16);
#pragma unroll
                for (int c = 0; c < C::CH; ++c) {
                    const int c0 = 32 * grp + 64 * c;
                    if (c0 < it.nvalid) {
                        my_sc[lane] = sw0 * xs[c];
                        my_sc[32 + lane] = sw1 * xs[c];
                        __syncwarp();
                        float p0[32], p1[32];
                        tmem_ld32x2(t0 + (uint32_t)c0, t0 + BN + (uint32_t)c0, p0, p1);
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            const float4 s0 = *reinterpret_cast<const float4*>(my_sc + j);
                            const float4 s1 = *reinterpret_cast<const float4*>(my_sc + 32 + j);
                            acc0[c][j + 0] = fmaf(p0[j + 0], s0.x, acc0[c][j + 0]);
                            acc0[c][j + 1] = fmaf(p0[j + 1], s0.y, acc0[c][j + 1]);
                            acc0[c][j + 2] = fmaf(p0[j + 2], s0.z, acc0[c][j + 2]);
                            acc0[c][j + 3] = fmaf(p0[j + 3], s0.w, acc0[c][j + 3]);
                            acc1[c][j + 0] = fmaf(p1[j + 0], s1.x, acc1[c][j + 0]);
                            acc1[c][j + 1] = fmaf(p1[j + 1], s1.y, acc1[c][j + 1]);
                            acc1[c][j + 2] = fmaf(p1[j + 2], s1.z, acc1[c][j + 2]);
                            acc1[c][j + 3] = fmaf(p1[j + 3], s1.w, acc1[c][j + 3]);
                        }
                        __syncwarp();
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&pempty[pb]);
                if (++pb == C::NUM_P) { pb = 0; pb_phase ^= 1u; }
            }

            if (MODE == GEMM_GATEUP) {
                // the final epilogue synchronises the group's four warps: agree
                // first that none of them gave up on a wait
                if (lane == 0) warp_ok[wi] = alive ? 1 : 0;
                named_bar_sync(2 + grp, 128);
                alive = warp_ok[4 * grp] && warp_ok[4 * grp + 1] && warp_ok[4 * grp + 2] && warp_ok[4 * grp + 3];
            }
            if (!alive) break;

            if (MODE == GEMM_GATEUP) {
                const int f = it.m * 128 + q * 32 + lane;
                float* ax = amax_x + grp * 128;  // [4 quarters][32 columns]
#pragma unroll
                for (int c = 0; c < C::CH; ++c) {
                    const int c0 = 32 * grp + 64 * c;
                    const bool live = c0 < it.nvalid;  // uniform over the group's four warps
                    // h = SiLU(gate) * up in place of the gate sums; the up sums,
                    // no longer needed, hold |h| for the reduction
                    float* h = acc0[c];
                    float* m = acc1[c];
                    if (live) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            h[j] = silu_mul(acc0[c][j], acc1[c][j]);
                            m[j] = fabsf(h[j]);
                        }
                        // max over the 32 lanes of each column: lane l ends with column l
#pragma unroll
                        for (int off = 16; off >= 1; off >>= 1) {
                            const bool upper = (lane & off) != 0;
#pragma unroll
                            for (int j = 0; j < off; ++j) {
                                const float send = upper ? m[j] : m[j + off];
                                const float keep = upper ? m[j + off] : m[j];
                                m[j] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, off));
                            }
                        }
                        ax[q * 32 + lane] = m[0];
                    }
                    named_bar_sync(2 + grp, 128);
                    if (live) {
                        const float amax = fmaxf(fmaxf(ax[lane], ax[32 + lane]), fmaxf(ax[64 + lane], ax[96 + lane]));
                        const float scale = amax > 0.0f ? amax / 448.0f : 1.0f;
                        const int col = c0 + lane;
                        if (q == 0 && col < it.nvalid) P.hsT[(size_t)it.m * P.hs_ld + it.row0 + col] = scale;
                        m[0] = 1.0f / scale;   // this lane's column
                    }
                    named_bar_sync(2 + grp, 128);   // ax is reused by the next chunk
                    if (live) {
                        uint8_t* dst = P.hq + (size_t)(it.row0 + c0) * P.ldh + f;
#pragma unroll
                        for (int j = 0; j < 32; j += 2) {
                            const float i0 = __shfl_sync(0xffffffffu, m[0], j);
                            const float i1 = __shfl_sync(0xffffffffu, m[0], j + 1);
                            const uint32_t pk = cvt_e4m3x2(h[j + 1] * i1, h[j] * i0);
                            if (c0 + j < it.nvalid) dst[(size_t)j * P.ldh] = (uint8_t)(pk & 0xff);
                            if (c0 + j + 1 < it.nvalid) dst[(size_t)(j + 1) * P.ldh] = (uint8_t)(pk >> 8);
                        }
                    }
                }
            } else {
                const int f0 = it.m * 256 + q * 32 + lane;
                const int f1 = f0 + 128;
                const bool ok0 = f0 < P.ldy, ok1 = f1 < P.ldy;
#pragma unroll
                for (int c = 0; c < C::CH; ++c) {
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
                                if (ok0) atomicAdd(yr + f0, acc0[c][j] * cf);
                                if (ok1) atomicAdd(yr + f1, acc1[c][j] * cf);
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
        tmem_dealloc<C::TMEM_COLS>(tmem_base);
    }
}

}  // namespace moe
