// Grouped GEMM on CTA pairs (tcgen05.mma.cta_group::2) for the wide-token
// shapes of the MoE expert projections (prefill and beyond: an expert holds
// 100+ token rows).
//
// Same formulation as moe_gemm.cuh (weights as M, tokens as N, persistent
// tile walk over the device-built schedule), but a cluster of two CTAs on two
// SMs works each item together:
//   - each CTA loads its own 128-row slices of two weight tiles (A) and HALF of
//     the item's token rows (B); one 2-SM MMA (M = 256, N <= 256) reads A from
//     both CTAs and B from both halves, and writes each CTA's 128 rows x N
//     columns into that CTA's TMEM;
//   - so every SM streams its weights once and only half of the token tile:
//     the token rows, which every weight block of an expert re-reads, cost
//     half the L2 -> SM traffic of the single-CTA kernel.
// Per item the pair covers GATEUP: 256 features (gate + up accumulators, one
// CTA per 128 features), DOWN: 512 output features (two 256-row MMAs).
// Roles per CTA: warp 0 TMA producer, warp 1 TMEM allocator (both CTAs) and
// MMA issuer (leader CTA only), warps 2-17 epilogue on the CTA's own TMEM.
// Synchronisation across the pair: the peer's TMA loads complete on the
// leader's stage barrier (.cta_group::2 addressing, no multicast); the MMA's
// commits arrive on the barrier of both CTAs (tcgen05.commit multicast); the
// peer's epilogue releases the accumulators on the leader's barrier (remote
// mbarrier.arrive).  All waits are bounded as in the single-CTA kernel.
#pragma once

#include "moe_gemm.cuh"

namespace moe {

constexpr int PAIR_BN = 256;       // token rows per item (whole pair)
// Token rows per B TMA box (each CTA loads N/2 rows, rounded up to whole boxes;
// rows past the item's own are loaded and ignored).  Wide boxes: one TMA
// instruction costs a few hundred cycles of the issuing thread whatever its
// size, so a stage is loaded in as few instructions as its tiles allow.
constexpr int PAIR_BOX_ROWS = 64;
// Sixteen epilogue warps (four per TMEM lane quarter): the accumulators are
// single-buffered, so the MMA of the next item waits for the epilogue to drain
// them, and four warps per SM sub-partition drain them about twice as fast as
// two.  576 threads leave 112 registers a thread.
constexpr int PAIR_EPI_WARPS = 16;
constexpr int PAIR_EPI_THREADS = PAIR_EPI_WARPS * 32;
constexpr int PAIR_THREADS = 64 + PAIR_EPI_THREADS;

struct Gemm2Cfg {
    static constexpr int A_TILE = 128 * 128;
    static constexpr int A_BYTES = 2 * A_TILE;              // this CTA's slices of the two tiles
    static constexpr int B_BYTES = PAIR_BN / 2 * 128;       // this CTA's half of the token rows
    static_assert(B_BYTES % (PAIR_BOX_ROWS * 128) == 0, "B tile holds whole boxes");
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int MISC_BYTES = 1024;
    static constexpr int STAGES = (227 * 1024 - 1024 - MISC_BYTES) / STAGE_BYTES > 6
                                      ? 6 : (227 * 1024 - 1024 - MISC_BYTES) / STAGE_BYTES;
    static constexpr int ACC_COLS = 2 * PAIR_BN;            // [tile 0: 256][tile 1: 256]
    static constexpr int TMEM_COLS = 512;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + MISC_BYTES;
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// shared::cluster address of the same shared-memory location in CTA `rank`
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// TMA tile load into this CTA's shared memory whose completion is counted on
// an mbarrier of either CTA of the pair (shared::cluster address).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, int x, int y,
                                                 uint32_t mbar_cluster, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(mbar_cluster), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void mma2_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive, when every 2-SM MMA issued so far has completed, on the mbarrier at
// this shared-memory offset in each CTA of `cta_mask`.
__device__ __forceinline__ void mma2_commit_pair(uint64_t* bar, uint16_t cta_mask) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 ::"r"(smem_u32(bar)), "h"(cta_mask)
                 : "memory");
}

__device__ __forceinline__ void mma2_commit_local(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Arrive on an mbarrier of either CTA of the pair (shared::cluster address).
// Used to hand TMEM back to the MMA issuer after tcgen05.fence::before_thread_sync;
// no data other than TMEM is published, so no cluster-scope release is needed.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}

// Arrive with release at cluster scope: the peer's acquire-wait then sees this
// thread's earlier stores to its shared memory.
__device__ __forceinline__ void mbar_arrive_cluster_release(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem) {  // one warp in each CTA of the pair
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "n"(Gemm2Cfg::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "n"(Gemm2Cfg::TMEM_COLS)
                 : "memory");
}

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PAIR_THREADS, 1)
    moe_gemm2_kernel(const __grid_constant__ GemmArgs P) {
    using C = Gemm2Cfg;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t* full = bars;                 // leader: stage loaded (both CTAs' bytes)
    uint64_t* empty = bars + C::STAGES;    // both: stage consumed by the MMA
    uint64_t* tfull = bars + 2 * C::STAGES;  // both: accumulators written
    uint64_t* tempty = tfull + 1;          // leader: accumulators read by both epilogues
    uint64_t* drain = tempty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* epi_ok = reinterpret_cast<volatile int*>(tmem_slot + 2);  // [2]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tfull, 1);
        mbar_init(tempty, 2 * PAIR_EPI_WARPS);
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
    cluster_sync_all();  // both CTAs' barriers initialised and TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int total = __ldg(&P.item_off[P.n_groups]);
    const int cluster_id = blockIdx.x >> 1;
    const int n_clusters = gridDim.x >> 1;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer (both CTAs)
            // chunk-major items (see decode_item): a chunk's token rows are read by its items
            // at about the same time (normal priority), a multi-chunk expert's weight tiles
            // again by every chunk (evict-last); single-chunk tiles stream (evict-first)
            const uint64_t pol_w = l2_policy_evict_first();
            const uint64_t pol_keep = l2_policy_evict_last();
            const uint64_t pol_x = l2_policy_evict_normal();
            const uint32_t full0 = mapa_shared(smem_u32(&full[0]), 0);
            int stage = 0;
            uint32_t phase = 0;
            for (int i = cluster_id; i < total; i += n_clusters) {
                const Item it = decode_item<PAIR_BN>(P, i);
                // weights read by several items stay in L2 for the others; the rest stream
                const uint64_t pw = it.nch > 1 ? pol_keep : pol_w;
                const int KB = it.K / 64;
                int n_mma = (it.nvalid + 31) & ~31;
                const int nh = n_mma / 2;                          // this CTA's token rows
                const int nbox = (nh + PAIR_BOX_ROWS - 1) / PAIR_BOX_ROWS;
                const uint32_t bytes = 2u * (uint32_t)(C::A_BYTES + nbox * PAIR_BOX_ROWS * 128);
                const CUtensorMap* m0;
                const CUtensorMap* m1;
                int r0, r1;
                const int base = it.shared ? 0 : it.g * P.rows_per_expert;
                if (MODE == GEMM_GATEUP) {  // gate and up rows of this CTA's 128 features
                    m0 = it.shared ? &P.s0 : &P.a0;
                    m1 = it.shared ? &P.s1 : &P.a1;
                    r0 = r1 = base + it.m * 256 + (int)rank * 128;
                } else {                    // rows m*512 + rank*128 and + 256
                    m0 = m1 = it.shared ? &P.s0 : &P.a0;
                    r0 = base + it.m * 512 + (int)rank * 128;
                    r1 = r0 + 256;
                }
                const int brow = it.row0 + (int)rank * nh;
                bool ok = true;
                for (int kb = item_kb0(it, KB); kb < item_kb1(it, KB); ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
                    uint8_t* sa = ring + stage * C::STAGE_BYTES;
                    uint8_t* sb = sa + C::A_BYTES;
                    const uint32_t fb = full0 + (uint32_t)(stage * 8);
                    if (leader) mbar_arrive_expect_tx(&full[stage], bytes);
                    tma_load_2d_pair(sa, m0, kb * 64, r0, fb, pw);
                    tma_load_2d_pair(sa + C::A_TILE, m1, kb * 64, r1, fb, pw);
                    for (int bx = 0; bx < nbox; ++bx)
                        tma_load_2d_pair(sb + bx * PAIR_BOX_ROWS * 128, &P.b, kb * 64, brow + bx * PAIR_BOX_ROWS, fb,
                                         pol_x);
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------------------------ 2-SM MMA issuer (leader CTA)
            int stage = 0;
            uint32_t phase = 0;
            uint32_t acc_phase = 0;
            bool issued = false;
            for (int i = cluster_id; i < total; i += n_clusters) {
                const Item it = decode_item<PAIR_BN>(P, i);
                const int KB = it.K / 64;
                const uint32_t n_mma = (uint32_t)((it.nvalid + 31) & ~31);
                const uint32_t idesc = idesc_bf16_f32(256, n_mma);
                if (!mbar_wait_bounded(tempty, acc_phase ^ 1u, abort_flag)) break;
                tc_fence_after();
                const uint32_t d0 = tmem_base;
                const uint32_t d1 = tmem_base + PAIR_BN;
                bool ok = true;
                const int kb0 = item_kb0(it, KB), kb1 = item_kb1(it, KB);
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
                        mma2_bf16(d0, adesc0 + 2ull * k, bdesc + 2ull * k, idesc, accum);
                        mma2_bf16(d1, adesc1 + 2ull * k, bdesc + 2ull * k, idesc, accum);
                    }
                    mma2_commit_pair(&empty[stage], 0x3);
                    issued = true;
                    if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                mma2_commit_pair(tfull, 0x3);
                acc_phase ^= 1u;
            }
            if (*abort_flag && issued) {
                mma2_commit_local(drain);
                volatile int dummy = 0;
                mbar_wait_bounded(drain, 0, &dummy, 100000000ull);
            }
        }
    } else {
        // ---------------------------------------------------- epilogue (both CTAs, own TMEM)
        const int q = warp & 3;
        const int grp = (warp - 2) >> 2;
        const int et = threadIdx.x - 64;
        const uint32_t tempty_leader = mapa_shared(smem_u32(tempty), 0);
        uint32_t acc_phase = 0;
        int n_done = 0;
        for (int i = cluster_id; i < total; i += n_clusters, ++n_done) {
            const Item it = decode_item<PAIR_BN>(P, i);
            if (et == 0) epi_ok[n_done & 1] = mbar_wait_bounded(tfull, acc_phase, abort_flag) ? 1 : 0;
            named_bar_sync(1, PAIR_EPI_THREADS);
            if (!epi_ok[n_done & 1]) break;
            tc_fence_after();
            const uint32_t t0 = tmem_base + ((uint32_t)(q * 32) << 16);
            const uint32_t t1 = t0 + PAIR_BN;
            for (int c0 = 32 * grp; c0 < it.nvalid; c0 += 32 * (PAIR_EPI_WARPS / 4)) {
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
                    const int f = it.m * 256 + (int)rank * 128 + q * 32 + lane;
                    __nv_bfloat16* dst = P.h + (size_t)(it.row0 + c0) * P.ldh + f;
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj)
                        if (c0 + jj < it.nvalid) dst[(size_t)jj * P.ldh] = __float2bfloat16_rn(silu_mul(v0[jj], v1[jj]));
                } else {
                    const int f0 = it.m * 512 + (int)rank * 128 + q * 32 + lane;
                    const int f1 = f0 + 256;
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
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty_leader);
            acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // no CTA leaves while its peer may still signal it
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base);
    }
}

}  // namespace moe
