// Host-side launch interface between the C ABI (moe_api.cu) and the kernels
// (moe_kernels.cu).  Internal; not installed.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Arguments of the grouped GEMM kernel (moe_gemm.cuh), passed by value.
struct GemmArgs {
    CUtensorMap a0;  // routed A: GATEUP W_gate [E*H, d] (box 64x64) | DOWN W_down [E*d, H] (box 128x64) | LOGITS Wr [E, d]
    CUtensorMap a1;  // GATEUP: W_up [E*H, d] (box 64x64)
    CUtensorMap s0;  // shared A: GATEUP Ws_gate [Hs, d] | DOWN Ws_down [d, Hs]
    CUtensorMap s1;  // GATEUP: Ws_up [Hs, d]
    CUtensorMap b;   // B rows: x_perm [rows, d] | h_perm [rows, ldh] | x [T, d]; box BN x 64
    const int* item_off;   // [n_groups + 1] prefix of work items per group; NULL: one group of n_rows_single rows
    const int* row_off;    // [n_groups + 1] first B row of each group
    int n_groups;
    int n_routed;          // groups >= n_routed are the shared expert
    int n_rows_single;
    int K_routed, K_shared;
    int mt_routed, mt_shared;  // M tiles per group
    int rows_per_expert;       // A rows per routed expert (H for GATEUP, d for DOWN)
    __nv_bfloat16* h;          // GATEUP output
    int ldh;
    float* y;                  // DOWN output (fp32, accumulated)
    const float* row_coef;
    const int* row_tok;
    int ldy;
    float* logits;             // LOGITS output
    int n_logit_cols;
    int k_splits;              // LOGITS: K split over this many items (>= 1)
    float* part;               // LOGITS with k_splits > 1: partial logits [k_splits][T][E]
    // FP8 (e4m3) operands: per-128x128-block weight scales, per-row block scales of B
    const float* sa0;          // routed A scales, tile 0: [E][a_rb_routed][K/128]
    const float* sa1;          // routed A scales, tile 1
    const float* ss0;          // shared expert A scales, tile 0: [a_rb_shared][K/128]
    const float* ss1;
    int a_rb_routed, a_rb_shared;  // 128-row scale blocks per routed / shared weight matrix
    const float* sbT;          // B scales, K-block major: [K/128][sb_ld]
    int sb_ld;
    uint8_t* hq;               // GATEUP FP8 output codes [rows, ldh]
    float* hsT;                // GATEUP FP8 output scales [ldh/128][hs_ld]
    int hs_ld;
    // checking build: rows of the B / h buffers (0: items are not checked) and of y
    int rows_cap;
    int y_rows;
    // grouped items token chunk outer, weight tile inner (else weight tile outer)
    int chunk_major;
};

enum { MODE_GATEUP = 0, MODE_DOWN = 1, MODE_LOGITS = 2 };

struct PermuteArgs {
    const int32_t* idx;
    int T, k, E;
    // expert id e of a pair maps to group e - id_lo; ids outside [id_lo, id_lo + E)
    // are errors (MOE_DEVERR_BAD_EXPERT), or with foreign_ok another rank's experts
    // that this call skips silently
    int id_lo, foreign_ok;
    int32_t* counts;   // [E]
    int32_t* offsets;  // [E + 1]
    int32_t* src;      // [T * k]
    int32_t* inv;      // [T * k]
    // forward mode (row_off != nullptr): per-row token / coefficient tables and
    // the tile schedules of the two grouped GEMMs
    const float* topk_w;
    float routed_scale;
    int n_shared;
    int32_t* row_tok;      // [T * k + n_shared * T]
    float* row_coef;       // [T * k + n_shared * T]
    int32_t* row_off;      // [E + n_shared + 1]
    int32_t* item_off_gu;  // [E + n_shared + 1]
    int32_t* item_off_dn;  // [E + n_shared + 1]
    int bn_gu, bn_dn;
    int mt_gu_routed, mt_gu_shared, mt_dn;
};

size_t gemm_args_size();
int gemm_smem_bytes(int mode, int bn);
// grid: persistent CTAs (one per SM at most).
cudaError_t launch_gemm(int mode, int bn, const GemmArgs* args, int grid, cudaStream_t s);
cudaError_t launch_router_f32(const float* x, const __nv_bfloat16* wr, int T, int d, int E, float* logits,
                              cudaStream_t s);
// parts != nullptr: logits[t, e] = sum over s < n_parts of parts[s][t][e] (fixed order), written first
cudaError_t launch_select(const float* logits, const float* bias, int T, int E, int G, int tg, int k,
                          int32_t* idx, float* w, cudaStream_t s, const float* parts = nullptr, int n_parts = 1);
cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s);
// Forward mode only, many CTAs: needs hist [permute_blocks(T) * E] int32 of scratch.
int permute_blocks(int T);
cudaError_t launch_permute_multi(const PermuteArgs& a, int32_t* hist, cudaStream_t s);
// Expert parallelism over R ranks (contiguous blocks of E / R experts, R <= 32):
// counts[R], offsets[R + 1], and per send row (rank-major, ascending token) its
// origin token, x row (bf16) and the token's k expert ids and weights.
cudaError_t launch_ep_dispatch(const int32_t* idx, const float* w, int T, int k, int E, int R, const void* x,
                               bool x_f32, int d, int32_t* counts, int32_t* offsets, int32_t* send_tok,
                               __nv_bfloat16* send_x, int32_t* send_idx, float* send_w, int n_sm, cudaStream_t s);
// Fixed-capacity packed dispatch: rank q's rows at [q * capacity, q * capacity + counts[q]),
// padding slots token -1 and ids -1; packed rows bf16 x | ids | weights (row_bytes each).
// dst_rank set (peer form): the rows of rank q go to dst_rank[q] at slots dst_row0 + i
// instead of packed (dst_rank: device array of R pointers).
cudaError_t launch_ep_dispatch_packed(const int32_t* idx, const float* w, int T, int k, int E, int R, int capacity,
                                      const void* x, bool x_f32, int d, int32_t* counts, int32_t* send_tok,
                                      uint8_t* packed, int row_bytes, cudaStream_t s,
                                      uint8_t* const* dst_rank = nullptr, int dst_row0 = 0);
// packed rows -> x_rows [n, d] bf16, ids [n, k], w [n, k] (padding rows: ids -1, w 0)
cudaError_t launch_ep_unpack(const uint8_t* packed, int n_rows, int row_bytes, int d, int k, __nv_bfloat16* x_rows,
                             int32_t* ids, float* w, cudaStream_t s);
// acc[send_tok[r], :] += back[r, :] for r < n_rows (fp32 atomics; d % 4 == 0); a token
// of -1 is a padding slot and skipped, any other outside [0, T) sets
// MOE_DEVERR_BAD_ROWS and its row is skipped.  src_rank set (peer form): row r read from
// src_rank[r / capacity] at row src_row0 + r % capacity instead of back.
cudaError_t launch_ep_combine(const float* back, const int32_t* send_tok, int n_rows, int T, int d, float* acc,
                              int n_sm, cudaStream_t s, const float* const* src_rank = nullptr, int capacity = 0,
                              int src_row0 = 0);
// x_perm[r, :] = x[row_tok[r], :] (fp32 input rounded to bf16) for r < row_off[n_groups]
// (checking build: row_tok entries against n_tok, the row count against max_rows)
cudaError_t launch_gather(const void* x, bool x_f32, int d, int n_tok, const int32_t* row_tok,
                          const int32_t* n_rows_dev, int max_rows, __nv_bfloat16* x_perm, int n_sm, cudaStream_t s);
// token-major copy into x_perm: token t's row to rows inv[t*k + j] (>= 0) and, when
// shared_base_dev is set, to row *shared_base_dev + t
cudaError_t launch_scatter_rows(const void* x, bool x_f32, int d, int T, int k, const int32_t* inv,
                                const int32_t* shared_base_dev, int rows_cap, __nv_bfloat16* x_perm, int n_sm,
                                cudaStream_t s);
// q[t, :], sx[t, b]: per-token, per-128-channel e4m3 quantisation of bf16 x
cudaError_t launch_quant_act(const __nv_bfloat16* x, int T, int d, uint8_t* q, float* sx, cudaStream_t s);
// S6 + copy into expert order, token-major (xq_in set: copy codes and scales made earlier)
cudaError_t launch_quant_scatter_fp8(const __nv_bfloat16* x, const uint8_t* xq_in, const float* sx_in, int d, int T,
                                     int k, const int32_t* inv, const int32_t* shared_base_dev, int rows_ld,
                                     uint8_t* xpq, float* sxT, int n_sm, cudaStream_t s);
// checking build, tests only: *p = v on the stream
cudaError_t launch_debug_poke(int32_t* p, int v, cudaStream_t s);
int gemm_fp8_smem_bytes(int mode, int bn);
// CTA-pair (2-SM MMA) bf16 grouped GEMM, 256 token rows per item; grid even.
cudaError_t launch_gemm2(int mode, const GemmArgs* args, int grid, cudaStream_t s);
// CTA-pair FP8 grouped GEMM, 128 token rows per item; grid even.
cudaError_t launch_gemm2_fp8(int mode, const GemmArgs* args, int grid, cudaStream_t s);
cudaError_t launch_gemm_fp8(int mode, int bn, const GemmArgs* args, int grid, cudaStream_t s);
// number of kernels launched so far (every launcher counts its launches)
unsigned long long launch_count();
// bias[e] -/+= gamma by counts[e] against the mean count
cudaError_t launch_update_bias(const int32_t* counts, int E, float* bias, float gamma, cudaStream_t s);
// y[i] = bf16(acc[i] (+ y[i]))
cudaError_t launch_finalize_bf16(const float* acc, const __nv_bfloat16* residual, __nv_bfloat16* y, size_t n,
                                 cudaStream_t s);
// a bounded mbarrier wait that runs out after limit_ns (sets MOE_DEVERR_TIMEOUT)
cudaError_t launch_wait_selftest(unsigned long long limit_ns, cudaStream_t s);
// dense FFN tables: one group of T rows, identity rows, coefficient 1
cudaError_t launch_dense_schedule(int T, int bn, int mt_gu, int mt_dn, int32_t* row_off, int32_t* item_gu,
                                  int32_t* item_dn, int32_t* row_tok, float* row_coef, cudaStream_t s);
// pre-norm: out = bf16(bf16(h * r) * g) per token row (+ e4m3 codes / scales when q, sx are set)
constexpr int NORM_THREADS = 128;
constexpr int NORM_MAX_VEC = 8;  // 8-feature vectors per thread: d <= 8 * 8 * 128
cudaError_t launch_rmsnorm(const __nv_bfloat16* h, const __nv_bfloat16* g, int T, int d, float eps,
                           __nv_bfloat16* out, uint8_t* q, float* sx, cudaStream_t s);
cudaError_t read_clear_dev_error(unsigned int* flags, cudaStream_t s);

}  // namespace moe
