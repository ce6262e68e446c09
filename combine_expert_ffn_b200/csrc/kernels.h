// kernels.h -- internal launch functions of libmoe (not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace moe {

// Counts one kernel launch (process-wide, for moe_launch_count()).
void count_launch();

// tmap.cu: bf16 tensor maps, box = box_cols x box_rows (x 1), swizzle of
// swizzle_bytes (64 or 128 = the box's row length in bytes; 0 = none)
bool tensor_maps_available();
bool tensor_map_2d_bf16(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols,
                        uint32_t box_cols, uint32_t box_rows, uint32_t swizzle_bytes = 128);
bool tensor_map_3d_bf16(CUtensorMap *m, const void *base, uint64_t n_mat, uint64_t rows,
                        uint64_t cols, uint32_t box_cols, uint32_t box_rows,
                        uint32_t swizzle_bytes = 128);
// byte tiles (FP8 payload), row-major box without swizzle
bool tensor_map_2d_u8(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols,
                      uint32_t box_cols, uint32_t box_rows);

// route.cu
cudaError_t launch_route_select(const float *scores, const float *bias, int T, int E, int G,
                                int K, int M, int32_t *topk_idx, float *topk_w, cudaStream_t st);

// dispatch.cu
struct DispatchWs {
    int32_t *hist_t;       // [E, nblk] copies of expert e in token block b
    int32_t *base_t;       // [E, nblk] exclusive prefix of hist_t along b
    int32_t *send_part;    // [nblk, G*G]
    int32_t *sendtok_part; // [nblk, G*G]
};
constexpr int DISPATCH_BLOCK = 256;  // tokens per dispatch block
inline int dispatch_nblk(int T) { return (T + DISPATCH_BLOCK - 1) / DISPATCH_BLOCK; }
cudaError_t launch_dispatch(const void *x, const int32_t *topk_idx, int T, int d, int E, int G,
                            int K, int32_t *counts, int32_t *offsets, int32_t *send,
                            int32_t *send_tok, int32_t *perm_token, int32_t *inv_perm,
                            void *x_perm, const DispatchWs &ws, int32_t *status, cudaStream_t st);

// dispatch.cu: the gather-permute alone, x_perm[inv_perm[t][j]] = x[t]
// (rows of up to 14 KB through the copy engine with bounded waits recording into
// status, which may be null; wider rows by 16-byte thread copies)
cudaError_t launch_permute(const void *x, const int32_t *inv_perm, int T, int d, int K,
                           void *x_perm, cudaStream_t st, int32_t *status = nullptr,
                           int64_t timeout_ns = 2000000000LL);
// dispatch.cu, FP8 payload: x_perm_q[row] = E4M3(x[token] / s) and x_scale[row][b] = s
// (one scale per 128 channels, s = amax / 448); d % 128 == 0
cudaError_t launch_gather_fp8(const void *x, const int32_t *inv_perm, int T, int d, int K,
                              uint8_t *x_perm_q, float *x_scale, cudaStream_t st);

// ep.cu: expert parallelism over `world` ranks (E / world experts each)
cudaError_t launch_ep_plan(const int32_t *counts_all, int world, int E, int me, int32_t *base,
                           int32_t *local_offsets, cudaStream_t st);
cudaError_t launch_ep_dispatch(const void *x, const int32_t *topk_idx, const int32_t *offsets,
                               const int32_t *inv_perm, const int32_t *base, void *const *recv_x,
                               int64_t recv_rows, int T, int d, int E, int K, int world,
                               int32_t *status, cudaStream_t st);
cudaError_t launch_ep_dispatch_fp8(const void *x, const int32_t *topk_idx,
                                   const int32_t *offsets, const int32_t *inv_perm,
                                   const int32_t *base, void *const *recv_q,
                                   void *const *recv_scale, int64_t recv_rows, int T, int d, int E,
                                   int K, int world, int32_t *status, cudaStream_t st);
cudaError_t launch_ep_token_plan(const int32_t *topk_idx, int T, int E, int K, int world,
                                  int32_t *tok_slot, int32_t *tok_counts, cudaStream_t st);
cudaError_t launch_ep_token_base(const int32_t *tok_counts_all, int world, int me,
                                 int32_t *tok_base, cudaStream_t st);
cudaError_t launch_ep_dispatch_dedup(const void *x, const int32_t *topk_idx, const int32_t *offsets,
                                     const int32_t *inv_perm, const int32_t *base,
                                     const int32_t *tok_slot, const int32_t *tok_base,
                                     void *const *recv_tok, int32_t *const *recv_idx,
                                     int64_t tok_rows, int64_t recv_rows, int T, int d, int E, int K,
                                     int world, int32_t *status, cudaStream_t st,
                                     const float *topk_w = nullptr, int32_t *const *list = nullptr,
                                     float *const *lw = nullptr, int32_t *const *lcnt = nullptr);
cudaError_t launch_ep_fanout(const void *recv_tok, const int32_t *recv_idx,
                             const int32_t *local_offsets, int El, int64_t tok_rows,
                             int64_t recv_rows, int d, void *recv_x, int32_t *status,
                             cudaStream_t st);
cudaError_t launch_ep_dispatch_dedup_fp8(const void *x, const int32_t *topk_idx,
                                         const int32_t *offsets, const int32_t *inv_perm,
                                         const int32_t *base, const int32_t *tok_slot,
                                         const int32_t *tok_base, void *const *recv_tq,
                                         void *const *recv_ts, int32_t *const *recv_idx,
                                         int64_t tok_rows, int64_t recv_rows, int T, int d, int E,
                                         int K, int world, int32_t *status, cudaStream_t st);
cudaError_t launch_ep_fanout_fp8(const void *recv_tq, const float *recv_ts,
                                 const int32_t *recv_idx, const int32_t *local_offsets, int El,
                                 int64_t tok_rows, int64_t recv_rows, int d, void *recv_q,
                                 float *recv_scale, int32_t *status, cudaStream_t st);
cudaError_t launch_ep_combine_plan(const int32_t *topk_idx, const float *topk_w,
                                   const int32_t *offsets, const int32_t *inv_perm,
                                   const int32_t *base, const int32_t *tok_slot,
                                   const int32_t *tok_base, int32_t *const *list,
                                   float *const *lw, int32_t *const *lcnt, int64_t tok_rows,
                                   int64_t recv_rows, int T, int E, int K, int world,
                                   int32_t *status, cudaStream_t st);
cudaError_t launch_ep_precombine(const void *recv_y, const int32_t *list, const float *lw,
                                 const int32_t *lcnt, const int32_t *tok_base, int world,
                                 int64_t tok_rows, int64_t recv_rows, int d, int K, void *partial,
                                 int32_t *status, cudaStream_t st);
cudaError_t launch_ep_combine_dedup(const int32_t *topk_idx, const int32_t *tok_slot,
                                    const int32_t *tok_base, const void *const *partial,
                                    const void *y_shared, int64_t tok_rows, int T, int d, int E,
                                    int K, int world, void *out, int32_t *status,
                                    cudaStream_t st);
cudaError_t launch_ep_combine(const int32_t *topk_idx, const float *topk_w, const int32_t *offsets,
                              const int32_t *inv_perm, const int32_t *base,
                              const void *const *recv_y, int64_t recv_rows, const void *y_shared,
                              int T, int d, int E, int K, int world, void *out, int32_t *status,
                              cudaStream_t st);

// pack.cu: expert weights as tile-contiguous, pre-swizzled 32 KB blocks
// (byte offsets of the four regions inside the packed buffer)
struct PackedLayout {
    int nt1, kb1, nt2, kb2, nt1s, kb2s;  // column tiles / k blocks per region
    size_t gu, down, gu_s, down_s, total;
};
PackedLayout packed_layout(int E, int d, int d_ff, int n_shared, int d_ff_shared);
cudaError_t launch_pack_weights(int E, int d, int d_ff, int n_shared, int d_ff_shared,
                                const void *w_gate, const void *w_up, const void *w_down,
                                const void *ws_gate, const void *ws_up, const void *ws_down,
                                void *packed, cudaStream_t st);

// combine.cu
cudaError_t launch_combine(const void *y_perm, const int32_t *inv_perm, const float *topk_w,
                           const void *y_shared, int T, int d, int K, int64_t n_rows, void *out,
                           cudaStream_t st);

// gemm_sm100.cu
struct FfnArgs {
    int T, d, E, K, d_ff, n_shared, d_ff_shared;
    const void *x_perm;        // [T*K, d] bf16, or unused when perm_token / x_perm_q is set
    const int32_t *perm_token; // [T*K] or nullptr: routed row r of GEMM1 is x[perm_token[r]]
    const uint8_t *x_perm_q;   // [T*K, d] FP8 E4M3 payload or nullptr (with x_scale)
    const float *x_scale;      // [T*K, d/128]
    const int32_t *offsets;
    const void *w_gate, *w_up, *w_down;
    void *h;        // [T*K, d_ff] bf16 scratch
    void *y_perm;   // [T*K, d] bf16
    const void *x;  // [T, d]
    const void *ws_gate, *ws_up, *ws_down;
    const void *packed;  // weights from launch_pack_weights, or null: the row-major ones above
    void *h_shared; // [T, n_shared*d_ff_shared] bf16 scratch
    void *y_shared; // [T, d]
    int32_t *status;   // the workspace's 256-byte status block: word 0 the status,
                       // words 16 and 17 the grouped GEMMs' tile counters
    int64_t timeout_ns;
};
cudaError_t launch_expert_ffn(const FfnArgs &a, cudaStream_t st);
// router_tc.cu: router affinities on the tensor cores; e (fp32 [E, d]) is
// split into three bf16 parts in e_split ([3, E, d] bf16 scratch);
// scores = f(x.e + off), f = sigmoid (affinity 0) or sqrt(softplus) (1).
// Work is split over d into router_splits(T, E, d) ranges when the batch has
// too few 128 x 128 tiles to fill the SMs; partial ([splits, T, E] fp32
// scratch, needed when splits > 1) holds their logits.
inline int router_splits(int T, int E, int d) {
    const int tiles = ((T + 127) / 128) * ((E + 127) / 128);
    const int kmax = d / 64 / 4;  // at least four k blocks per range
    int s = tiles > 0 ? 148 / tiles : 1;
    if (s > kmax) s = kmax;
    return s < 1 ? 1 : s;
}
cudaError_t launch_router_logits_tc(const void *x, const float *e, const float *off, int T, int d,
                                    int E, int affinity, void *e_split, float *partial,
                                    float *scores, int32_t *status, int64_t timeout_ns,
                                    cudaStream_t st);

// router_tc.cu: e (fp32 [E, d]) -> its three exact bf16 parts e_split [3, E, d]
cudaError_t launch_router_split(const float *e, int E, int d, void *e_split, cudaStream_t st);

// router_fused.cu: affinities and node-limited top-K in one kernel (E <= 256,
// G <= 32, E/G <= 32), from the bf16 parts written by launch_router_split;
// scores (nullable) receives the affinities.  The reduction over d is split
// over a cluster of router_fused_cluster(T, d) CTAs.
bool router_fused_supported(int E, int G, int K);
int router_fused_cluster(int T, int d);
cudaError_t launch_router_select_fused(const void *x, const void *e_split, const float *off,
                                       const float *bias, int T, int d, int E, int G, int K,
                                       int M, int affinity, float *scores, int32_t *topk_idx,
                                       float *topk_w, int32_t *status, int64_t timeout_ns,
                                       cudaStream_t st);

// route_variants.cu: the hash router (token ids -> K experts in M groups,
// gates 1/K; token_ids NULL = row index) and the per-expert bias update.
cudaError_t launch_hash_route(const int64_t *token_ids, int T, int E, int G, int K, int M,
                              int32_t *topk_idx, float *topk_w, cudaStream_t st);
cudaError_t launch_bias_update(const int32_t *counts, int E, int T, int K, float gamma,
                               float *bias, cudaStream_t st);
cudaError_t launch_bounded_wait_selftest(int64_t timeout_ns, int32_t *status, cudaStream_t st);

}  // namespace moe
