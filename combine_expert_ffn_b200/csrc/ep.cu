// ep.cu -- expert parallelism: the dispatch and combine all-to-alls fused
// with their gather and reduce, over peer memory.
//
// The pages' layout: experts are partitioned over the ranks (contiguous blocks
// of E / world per rank, "four experts per GPU", deepnotes "The real cluster,
// and the mesh DeepSeek actually disclosed"), each rank routes its own tokens,
// and the dispatch all-to-all sends every token copy to the rank owning its
// expert; the combine all-to-all brings the expert outputs back
// ("moe-node-limited-routing", "Why all to all dominates MoE step time").
//
// Receive layout at owner o: its experts' segments in expert order; inside a
// segment, the copies from source rank 0, then 1, ... , each source's in its
// token order.  With the batch split into equal contiguous rank chunks this
// is exactly the single-GPU x_perm restricted to o's experts, so every row
// meets the same expert GEMM arithmetic and the layer's output is the same.
//
// Per rank, with counts_all[r][e] the copies of rank r to expert e:
//   base[e]          = first row of this rank's copies for e at owner(e)
//                    = seg_start(e) + sum_{r < me} counts_all[r][e]
//   local_offsets[i] = seg_start(me * El + i) at this rank as owner
// dispatch: x row of copy (t, j) -> recv_x[owner(e)][base[e] + rank of t
//           among this rank's tokens choosing e]; one load, K peer stores
// combine:  out[t] = y_shared[t] + sum_j w_j recv_y[owner(e_j)][same row],
//           fp32 multiply-adds in slot order (as the single-GPU combine)
// FP8 payload (E4M3 codes + one fp32 scale per 128 channels, quantized once
// at the source with the single-GPU FP8 gather's quantizer): recv_q [cap, d]
// bytes and recv_scale [cap, d / 128] fp32 per owner take the place of recv_x,
// and the owner's expert FFN widens the codes inside its GEMM.
// Deduplicated dispatch ("moe-node-limited-routing": the node limit bounds the
// nodes a token's activations must reach): a token's row crosses to each owner
// holding one of its experts once, into recv_tok[owner] (rows: rank 0's
// tokens, then rank 1's, ..., each in token order; tok_base[o] = this rank's
// first row there, tok_slot[t][o] = t's position among this rank's tokens
// for o), and each copy (t, j) writes only its 4-byte index
// recv_idx[owner][copy row] = token row.  The owner's fan-out then builds
// recv_x[r] = recv_tok[recv_idx[r]] locally: the same rows, so the same GEMM
// input as without deduplication.
// recv_x / recv_y are device arrays of `world` device pointers: this GPU's
// buffers and peers' buffers mapped into its address space; the kernels use
// plain loads and stores through them.  Each block first builds in shared
// memory, per expert, delta[e] = base[e] - offsets[e] and the address of the
// row delta[e] in owner(e)'s buffer, so a copy's address is that pointer plus
// inv_perm[t][j] rows: one global load (beside topk_idx) before the row itself,
// as in the single-GPU gather and combine.
#include "fp8_payload.cuh"
#include "kernels.h"

namespace moe {

namespace {

__global__ void ep_plan_kernel(const int32_t *__restrict__ counts_all, int world, int E, int me,
                               int32_t *__restrict__ base, int32_t *__restrict__ local_offsets) {
    // one block; thread e owns expert e (E <= 1024)
    __shared__ int32_t col[1024];   // sum over ranks of counts_all[.][e]
    __shared__ int32_t start[1024]; // seg_start(e) within owner(e)'s buffer
    const int e = threadIdx.x;
    const int El = E / world;
    if (e < E) {
        int s = 0;
        for (int r = 0; r < world; ++r) s += counts_all[r * E + e];
        col[e] = s;
    }
    __syncthreads();
    if (e < E) {
        const int first = (e / El) * El;  // first expert of owner(e)
        int st = 0;
        for (int q = first; q < e; ++q) st += col[q];
        start[e] = st;
        int b = st;
        for (int r = 0; r < me; ++r) b += counts_all[r * E + e];
        base[e] = b;
    }
    __syncthreads();
    if (e < El) local_offsets[e] = start[me * El + e];
    // the end of the last local segment; written by thread 0 because El may be 1024,
    // one past the last thread of the block
    if (e == 0) local_offsets[El] = start[me * El + El - 1] + col[me * El + El - 1];
}

constexpr int EP_MAX_E = 1024, EP_MAX_WORLD = 64;

// delta[e] = base[e] - offsets[e] and the address of row delta[e] of
// owner(e)'s buffer, for every expert, in shared memory
template <typename P>
__device__ __forceinline__ void ep_stage_rows(const int32_t *__restrict__ offsets,
                                              const int32_t *__restrict__ base,
                                              P const *__restrict__ table, int E, int El,
                                              int chunks, int32_t *delta_s, P *rowbase_s) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int32_t dl = base[e] - offsets[e];
        delta_s[e] = dl;
        rowbase_s[e] = table[e / El] + (int64_t)dl * chunks;
    }
    __syncthreads();
}

__global__ void __launch_bounds__(256, 4)
ep_dispatch_kernel(const uint4 *__restrict__ x, const int32_t *__restrict__ topk_idx,
                   const int32_t *__restrict__ offsets, const int32_t *__restrict__ inv_perm,
                   const int32_t *__restrict__ base, uint4 *const *__restrict__ recv_x,
                   int64_t recv_rows, int T, int chunks, int E, int K, int El, int32_t *status) {
    __shared__ int32_t delta_s[EP_MAX_E];
    __shared__ uint4 *rowbase_s[EP_MAX_E];
    ep_stage_rows(offsets, base, recv_x, E, El, chunks, delta_s, rowbase_s);
    const int64_t total = (int64_t)T * chunks;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / chunks;
        const int c = (int)(i - t * chunks);
        const uint4 v = __ldg(x + i);
        for (int j0 = 0; j0 < K; j0 += 8) {
            int e8[8], r8[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int j = j0 + q;
                e8[q] = -1;
                if (j < K) {
                    e8[q] = __ldg(topk_idx + t * K + j);
                    r8[q] = __ldg(inv_perm + t * K + j);
                }
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int e = e8[q];
                if (e < 0 || e >= E) continue;  // flagged by the local dispatch plan
                const int64_t row = (int64_t)delta_s[e] + r8[q];
                if (row < 0 || row >= recv_rows) {
                    if (status) record_status(status, MOE_ERR_DEVICE_FAULT);
                    continue;
                }
                rowbase_s[e][(int64_t)r8[q] * chunks + c] = v;
            }
        }
    }
}

// FP8 payload: one 16-lane group per (token, 128-channel block), as the
// single-GPU FP8 gather; the codes and the scale go to the K owners' rows.
__global__ void __launch_bounds__(256, 4)
ep_dispatch_fp8_kernel(const uint4 *__restrict__ x, const int32_t *__restrict__ topk_idx,
                       const int32_t *__restrict__ offsets, const int32_t *__restrict__ inv_perm,
                       const int32_t *__restrict__ base, uint2 *const *__restrict__ recv_q,
                       float *const *__restrict__ recv_scale, int64_t recv_rows, int T, int chunks,
                       int E, int K, int El, int32_t *status) {
    __shared__ int32_t delta_s[EP_MAX_E];
    __shared__ uint2 *rowq_s[EP_MAX_E];
    __shared__ float *rows_s[EP_MAX_E];
    const int blocks = chunks >> 4;  // 128-channel blocks per row
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int32_t dl = base[e] - offsets[e];
        delta_s[e] = dl;
        rowq_s[e] = recv_q[e / El] + (int64_t)dl * chunks;
        rows_s[e] = recv_scale[e / El] + (int64_t)dl * blocks;
    }
    __syncthreads();
    const int64_t total = (int64_t)T * chunks;  // a multiple of 16: groups never straddle it
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i0 = blockIdx.x * (int64_t)blockDim.x + (threadIdx.x & ~31); i0 < total;
         i0 += stride) {
        const int64_t i = i0 + lane;
        const bool in = i < total;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (in) v = __ldg(x + i);
        float sc;
        const uint2 packed = e4m3_quantize_chunk(v, &sc);
        if (!in) continue;
        const int64_t t = i / chunks;
        const int c = (int)(i - t * chunks);
        for (int j = 0; j < K; ++j) {
            const int e = __ldg(topk_idx + t * K + j);
            const int r = __ldg(inv_perm + t * K + j);
            if (e < 0 || e >= E) continue;  // flagged by the local dispatch plan
            const int64_t row = (int64_t)delta_s[e] + r;
            if (row < 0 || row >= recv_rows) {
                if (status) record_status(status, MOE_ERR_DEVICE_FAULT);
                continue;
            }
            rowq_s[e][(int64_t)r * chunks + c] = packed;
            if ((c & 15) == 0) rows_s[e][(int64_t)r * blocks + (c >> 4)] = sc;
        }
    }
}

// tok_slot / tok_counts of one owner o = blockIdx.x: a block-wide exclusive
// scan over this rank's tokens of "t has an expert at o", in token order.
__global__ void __launch_bounds__(1024)
ep_token_plan_kernel(const int32_t *__restrict__ topk_idx, int T, int K, int E, int El, int world,
                     int32_t *__restrict__ tok_slot, int32_t *__restrict__ tok_counts) {
    __shared__ int warp_excl[32];
    __shared__ int total_s, carry_s;
    const int o = blockIdx.x;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    if (threadIdx.x == 0) carry_s = 0;
    __syncthreads();
    for (int t0 = 0; t0 < T; t0 += blockDim.x) {
        const int t = t0 + threadIdx.x;
        int flag = 0;
        if (t < T) {
            for (int j = 0; j < K; ++j) {
                const int e = __ldg(topk_idx + (int64_t)t * K + j);
                if (e >= 0 && e < E && e / El == o) flag = 1;
            }
        }
        const unsigned bal = __ballot_sync(0xFFFFFFFFu, flag);
        const int in_warp = __popc(bal & ((1u << lane) - 1u));
        if (lane == 0) warp_excl[wid] = __popc(bal);
        __syncthreads();
        if (wid == 0) {
            const int v = lane < nwarps ? warp_excl[lane] : 0;
            int incl = v;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int n = __shfl_up_sync(0xFFFFFFFFu, incl, d);
                if (lane >= d) incl += n;
            }
            if (lane < nwarps) warp_excl[lane] = incl - v;
            if (lane == 31) total_s = incl;
        }
        __syncthreads();
        const int carry = carry_s;
        if (t < T) tok_slot[(int64_t)t * world + o] = flag ? carry + warp_excl[wid] + in_warp : -1;
        __syncthreads();  // every thread has read carry_s and warp_excl
        if (threadIdx.x == 0) carry_s = carry + total_s;
        __syncthreads();
    }
    if (threadIdx.x == 0) tok_counts[o] = carry_s;
}

// tok_base[o] = sum over ranks r < me of tok_counts_all[r][o]; tok_base[world]
// = the token rows this rank receives as an owner
__global__ void ep_token_base_kernel(const int32_t *__restrict__ tok_counts_all, int world, int me,
                                     int32_t *__restrict__ tok_base) {
    const int o = threadIdx.x;
    if (o < world) {
        int s = 0;
        for (int r = 0; r < me; ++r) s += tok_counts_all[r * world + o];
        tok_base[o] = s;
    } else if (o == world) {
        int s = 0;
        for (int r = 0; r < world; ++r) s += tok_counts_all[r * world + me];
        tok_base[world] = s;
    }
}

// Thread per 16-byte chunk of an x row: one store per (token, owner) of the
// row, one 4-byte index store per copy (by the chunk-0 thread).
__global__ void __launch_bounds__(256, 4)
ep_dispatch_dedup_kernel(const uint4 *__restrict__ x, const int32_t *__restrict__ topk_idx,
                         const int32_t *__restrict__ offsets, const int32_t *__restrict__ inv_perm,
                         const int32_t *__restrict__ base, const int32_t *__restrict__ tok_slot,
                         const int32_t *__restrict__ tok_base, uint4 *const *__restrict__ recv_tok,
                         int32_t *const *__restrict__ recv_idx, int64_t tok_rows,
                         int64_t recv_rows, int T, int chunks, int E, int K, int El, int world,
                         int32_t *status) {
    __shared__ int32_t delta_s[EP_MAX_E];
    __shared__ int32_t tokbase_s[EP_MAX_WORLD];
    __shared__ uint4 *tok_tab_s[EP_MAX_WORLD];
    __shared__ int32_t *idx_tab_s[EP_MAX_WORLD];
    for (int e = threadIdx.x; e < E; e += blockDim.x) delta_s[e] = base[e] - offsets[e];
    for (int o = threadIdx.x; o < world; o += blockDim.x) {
        tokbase_s[o] = tok_base[o];
        tok_tab_s[o] = recv_tok[o];
        idx_tab_s[o] = recv_idx[o];
    }
    __syncthreads();
    const int64_t total = (int64_t)T * chunks;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / chunks;
        const int c = (int)(i - t * chunks);
        const uint4 v = __ldg(x + i);
        const int32_t *idx_t = topk_idx + t * K;
        uint64_t sent = 0;  // owners this token's row has gone to (world <= 64)
        for (int j0 = 0; j0 < K; j0 += 8) {
            int o8[8], s8[8], r8[8];
            int e8[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {  // independent loads first
                const int j = j0 + q;
                e8[q] = -1;
                r8[q] = 0;
                if (j < K) {
                    e8[q] = __ldg(idx_t + j);
                    if (c == 0) r8[q] = __ldg(inv_perm + t * K + j);
                }
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int e = e8[q];
                o8[q] = e >= 0 && e < E ? e / El : -1;  // invalid ids: flagged by the local plan
                s8[q] = o8[q] >= 0 ? __ldg(tok_slot + t * world + o8[q]) : -1;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int o = o8[q];
                if (o < 0) continue;
                const int64_t trow = (int64_t)tokbase_s[o] + s8[q];
                if (s8[q] < 0 || trow >= tok_rows) {
                    if (status) record_status(status, MOE_ERR_DEVICE_FAULT);
                    continue;
                }
                if (!((sent >> o) & 1ull)) {  // the token's first slot at owner o
                    sent |= 1ull << o;
                    tok_tab_s[o][trow * chunks + c] = v;
                }
                if (c == 0) {
                    const int64_t row = (int64_t)delta_s[e8[q]] + r8[q];
                    if (row < 0 || row >= recv_rows) {
                        if (status) record_status(status, MOE_ERR_DEVICE_FAULT);
                        continue;
                    }
                    idx_tab_s[o][row] = (int32_t)trow;
                }
            }
        }
    }
}

// The deduplicated dispatch on the copy engine.  Warp per token row: lane 0
// loads the row into a shared-memory buffer of the warp (cp.async.bulk,
// completion on an mbarrier); lane o < world (and o + 32) stores it to owner o's token buffer at
// tok_base[o] + tok_slot[t][o] when the token has an expert there
// (cp.async.bulk shared -> global, through the owner's pointer); lane j < K
// writes copy (t, j)'s 4-byte token row into the owner's recv_idx.  The token
// plan already lists every destination, so no lane walks the copies to find
// them.
// NB row buffers per warp: 2 (4 warps per CTA) overlaps a row's load with
// the previous row's stores when a warp walks several rows; 1 (8 warps per
// CTA) puts twice as many rows in flight when there are about as many rows as
// warps (the per-rank batches of an expert-parallel step).
// PLAN: the same launch also writes the deduplicated combine's lists (what
// ep_combine_plan_kernel writes): lane j < K knows copy (t, j)'s owner, token
// row and copy row, and its slot k among the token's copies at that owner is
// the number of lower lanes with the same owner (a warp match).
template <int NB>
__host__ __device__ constexpr int db_warps() { return NB == 2 ? 4 : 8; }

__device__ __forceinline__ void db_drain(uint32_t bar, uint32_t parity, int64_t timeout_ns) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity) && (int64_t)(globaltimer_ns() - t0) < timeout_ns) {
    }
}

template <int NB, bool PLAN>
__global__ void __launch_bounds__(db_warps<NB>() * 32)
ep_dispatch_dedup_bulk_kernel(const char *__restrict__ x, const int32_t *__restrict__ topk_idx,
                              const int32_t *__restrict__ offsets,
                              const int32_t *__restrict__ inv_perm,
                              const int32_t *__restrict__ base, const int32_t *__restrict__ tok_slot,
                              const int32_t *__restrict__ tok_base, char *const *__restrict__ recv_tok,
                              int32_t *const *__restrict__ recv_idx, int64_t tok_rows,
                              int64_t recv_rows, int T, int row_bytes, int E, int K, int El,
                              int world, int32_t *status, int64_t timeout_ns,
                              const float *__restrict__ topk_w, int32_t *const *__restrict__ list,
                              float *const *__restrict__ lw, int32_t *const *__restrict__ lcnt) {
    constexpr int WARPS = db_warps<NB>();
    extern __shared__ __align__(128) uint8_t dsm_rows[];
    __shared__ int32_t delta_s[EP_MAX_E];
    __shared__ int32_t tokbase_s[EP_MAX_WORLD];
    __shared__ char *tok_tab_s[EP_MAX_WORLD];
    __shared__ int32_t *idx_tab_s[EP_MAX_WORLD];
    __shared__ int32_t *list_s[PLAN ? EP_MAX_WORLD : 1];
    __shared__ float *lw_s[PLAN ? EP_MAX_WORLD : 1];
    __shared__ int32_t *lcnt_s[PLAN ? EP_MAX_WORLD : 1];
    __shared__ __align__(8) uint64_t lbar[WARPS][2];
    __shared__ int abort_s[WARPS];
    for (int e = threadIdx.x; e < E; e += blockDim.x) delta_s[e] = base[e] - offsets[e];
    for (int o = threadIdx.x; o < world; o += blockDim.x) {
        tokbase_s[o] = tok_base[o];
        tok_tab_s[o] = recv_tok[o];
        idx_tab_s[o] = recv_idx[o];
        if (PLAN) {
            list_s[o] = list[o];
            lw_s[o] = lw[o];
            lcnt_s[o] = lcnt[o];
        }
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t buf0 = smem_u32(dsm_rows) + (uint32_t)(warp * NB * row_bytes);
    const uint32_t bar0 = smem_u32(&lbar[warp][0]), bar1 = smem_u32(&lbar[warp][1]);
    if (lane == 0) {
        mbar_init(bar0, 1);
        mbar_init(bar1, 1);
        abort_s[warp] = 0;
        fence_barrier_init();
    }
    __syncthreads();
    const int nw = gridDim.x * WARPS;
    int t = blockIdx.x * WARPS + warp;
    uint32_t in_flight = 0, ph = 0;
    if (NB == 2 && t < T && lane == 0) {
        mbar_arrive_expect_tx(bar0, row_bytes);
        bulk_load(buf0, x + (size_t)t * row_bytes, row_bytes, bar0);
        in_flight = 1u;
    }
    for (int i = 0; t < T; t += nw, ++i) {
        const int b = NB == 2 ? (i & 1) : 0;
        const int tn = t + nw;
        // this token's destinations: owner lane (and lane + 32) and copy lane j < K
        int64_t trow0 = -1, trow1 = -1;
        if (lane < world) {
            const int sl = __ldg(tok_slot + (int64_t)t * world + lane);
            if (sl >= 0) trow0 = (int64_t)tokbase_s[lane] + sl;
        }
        if (lane + 32 < world) {
            const int sl = __ldg(tok_slot + (int64_t)t * world + lane + 32);
            if (sl >= 0) trow1 = (int64_t)tokbase_s[lane + 32] + sl;
        }
        int po = -1;           // owner of copy (t, lane); -1: no copy in this lane
        int64_t ptrow = -1, prow = -1;  // its token row and copy row there (-1: out of bounds)
        if (lane < K) {
            const int e = __ldg(topk_idx + (int64_t)t * K + lane);
            if (e >= 0 && e < E) {  // invalid ids: flagged by the local plan
                const int o = e / El;
                po = o;
                const int sl = __ldg(tok_slot + (int64_t)t * world + o);
                const int64_t trow = (int64_t)tokbase_s[o] + sl;
                const int64_t row = (int64_t)delta_s[e] + __ldg(inv_perm + (int64_t)t * K + lane);
                if (sl < 0 || trow >= tok_rows || row < 0 || row >= recv_rows) {
                    if (status) record_status(status, MOE_ERR_DEVICE_FAULT);
                } else {
                    idx_tab_s[o][row] = (int32_t)trow;
                    ptrow = trow;
                    prow = row;
                }
            }
        }
        if (PLAN) {  // the token's lanes at one owner, in slot order (warp-uniform loop)
            const unsigned grp = __match_any_sync(0xFFFFFFFFu, po >= 0 ? po : -1 - lane);
            if (prow >= 0) {
                const int k = __popc(grp & ((1u << lane) - 1u));
                list_s[po][ptrow * K + k] = (int32_t)prow;
                lw_s[po][ptrow * K + k] = __ldg(topk_w + (int64_t)t * K + lane);
                if (k == 0) lcnt_s[po][ptrow] = __popc(grp);
            }
        }
        // the buffer to load next: every store that read it has read it
        bulk_wait_group_read<0>();
        __syncwarp();
        if (lane == 0) {
            if (NB == 1) {  // this row, into the warp's single buffer
                mbar_arrive_expect_tx(bar0, row_bytes);
                bulk_load(buf0, x + (size_t)t * row_bytes, row_bytes, bar0);
                in_flight = 1u;
            } else if (tn < T) {  // the next row, into the other buffer
                const uint32_t nb = b ? bar0 : bar1;
                mbar_arrive_expect_tx(nb, row_bytes);
                bulk_load(buf0 + (uint32_t)((b ^ 1) * row_bytes), x + (size_t)tn * row_bytes,
                          row_bytes, nb);
                in_flight |= 1u << (b ^ 1);
            }
        }
        const uint32_t bar = b ? bar1 : bar0, par = (ph >> b) & 1u;
        int ok = 1;
        if (lane == 0) {
            ok = mbar_wait_bounded(bar, par, &abort_s[warp], status, timeout_ns);
            if (ok) in_flight &= ~(1u << b);
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (!ok) break;
        ph ^= 1u << b;
        const bool st0 = trow0 >= 0 && trow0 < tok_rows, st1 = trow1 >= 0 && trow1 < tok_rows;
        if ((trow0 >= tok_rows || trow1 >= tok_rows) && status)
            record_status(status, MOE_ERR_DEVICE_FAULT);
        if (st0 || st1) mbar_try_wait(bar, par);  // observe the completed phase before reading
        const uint32_t src = buf0 + (uint32_t)(b * row_bytes);
        if (st0) bulk_store(tok_tab_s[lane] + trow0 * row_bytes, src, row_bytes);
        if (st1) bulk_store(tok_tab_s[lane + 32] + trow1 * row_bytes, src, row_bytes);
        bulk_commit_group();
    }
    bulk_wait_group_all();
    if (lane == 0) {  // after a timeout: loads still in flight into this warp's buffers
        if (in_flight & 1u) db_drain(bar0, ph & 1u, timeout_ns);
        if (in_flight & 2u) db_drain(bar1, (ph >> 1) & 1u, timeout_ns);
    }
}

__device__ __forceinline__ void ep_acc_row(float (&acc)[8], float wj, const uint4 &v) {
    acc[0] = fmaf(wj, bf16_lo(v.x), acc[0]); acc[1] = fmaf(wj, bf16_hi(v.x), acc[1]);
    acc[2] = fmaf(wj, bf16_lo(v.y), acc[2]); acc[3] = fmaf(wj, bf16_hi(v.y), acc[3]);
    acc[4] = fmaf(wj, bf16_lo(v.z), acc[4]); acc[5] = fmaf(wj, bf16_hi(v.z), acc[5]);
    acc[6] = fmaf(wj, bf16_lo(v.w), acc[6]); acc[7] = fmaf(wj, bf16_hi(v.w), acc[7]);
}

// Deduplicated combine, source side, before the exchange: for every token t
// and owner o holding cnt of its copies, the owner's list entry of token row
// trow = tok_base[o] + tok_slot[t][o]: copy rows and gates of those copies in
// slot order (list[trow * K + k], lw[trow * K + k], k < cnt = lcnt[trow]).
// Thread per copy (t, j).
__global__ void __launch_bounds__(256)
ep_combine_plan_kernel(const int32_t *__restrict__ topk_idx, const float *__restrict__ topk_w,
                       const int32_t *__restrict__ offsets, const int32_t *__restrict__ inv_perm,
                       const int32_t *__restrict__ base, const int32_t *__restrict__ tok_slot,
                       const int32_t *__restrict__ tok_base, int32_t *const *__restrict__ list,
                       float *const *__restrict__ lw, int32_t *const *__restrict__ lcnt,
                       int64_t tok_rows, int64_t recv_rows, int T, int E, int K, int El, int world,
                       int32_t *status) {
    __shared__ int32_t delta_s[EP_MAX_E];
    for (int e = threadIdx.x; e < E; e += blockDim.x) delta_s[e] = base[e] - offsets[e];
    __syncthreads();
    const int64_t copy = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (copy >= (int64_t)T * K) return;
    const int64_t t = copy / K;
    const int j = (int)(copy - t * K);
    const int32_t *idx_t = topk_idx + t * K;
    const int e = idx_t[j];
    if (e < 0 || e >= E) return;  // flagged by the local dispatch plan
    const int o = e / El;
    int k = 0, cnt = 0;  // earlier slots at o; all slots at o
    for (int q = 0; q < K; ++q) {
        const int eq = idx_t[q];
        if (eq >= 0 && eq < E && eq / El == o) {
            if (q < j) ++k;
            ++cnt;
        }
    }
    const int slot = tok_slot[(int64_t)t * world + o];
    const int64_t trow = (int64_t)tok_base[o] + slot;
    const int64_t row = (int64_t)delta_s[e] + inv_perm[(int64_t)t * K + j];
    if (slot < 0 || trow >= tok_rows || row < 0 || row >= recv_rows) {
        if (status) record_status(status, MOE_ERR_DEVICE_FAULT);
        return;
    }
    list[o][trow * K + k] = (int32_t)row;
    lw[o][trow * K + k] = topk_w[(int64_t)t * K + j];
    if (k == 0) lcnt[o][trow] = cnt;
}

// Deduplicated combine, owner side: partial[trow] = bf16(sum over k < cnt of
// lw[k] * recv_y[list[k]]), fp32 multiply-adds in slot order, for the token
// rows this rank received (tok_base[world] of them).
__global__ void __launch_bounds__(256, 4)
ep_precombine_kernel(const uint4 *__restrict__ recv_y, const int32_t *__restrict__ list,
                     const float *__restrict__ lw, const int32_t *__restrict__ lcnt,
                     const int32_t *__restrict__ tok_base, int world, int64_t tok_rows,
                     int64_t recv_rows, int chunks, int K, uint4 *__restrict__ partial,
                     int32_t *status) {
    int64_t n = tok_base[world];
    if (n < 0 || n > tok_rows) {
        if (status && blockIdx.x == 0 && threadIdx.x == 0) record_status(status, MOE_ERR_DEVICE_FAULT);
        n = n < 0 ? 0 : tok_rows;
    }
    const int64_t total = n * chunks;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t tr = i / chunks;
        const int c = (int)(i - tr * chunks);
        int cnt = __ldg(lcnt + tr);
        if (cnt < 1 || cnt > K) {
            if (status) record_status(status, MOE_ERR_DEVICE_FAULT);
            cnt = 0;
        }
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
        for (int k0 = 0; k0 < cnt; k0 += 8) {
            uint4 rows[8];
            float w[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int k = k0 + q;
                rows[q] = make_uint4(0u, 0u, 0u, 0u);
                w[q] = 0.f;
                if (k >= cnt) continue;
                const int64_t row = __ldg(list + tr * K + k);
                w[q] = __ldg(lw + tr * K + k);
                if (row < 0 || row >= recv_rows) {
                    if (status) record_status(status, MOE_ERR_DEVICE_FAULT);
                    continue;
                }
                rows[q] = __ldg(recv_y + row * chunks + c);
            }
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (k0 + q < cnt) ep_acc_row(acc, w[q], rows[q]);
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        partial[i] = o;
    }
}

// Deduplicated combine, source side, after the exchange: out[t] = y_shared[t]
// + the partial rows of t's owners (one peer load per owner), added in fp32 in
// the order of each owner's first slot.
__global__ void __launch_bounds__(256, 4)
ep_combine_dedup_kernel(const int32_t *__restrict__ topk_idx, const int32_t *__restrict__ tok_slot,
                        const int32_t *__restrict__ tok_base,
                        const uint4 *const *__restrict__ partial, const uint4 *__restrict__ y_shared,
                        int64_t tok_rows, int T, int chunks, int E, int K, int El, int world,
                        uint4 *__restrict__ out, int32_t *status) {
    __shared__ int32_t tokbase_s[EP_MAX_WORLD];
    __shared__ const uint4 *tab_s[EP_MAX_WORLD];
    for (int o = threadIdx.x; o < world; o += blockDim.x) {
        tokbase_s[o] = tok_base[o];
        tab_s[o] = partial[o];
    }
    __syncthreads();
    const int64_t total = (int64_t)T * chunks;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / chunks;
        const int c = (int)(i - t * chunks);
        float acc[8];
        if (y_shared) {
            const uint4 v = __ldg(y_shared + i);
            acc[0] = bf16_lo(v.x); acc[1] = bf16_hi(v.x);
            acc[2] = bf16_lo(v.y); acc[3] = bf16_hi(v.y);
            acc[4] = bf16_lo(v.z); acc[5] = bf16_hi(v.z);
            acc[6] = bf16_lo(v.w); acc[7] = bf16_hi(v.w);
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = 0.f;
        }
        const int32_t *idx_t = topk_idx + t * K;
        uint64_t seen = 0;
        for (int j0 = 0; j0 < K; j0 += 8) {
            uint4 rows[8];
            bool use[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int j = j0 + q;
                rows[q] = make_uint4(0u, 0u, 0u, 0u);
                use[q] = false;
                if (j >= K) continue;
                const int e = __ldg(idx_t + j);
                if (e < 0 || e >= E) continue;
                const int o = e / El;
                if ((seen >> o) & 1ull) continue;  // this owner's partial is counted once
                seen |= 1ull << o;
                const int slot = __ldg(tok_slot + t * world + o);
                const int64_t trow = (int64_t)tokbase_s[o] + slot;
                if (slot < 0 || trow >= tok_rows) {
                    if (status) record_status(status, MOE_ERR_DEVICE_FAULT);
                    continue;
                }
                rows[q] = tab_s[o][trow * chunks + c];
                use[q] = true;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (use[q]) ep_acc_row(acc, 1.0f, rows[q]);
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        out[i] = o;
    }
}

// Deduplicated dispatch of the FP8 payload: codes and scale of a token go
// once to each owner holding one of its experts (recv_tq / recv_ts token rows),
// plus the 4-byte fan-out index per copy.  One 16-lane group per (token,
// 128-channel block), as the FP8 gather.
__global__ void __launch_bounds__(256, 4)
ep_dispatch_dedup_fp8_kernel(const uint4 *__restrict__ x, const int32_t *__restrict__ topk_idx,
                             const int32_t *__restrict__ offsets,
                             const int32_t *__restrict__ inv_perm,
                             const int32_t *__restrict__ base, const int32_t *__restrict__ tok_slot,
                             const int32_t *__restrict__ tok_base, uint2 *const *__restrict__ recv_tq,
                             float *const *__restrict__ recv_ts,
                             int32_t *const *__restrict__ recv_idx, int64_t tok_rows,
                             int64_t recv_rows, int T, int chunks, int E, int K, int El, int world,
                             int32_t *status) {
    __shared__ int32_t delta_s[EP_MAX_E];
    __shared__ int32_t tokbase_s[EP_MAX_WORLD];
    __shared__ uint2 *tq_s[EP_MAX_WORLD];
    __shared__ float *ts_s[EP_MAX_WORLD];
    __shared__ int32_t *idx_tab_s[EP_MAX_WORLD];
    for (int e = threadIdx.x; e < E; e += blockDim.x) delta_s[e] = base[e] - offsets[e];
    for (int o = threadIdx.x; o < world; o += blockDim.x) {
        tokbase_s[o] = tok_base[o];
        tq_s[o] = recv_tq[o];
        ts_s[o] = recv_ts[o];
        idx_tab_s[o] = recv_idx[o];
    }
    __syncthreads();
    const int blocks = chunks >> 4;
    const int64_t total = (int64_t)T * chunks;  // a multiple of 16: groups never straddle it
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i0 = blockIdx.x * (int64_t)blockDim.x + (threadIdx.x & ~31); i0 < total;
         i0 += stride) {
        const int64_t i = i0 + lane;
        const bool in = i < total;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (in) v = __ldg(x + i);
        float sc;
        const uint2 packed = e4m3_quantize_chunk(v, &sc);
        if (!in) continue;
        const int64_t t = i / chunks;
        const int c = (int)(i - t * chunks);
        const int32_t *idx_t = topk_idx + t * K;
        uint64_t sent = 0;
        for (int j = 0; j < K; ++j) {
            const int e = __ldg(idx_t + j);
            if (e < 0 || e >= E) continue;  // flagged by the local dispatch plan
            const int o = e / El;
            const int slot = __ldg(tok_slot + t * world + o);
            const int64_t trow = (int64_t)tokbase_s[o] + slot;
            if (slot < 0 || trow >= tok_rows) {
                if (status) record_status(status, MOE_ERR_DEVICE_FAULT);
                continue;
            }
            if (!((sent >> o) & 1ull)) {
                sent |= 1ull << o;
                tq_s[o][trow * chunks + c] = packed;
                if ((c & 15) == 0) ts_s[o][trow * blocks + (c >> 4)] = sc;
            }
            if (c == 0) {
                const int64_t row = (int64_t)delta_s[e] + __ldg(inv_perm + t * K + j);
                if (row < 0 || row >= recv_rows) {
                    if (status) record_status(status, MOE_ERR_DEVICE_FAULT);
                    continue;
                }
                idx_tab_s[o][row] = (int32_t)trow;
            }
        }
    }
}

// The owner's fan-out of the FP8 payload: codes (16-byte units) and scales of
// token row recv_idx[r] into copy row r.
__global__ void __launch_bounds__(256, 4)
ep_fanout_fp8_kernel(const uint4 *__restrict__ recv_tq, const float *__restrict__ recv_ts,
                     const int32_t *__restrict__ recv_idx, const int32_t *__restrict__ local_offsets,
                     int El, int64_t tok_rows, int64_t recv_rows, int units, int blocks,
                     uint4 *__restrict__ recv_q, float *__restrict__ recv_scale, int32_t *status) {
    int64_t n = local_offsets[El];
    if (n < 0 || n > recv_rows) {
        if (status && blockIdx.x == 0 && threadIdx.x == 0) record_status(status, MOE_ERR_DEVICE_FAULT);
        n = n < 0 ? 0 : recv_rows;
    }
    const int per_row = units + blocks;
    const int64_t total = n * per_row;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / per_row;
        const int u = (int)(i - r * per_row);
        const int64_t src = __ldg(recv_idx + r);
        if (src < 0 || src >= tok_rows) {
            if (status) record_status(status, MOE_ERR_DEVICE_FAULT);
            continue;
        }
        if (u < units)
            recv_q[r * units + u] = __ldg(recv_tq + src * units + u);
        else
            recv_scale[r * blocks + (u - units)] = __ldg(recv_ts + src * blocks + (u - units));
    }
}

// The owner's fan-out: recv_x[r] = recv_tok[recv_idx[r]] for the rows it
// received (local_offsets[El] of them).
__global__ void __launch_bounds__(256, 4)
ep_fanout_kernel(const uint4 *__restrict__ recv_tok, const int32_t *__restrict__ recv_idx,
                 const int32_t *__restrict__ local_offsets, int El, int64_t tok_rows,
                 int64_t recv_rows, int chunks, uint4 *__restrict__ recv_x, int32_t *status) {
    int64_t n = local_offsets[El];
    if (n < 0 || n > recv_rows) {
        if (status && blockIdx.x == 0 && threadIdx.x == 0) record_status(status, MOE_ERR_DEVICE_FAULT);
        n = n < 0 ? 0 : recv_rows;
    }
    const int64_t total = n * chunks;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / chunks;
        const int c = (int)(i - r * chunks);
        const int64_t src = __ldg(recv_idx + r);
        if (src < 0 || src >= tok_rows) {
            if (status) record_status(status, MOE_ERR_DEVICE_FAULT);
            continue;
        }
        recv_x[i] = __ldg(recv_tok + src * chunks + c);
    }
}


__global__ void __launch_bounds__(256, 4)
ep_combine_kernel(const int32_t *__restrict__ topk_idx, const float *__restrict__ topk_w,
                  const int32_t *__restrict__ offsets, const int32_t *__restrict__ inv_perm,
                  const int32_t *__restrict__ base, const uint4 *const *__restrict__ recv_y,
                  int64_t recv_rows, const uint4 *__restrict__ y_shared, int T, int chunks,
                  int E, int K, int El, uint4 *__restrict__ out, int32_t *status) {
    __shared__ int32_t delta_s[EP_MAX_E];
    __shared__ const uint4 *rowbase_s[EP_MAX_E];
    ep_stage_rows(offsets, base, recv_y, E, El, chunks, delta_s, rowbase_s);
    const int64_t total = (int64_t)T * chunks;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / chunks;
        const int c = (int)(i - t * chunks);
        float acc[8];
        if (y_shared) {
            const uint4 v = __ldg(y_shared + i);
            acc[0] = bf16_lo(v.x); acc[1] = bf16_hi(v.x);
            acc[2] = bf16_lo(v.y); acc[3] = bf16_hi(v.y);
            acc[4] = bf16_lo(v.z); acc[5] = bf16_hi(v.z);
            acc[6] = bf16_lo(v.w); acc[7] = bf16_hi(v.w);
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = 0.f;
        }
        // slots in batches of 8: every peer load of a batch is in flight before
        // its multiply-adds, which run in slot order
        for (int j0 = 0; j0 < K; j0 += 8) {
            uint4 rows[8];
            float w[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int j = j0 + q;
                rows[q] = make_uint4(0u, 0u, 0u, 0u);
                w[q] = 0.f;
                if (j >= K) continue;
                w[q] = __ldg(topk_w + t * K + j);
                const int e = __ldg(topk_idx + t * K + j);
                const int r = __ldg(inv_perm + t * K + j);
                if (e < 0 || e >= E) continue;
                const int64_t row = (int64_t)delta_s[e] + r;
                if (row < 0 || row >= recv_rows) {
                    if (status) record_status(status, MOE_ERR_DEVICE_FAULT);
                    continue;
                }
                rows[q] = rowbase_s[e][(int64_t)r * chunks + c];
            }
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (j0 + q < K) ep_acc_row(acc, w[q], rows[q]);
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        out[i] = o;
    }
}

// one wave of resident blocks (4 per SM): each block stages its tables once
int grid_for(int64_t total) {
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (total + 255) / 256;
    return (int)(want < (int64_t)sms * 4 ? want : (int64_t)sms * 4);
}

}  // namespace

cudaError_t launch_ep_plan(const int32_t *counts_all, int world, int E, int me, int32_t *base,
                           int32_t *local_offsets, cudaStream_t st) {
    ep_plan_kernel<<<1, 1024, 0, st>>>(counts_all, world, E, me, base, local_offsets);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_ep_dispatch(const void *x, const int32_t *topk_idx, const int32_t *offsets,
                               const int32_t *inv_perm, const int32_t *base, void *const *recv_x,
                               int64_t recv_rows, int T, int d, int E, int K, int world,
                               int32_t *status, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int chunks = d / 8;
    ep_dispatch_kernel<<<grid_for((int64_t)T * chunks), 256, 0, st>>>(
        static_cast<const uint4 *>(x), topk_idx, offsets, inv_perm, base,
        reinterpret_cast<uint4 *const *>(recv_x), recv_rows, T, chunks, E, K, E / world, status);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_ep_dispatch_fp8(const void *x, const int32_t *topk_idx,
                                   const int32_t *offsets, const int32_t *inv_perm,
                                   const int32_t *base, void *const *recv_q,
                                   void *const *recv_scale, int64_t recv_rows, int T, int d, int E,
                                   int K, int world, int32_t *status, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int chunks = d / 8;
    ep_dispatch_fp8_kernel<<<grid_for((int64_t)T * chunks), 256, 0, st>>>(
        static_cast<const uint4 *>(x), topk_idx, offsets, inv_perm, base,
        reinterpret_cast<uint2 *const *>(recv_q), reinterpret_cast<float *const *>(recv_scale),
        recv_rows, T, chunks, E, K, E / world, status);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_ep_token_plan(const int32_t *topk_idx, int T, int E, int K, int world,
                                  int32_t *tok_slot, int32_t *tok_counts, cudaStream_t st) {
    ep_token_plan_kernel<<<world, 1024, 0, st>>>(topk_idx, T, K, E, E / world, world, tok_slot,
                                                 tok_counts);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_ep_token_base(const int32_t *tok_counts_all, int world, int me,
                                 int32_t *tok_base, cudaStream_t st) {
    ep_token_base_kernel<<<1, 96, 0, st>>>(tok_counts_all, world, me, tok_base);
    count_launch();
    return cudaGetLastError();
}

namespace {
// One wave of the bulk dedup dispatch with NB buffers per warp.
template <int NB, bool PLAN>
cudaError_t launch_dedup_bulk(const char *x, const int32_t *topk_idx, const int32_t *offsets,
                              const int32_t *inv_perm, const int32_t *base,
                              const int32_t *tok_slot, const int32_t *tok_base,
                              char *const *recv_tok, int32_t *const *recv_idx, int64_t tok_rows,
                              int64_t recv_rows, int T, int row_bytes, int E, int K, int world,
                              int32_t *status, const float *topk_w, int32_t *const *list,
                              float *const *lw, int32_t *const *lcnt, size_t smem, int sms,
                              cudaStream_t st) {
    constexpr int warps = db_warps<NB>();
    auto kern = ep_dispatch_dedup_bulk_kernel<NB, PLAN>;
    cudaError_t err =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    int per_sm = 1;  // CTAs resident per SM with this shared memory (one wave)
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 32 * warps, smem) !=
            cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const int want = (T + warps - 1) / warps;
    const int grid = want < per_sm * sms ? want : per_sm * sms;
    kern<<<grid, 32 * warps, smem, st>>>(x, topk_idx, offsets, inv_perm, base, tok_slot, tok_base,
                                        recv_tok, recv_idx, tok_rows, recv_rows, T, row_bytes, E,
                                        K, E / world, world, status, 2000000000LL, topk_w, list,
                                        lw, lcnt);
    count_launch();
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_ep_dispatch_dedup(const void *x, const int32_t *topk_idx, const int32_t *offsets,
                                     const int32_t *inv_perm, const int32_t *base,
                                     const int32_t *tok_slot, const int32_t *tok_base,
                                     void *const *recv_tok, int32_t *const *recv_idx,
                                     int64_t tok_rows, int64_t recv_rows, int T, int d, int E, int K,
                                     int world, int32_t *status, cudaStream_t st,
                                     const float *topk_w, int32_t *const *list, float *const *lw,
                                     int32_t *const *lcnt) {
    if (T == 0) return cudaSuccess;
    const bool plan = list != nullptr;
    const int row_bytes = d * 2;
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // one buffer per warp when one wave of eight-warp CTAs covers every row
    const bool one = (int64_t)T <= (int64_t)sms * db_warps<1>();
    const size_t db_smem = (size_t)(one ? db_warps<1>() : db_warps<2>() * 2) * row_bytes;
    if (db_smem <= 112 * 1024) {
        const char *xc = static_cast<const char *>(x);
        char *const *rt = reinterpret_cast<char *const *>(recv_tok);
        if (one && plan)
            return launch_dedup_bulk<1, true>(xc, topk_idx, offsets, inv_perm, base, tok_slot,
                                              tok_base, rt, recv_idx, tok_rows, recv_rows, T,
                                              row_bytes, E, K, world, status, topk_w, list, lw,
                                              lcnt, db_smem, sms, st);
        if (one)
            return launch_dedup_bulk<1, false>(xc, topk_idx, offsets, inv_perm, base, tok_slot,
                                               tok_base, rt, recv_idx, tok_rows, recv_rows, T,
                                               row_bytes, E, K, world, status, nullptr, nullptr,
                                               nullptr, nullptr, db_smem, sms, st);
        if (plan)
            return launch_dedup_bulk<2, true>(xc, topk_idx, offsets, inv_perm, base, tok_slot,
                                              tok_base, rt, recv_idx, tok_rows, recv_rows, T,
                                              row_bytes, E, K, world, status, topk_w, list, lw,
                                              lcnt, db_smem, sms, st);
        return launch_dedup_bulk<2, false>(xc, topk_idx, offsets, inv_perm, base, tok_slot,
                                           tok_base, rt, recv_idx, tok_rows, recv_rows, T,
                                           row_bytes, E, K, world, status, nullptr, nullptr,
                                           nullptr, nullptr, db_smem, sms, st);
    }
    // rows wider than the shared-memory buffers: thread per 16-byte chunk, and the
    // combine's lists (if asked for) from their own launch
    const int chunks = d / 8;
    ep_dispatch_dedup_kernel<<<grid_for((int64_t)T * chunks), 256, 0, st>>>(
        static_cast<const uint4 *>(x), topk_idx, offsets, inv_perm, base, tok_slot, tok_base,
        reinterpret_cast<uint4 *const *>(recv_tok), recv_idx, tok_rows, recv_rows, T, chunks, E,
        K, E / world, world, status);
    count_launch();
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess || !plan) return err;
    return launch_ep_combine_plan(topk_idx, topk_w, offsets, inv_perm, base, tok_slot, tok_base,
                                  list, lw, lcnt, tok_rows, recv_rows, T, E, K, world, status, st);
}

cudaError_t launch_ep_fanout(const void *recv_tok, const int32_t *recv_idx,
                             const int32_t *local_offsets, int El, int64_t tok_rows,
                             int64_t recv_rows, int d, void *recv_x, int32_t *status,
                             cudaStream_t st) {
    if (recv_rows == 0) return cudaSuccess;
    const int chunks = d / 8;
    ep_fanout_kernel<<<grid_for(recv_rows * chunks), 256, 0, st>>>(
        static_cast<const uint4 *>(recv_tok), recv_idx, local_offsets, El, tok_rows, recv_rows,
        chunks, static_cast<uint4 *>(recv_x), status);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_ep_combine_plan(const int32_t *topk_idx, const float *topk_w,
                                   const int32_t *offsets, const int32_t *inv_perm,
                                   const int32_t *base, const int32_t *tok_slot,
                                   const int32_t *tok_base, int32_t *const *list,
                                   float *const *lw, int32_t *const *lcnt, int64_t tok_rows,
                                   int64_t recv_rows, int T, int E, int K, int world,
                                   int32_t *status, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int64_t copies = (int64_t)T * K;
    ep_combine_plan_kernel<<<(unsigned)((copies + 255) / 256), 256, 0, st>>>(
        topk_idx, topk_w, offsets, inv_perm, base, tok_slot, tok_base, list, lw, lcnt, tok_rows,
        recv_rows, T, E, K, E / world, world, status);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_ep_precombine(const void *recv_y, const int32_t *list, const float *lw,
                                 const int32_t *lcnt, const int32_t *tok_base, int world,
                                 int64_t tok_rows, int64_t recv_rows, int d, int K, void *partial,
                                 int32_t *status, cudaStream_t st) {
    if (tok_rows == 0) return cudaSuccess;
    const int chunks = d / 8;
    ep_precombine_kernel<<<grid_for(tok_rows * chunks), 256, 0, st>>>(
        static_cast<const uint4 *>(recv_y), list, lw, lcnt, tok_base, world, tok_rows, recv_rows,
        chunks, K, static_cast<uint4 *>(partial), status);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_ep_combine_dedup(const int32_t *topk_idx, const int32_t *tok_slot,
                                    const int32_t *tok_base, const void *const *partial,
                                    const void *y_shared, int64_t tok_rows, int T, int d, int E,
                                    int K, int world, void *out, int32_t *status,
                                    cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int chunks = d / 8;
    ep_combine_dedup_kernel<<<grid_for((int64_t)T * chunks), 256, 0, st>>>(
        topk_idx, tok_slot, tok_base, reinterpret_cast<const uint4 *const *>(partial),
        static_cast<const uint4 *>(y_shared), tok_rows, T, chunks, E, K, E / world, world,
        static_cast<uint4 *>(out), status);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_ep_dispatch_dedup_fp8(const void *x, const int32_t *topk_idx,
                                         const int32_t *offsets, const int32_t *inv_perm,
                                         const int32_t *base, const int32_t *tok_slot,
                                         const int32_t *tok_base, void *const *recv_tq,
                                         void *const *recv_ts, int32_t *const *recv_idx,
                                         int64_t tok_rows, int64_t recv_rows, int T, int d, int E,
                                         int K, int world, int32_t *status, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int chunks = d / 8;
    ep_dispatch_dedup_fp8_kernel<<<grid_for((int64_t)T * chunks), 256, 0, st>>>(
        static_cast<const uint4 *>(x), topk_idx, offsets, inv_perm, base, tok_slot, tok_base,
        reinterpret_cast<uint2 *const *>(recv_tq), reinterpret_cast<float *const *>(recv_ts),
        recv_idx, tok_rows, recv_rows, T, chunks, E, K, E / world, world, status);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_ep_fanout_fp8(const void *recv_tq, const float *recv_ts,
                                 const int32_t *recv_idx, const int32_t *local_offsets, int El,
                                 int64_t tok_rows, int64_t recv_rows, int d, void *recv_q,
                                 float *recv_scale, int32_t *status, cudaStream_t st) {
    if (recv_rows == 0) return cudaSuccess;
    const int units = d / 16, blocks = d / 128;
    ep_fanout_fp8_kernel<<<grid_for(recv_rows * (units + blocks)), 256, 0, st>>>(
        static_cast<const uint4 *>(recv_tq), recv_ts, recv_idx, local_offsets, El, tok_rows,
        recv_rows, units, blocks, static_cast<uint4 *>(recv_q), recv_scale, status);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_ep_combine(const int32_t *topk_idx, const float *topk_w, const int32_t *offsets,
                              const int32_t *inv_perm, const int32_t *base,
                              const void *const *recv_y, int64_t recv_rows, const void *y_shared,
                              int T, int d, int E, int K, int world, void *out, int32_t *status,
                              cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int chunks = d / 8;
    ep_combine_kernel<<<grid_for((int64_t)T * chunks), 256, 0, st>>>(
        topk_idx, topk_w, offsets, inv_perm, base,
        reinterpret_cast<const uint4 *const *>(recv_y), recv_rows,
        static_cast<const uint4 *>(y_shared), T, chunks, E, K, E / world,
        static_cast<uint4 *>(out), status);
    count_launch();
    return cudaGetLastError();
}

}  // namespace moe
