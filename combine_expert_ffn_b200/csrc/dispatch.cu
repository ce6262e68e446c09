// dispatch.cu -- token copies -> expert-contiguous rows (stable counting sort).
//
// The dispatch all-to-all ("moe-node-limited-routing", "Why all to all
// dominates MoE step time") becomes a local permutation on one GPU: the T*K
// copies (t, j) are sorted by expert, tokens ascending inside each segment,
// with per-expert counts and offsets and the group-to-group send matrices
// ("send matrices", shivam2003 "5. Tail latency controls step time").
//
// Kernels, none using global atomics, so every output is deterministic:
//   count   : per 256-token block, a bitmask per expert (bit = token in the
//             block chose it) -> block histograms + partial send matrices
//   scan    : (more than 256 blocks only) warp per expert, prefix over blocks
//             -> counts, block bases; block 0 also sums the partial send
//             matrices.  Up to 256 blocks the scatter blocks do this themselves
//   scatter : per block, rank of a copy = popcount of the expert's mask below
//             its token; row = offsets[e] + base + rank -> perm, inv_perm;
//             offsets = exclusive scan of counts (recomputed per block)
//   gather  : x_perm[row] = x[t]: the copy engine moves whole rows (bulk
//             copies through shared memory), or, for rows wider than 14 KB,
//             16-byte thread copies reading each x row once

#include "fp8_payload.cuh"
#include "kernels.h"

namespace moe {

namespace {
constexpr int BLK = DISPATCH_BLOCK;       // tokens per block = threads per CTA
constexpr int WORDS = BLK / 32;           // mask words per expert

constexpr int KMAX = 32;                  // largest K (moe_check_config)

// Token t's K expert ids, all loads issued before any is used; -1 past K or T.
__device__ __forceinline__ void load_ids(const int32_t *__restrict__ topk_idx, int t, int T, int K,
                                         int (&ev)[KMAX]) {
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
        ev[j] = (t < T && j < K) ? __ldg(topk_idx + (size_t)t * K + j) : -1;
}

// Rebuilds the block's expert masks in smem: masks[e * WORDS + w] bit l set if
// token (block * BLK + 32 w + l) chose expert e (ev: this thread's token's ids).
// Flags bad ids and repeated experts of a token in `status`.
__device__ __forceinline__ void build_masks(const int (&ev)[KMAX], int T, int E, int K,
                                            uint32_t *masks, int32_t *status, bool flag_errors) {
    const int tid = threadIdx.x;
    for (int i = tid; i < E * WORDS; i += BLK) masks[i] = 0u;
    __syncthreads();
    const int t = blockIdx.x * BLK + tid;
    if (t < T) {
        const uint32_t bit = 1u << (tid & 31);
        const int w = tid >> 5;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j >= K) break;
            const int e = ev[j];
            if (e < 0 || e >= E) {
                if (flag_errors) record_status(status, MOE_ERR_DEVICE_FAULT);
                continue;
            }
            const uint32_t old = atomicOr(&masks[e * WORDS + w], bit);
            if ((old & bit) && flag_errors) record_status(status, MOE_ERR_DEVICE_FAULT);
        }
    }
    __syncthreads();
}
}  // namespace

__global__ void __launch_bounds__(BLK)
dispatch_count_kernel(const int32_t *__restrict__ topk_idx, int T, int E, int G, int K,
                      int32_t *__restrict__ hist_t, int32_t *__restrict__ send_part,
                      int32_t *__restrict__ sendtok_part, int32_t *status) {
    extern __shared__ uint32_t dsm[];
    uint32_t *masks = dsm;                                   // [E * WORDS]
    int32_t *send_s = reinterpret_cast<int32_t *>(dsm + E * WORDS);  // [G*G]
    int32_t *sendtok_s = send_s + G * G;                     // [G*G]
    const int tid = threadIdx.x, nblk = gridDim.x, blk = blockIdx.x;
    for (int i = tid; i < 2 * G * G; i += BLK) send_s[i] = 0;
    const int t = blk * BLK + tid;
    int ev[KMAX];
    load_ids(topk_idx, t, T, K, ev);
    build_masks(ev, T, E, K, masks, status, true);

    if (t < T) {
        const int gsz = E / G, src = t / (T / G);
        uint64_t hit = 0;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j >= K) break;
            const int e = ev[j];
            if (e < 0 || e >= E) continue;
            const int g = e / gsz;
            atomicAdd(&send_s[src * G + g], 1);
            hit |= 1ull << g;
        }
        while (hit) {
            const int g = __ffsll((long long)hit) - 1;
            hit &= hit - 1;
            atomicAdd(&sendtok_s[src * G + g], 1);
        }
    }
    for (int e = tid; e < E; e += BLK) {
        int c = 0;
#pragma unroll
        for (int w = 0; w < WORDS; ++w) c += __popc(masks[e * WORDS + w]);
        hist_t[(size_t)e * nblk + blk] = c;
    }
    __syncthreads();
    for (int i = tid; i < G * G; i += BLK) {
        send_part[(size_t)blk * G * G + i] = send_s[i];
        sendtok_part[(size_t)blk * G * G + i] = sendtok_s[i];
    }
}

// Warp per expert: exclusive prefix of hist_t[e, :] over the blocks.
__global__ void __launch_bounds__(256)
dispatch_scan_kernel(const int32_t *__restrict__ hist_t, int nblk, int E, int G,
                     const int32_t *__restrict__ send_part,
                     const int32_t *__restrict__ sendtok_part, int32_t *__restrict__ base_t,
                     int32_t *__restrict__ counts, int32_t *__restrict__ send,
                     int32_t *__restrict__ send_tok) {
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int e = blockIdx.x * 8 + warp;
    if (e < E) {
        const int32_t *h = hist_t + (size_t)e * nblk;
        int32_t *bo = base_t + (size_t)e * nblk;
        int carry = 0;
        for (int b0 = 0; b0 < nblk; b0 += 32) {
            const int b = b0 + lane;
            const int v = b < nblk ? h[b] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += n;
            }
            if (b < nblk) bo[b] = carry + incl - v;
            carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0) counts[e] = carry;
    }
    if (blockIdx.x == 0) {
        for (int i = threadIdx.x; i < G * G; i += blockDim.x) {
            int a = 0, c = 0;
            for (int b = 0; b < nblk; ++b) {
                a += send_part[(size_t)b * G * G + i];
                c += sendtok_part[(size_t)b * G * G + i];
            }
            send[i] = a;
            if (send_tok) send_tok[i] = c;
        }
    }
}

// With fused_scan (at most SCAN_FUSE_MAX_BLOCKS blocks) every block sums the
// block histograms hist_t itself -- counts[e] over all blocks, its base over
// the blocks before it -- and block 0 writes counts and the send matrices, so
// no separate scan launch is needed; otherwise counts and base_t come from
// dispatch_scan_kernel.
constexpr int SCAN_FUSE_MAX_BLOCKS = 256;

__global__ void __launch_bounds__(BLK)
dispatch_scatter_kernel(const int32_t *__restrict__ topk_idx, int T, int E, int G, int K,
                        int fused_scan, const int32_t *__restrict__ hist_t,
                        const int32_t *__restrict__ send_part,
                        const int32_t *__restrict__ sendtok_part, int32_t *__restrict__ counts,
                        const int32_t *__restrict__ base_t, int32_t *__restrict__ send,
                        int32_t *__restrict__ send_tok, int32_t *__restrict__ offsets,
                        int32_t *__restrict__ perm_token, int32_t *__restrict__ inv_perm) {
    extern __shared__ uint32_t dsm[];
    uint32_t *masks = dsm;                                          // [E * WORDS]
    int32_t *offs = reinterpret_cast<int32_t *>(dsm + E * WORDS);   // [E + 1]
    int32_t *wsum = offs + E + 1;                                   // [BLK / 32]
    int32_t *cnt_s = wsum + BLK / 32;                               // [E]
    int32_t *base_s = cnt_s + E;                                    // [E]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nblk = gridDim.x, blk = blockIdx.x;
    const int t = blk * BLK + tid;
    int ev[KMAX];  // issued first: their latency overlaps the histogram reads
    load_ids(topk_idx, t, T, K, ev);

    for (int e = tid; e < E; e += BLK) {
        int c, b;
        if (fused_scan) {
            const int32_t *h = hist_t + (size_t)e * nblk;
            c = 0;
            b = 0;
            // independent loads: unrolled so that many are in flight at once
#pragma unroll 16
            for (int q = 0; q < nblk; ++q) {
                const int v = h[q];
                c += v;
                if (q < blk) b += v;
            }
            if (blk == 0) counts[e] = c;
        } else {
            c = counts[e];
            b = base_t[(size_t)e * nblk + blk];
        }
        cnt_s[e] = c;
        base_s[e] = b;
    }
    if (fused_scan && blk == 0) {
        for (int i = tid; i < G * G; i += BLK) {
            int a = 0, c = 0;
#pragma unroll 16
            for (int q = 0; q < nblk; ++q) {
                a += send_part[(size_t)q * G * G + i];
                c += sendtok_part[(size_t)q * G * G + i];
            }
            send[i] = a;
            if (send_tok) send_tok[i] = c;
        }
    }
    __syncthreads();

    // offsets = exclusive scan of counts: each thread owns a run of experts
    const int per = (E + BLK - 1) / BLK;
    int run = 0;
    for (int i = 0; i < per; ++i) {
        const int e = tid * per + i;
        if (e < E) run += cnt_s[e];
    }
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) wsum[warp] = incl;
    build_masks(ev, T, E, K, masks, nullptr, false);  // contains __syncthreads
    int wpre = 0;
    for (int w = 0; w < warp; ++w) wpre += wsum[w];
    int acc = wpre + incl - run;
    for (int i = 0; i < per; ++i) {
        const int e = tid * per + i;
        if (e < E) {
            offs[e] = acc;
            acc += cnt_s[e];
        }
    }
    if (tid == BLK - 1) offs[E] = wpre + incl;
    __syncthreads();
    if (blk == 0)
        for (int e = tid; e <= E; e += BLK) offsets[e] = offs[e];

    if (t >= T) return;
    const int w = tid >> 5;
    const uint32_t below = (1u << lane) - 1u;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        if (j >= K) break;
        const int e = ev[j];
        if (e < 0 || e >= E) {
            inv_perm[(size_t)t * K + j] = -1;
            continue;
        }
        int rank = __popc(masks[e * WORDS + w] & below);
        for (int q = 0; q < w; ++q) rank += __popc(masks[e * WORDS + q]);
        const int row = offs[e] + base_s[e] + rank;
        perm_token[row] = t;
        inv_perm[(size_t)t * K + j] = row;
    }
}

// Thread per 16-byte chunk of a token row: one load, K stores.
__global__ void __launch_bounds__(256)
dispatch_gather_kernel(const uint4 *__restrict__ x, const int32_t *__restrict__ inv_perm, int T,
                       int chunks, int K, int64_t n_rows, uint4 *__restrict__ x_perm) {
    const int64_t total = (int64_t)T * chunks;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / chunks;
        const int c = (int)(i - t * chunks);
        const uint4 v = __ldg(x + i);
        for (int j = 0; j < K; ++j) {
            const int row = __ldg(inv_perm + t * K + j);
            if (row >= 0 && row < n_rows) x_perm[(int64_t)row * chunks + c] = v;
        }
    }
}

// Bulk-copy gather: the copy engine moves whole rows.  Each warp owns two row
// buffers in shared memory; lane 0 loads token t's row (cp.async.bulk, one
// mbarrier per buffer) while the previous row's stores drain, and lane j < K
// stores the row to x_perm[inv_perm[t][j]] (cp.async.bulk shared -> global).
// A buffer is reloaded only after every store that read it has read it.
constexpr int GB_WARPS = 4;

__device__ __forceinline__ void drain_wait_ns(uint32_t bar, uint32_t parity, int64_t timeout_ns) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity) && (int64_t)(globaltimer_ns() - t0) < timeout_ns) {
    }
}

__global__ void __launch_bounds__(GB_WARPS * 32)
dispatch_gather_bulk_kernel(const char *__restrict__ x, const int32_t *__restrict__ inv_perm,
                            int T, int row_bytes, int K, int64_t n_rows, char *__restrict__ x_perm,
                            int32_t *status, int64_t timeout_ns) {
    extern __shared__ __align__(128) uint8_t gsm[];
    __shared__ __align__(8) uint64_t lbar[GB_WARPS][2];
    __shared__ int abort_s[GB_WARPS];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t buf0 = smem_u32(gsm) + (uint32_t)(warp * 2 * row_bytes);
    const uint32_t bar0 = smem_u32(&lbar[warp][0]), bar1 = smem_u32(&lbar[warp][1]);
    if (lane == 0) {
        mbar_init(bar0, 1);
        mbar_init(bar1, 1);
        abort_s[warp] = 0;
        fence_barrier_init();
    }
    __syncwarp();
    const int nw = gridDim.x * GB_WARPS;
    int t = blockIdx.x * GB_WARPS + warp;
    uint32_t in_flight = 0;  // lane 0: bit b set while a load into buffer b is not waited for
    uint32_t ph = 0;         // bit b: phase parity of buffer b's barrier
    if (t < T && lane == 0) {
        mbar_arrive_expect_tx(bar0, row_bytes);
        bulk_load(buf0, x + (size_t)t * row_bytes, row_bytes, bar0);
        in_flight = 1u;
    }
    for (int i = 0; t < T; t += nw, ++i) {
        const int b = i & 1;
        const int tn = t + nw;
        const int row = lane < K ? __ldg(inv_perm + (size_t)t * K + lane) : -1;
        // the other buffer: every store of the previous row has read it
        if (lane < K) bulk_wait_group_read<0>();
        __syncwarp();
        if (lane == 0 && tn < T) {
            const uint32_t nb = b ? bar0 : bar1;
            mbar_arrive_expect_tx(nb, row_bytes);
            bulk_load(buf0 + (uint32_t)((b ^ 1) * row_bytes), x + (size_t)tn * row_bytes, row_bytes,
                      nb);
            in_flight |= 1u << (b ^ 1);
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
        // the storing lanes observe the completed phase themselves (it has completed:
        // one probe suffices) before their copies read the buffer
        if (lane < K) mbar_try_wait(bar, par);
        if (lane < K) {
            if (row >= 0 && row < n_rows)
                bulk_store(x_perm + (size_t)row * row_bytes, buf0 + (uint32_t)(b * row_bytes),
                           row_bytes);
            bulk_commit_group();
        }
    }
    bulk_wait_group_all();
    // after a timeout: wait (bounded) for loads still in flight into this warp's buffers
    if (lane == 0) {
        if (in_flight & 1u) drain_wait_ns(bar0, ph & 1u, timeout_ns);
        if (in_flight & 2u) drain_wait_ns(bar1, (ph >> 1) & 1u, timeout_ns);
    }
}

// FP8 payload gather.  One 16-lane group per (token, 128-channel block);
// lane l of the group holds channels 8l .. 8l+7.  s = amax / 448 in fp32,
// q = E4M3(x / s) (fp32 division, nearest-even, saturating), all-zero blocks
// give s = 0 and q = 0.  Each token's codes and scales are written to its K
// permuted rows.
__global__ void __launch_bounds__(256)
dispatch_gather_fp8_kernel(const uint4 *__restrict__ x, const int32_t *__restrict__ inv_perm,
                           int T, int chunks, int K, int64_t n_rows, uint2 *__restrict__ xq,
                           float *__restrict__ xs) {
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
            const int row = __ldg(inv_perm + t * K + j);
            if (row < 0 || row >= n_rows) continue;
            xq[(int64_t)row * chunks + c] = packed;
            if ((c & 15) == 0) xs[(int64_t)row * (chunks >> 4) + (c >> 4)] = sc;
        }
    }
}

cudaError_t launch_gather_fp8(const void *x, const int32_t *inv_perm, int T, int d, int K,
                              uint8_t *x_perm_q, float *x_scale, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int chunks = d / 8;
    const int64_t total = (int64_t)T * chunks;
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (total + 255) / 256;
    const int grid = (int)(want < (int64_t)sms * 16 ? want : (int64_t)sms * 16);
    dispatch_gather_fp8_kernel<<<grid, 256, 0, st>>>(static_cast<const uint4 *>(x), inv_perm, T,
                                                     chunks, K, (int64_t)T * K,
                                                     reinterpret_cast<uint2 *>(x_perm_q), x_scale);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_permute(const void *x, const int32_t *inv_perm, int T, int d, int K,
                           void *x_perm, cudaStream_t st, int32_t *status, int64_t timeout_ns) {
    if (T == 0) return cudaSuccess;
    const int row_bytes = d * 2;
    const size_t gb_smem = (size_t)GB_WARPS * 2 * row_bytes;
    if (K <= 32 && gb_smem <= 112 * 1024) {
        // one wave of four-warp CTAs (two per SM at 14 KB rows); every warp walks
        // about T / (warps resident) rows
        int sms = 148, dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess)
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaError_t err = cudaFuncSetAttribute(dispatch_gather_bulk_kernel,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)gb_smem);
        if (err != cudaSuccess) return err;
        int per_sm = 1;  // CTAs resident per SM with this shared memory (one wave)
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dispatch_gather_bulk_kernel,
                                                          GB_WARPS * 32, gb_smem) != cudaSuccess ||
            per_sm < 1)
            per_sm = 1;
        const int want = (T + GB_WARPS - 1) / GB_WARPS;
        const int grid = want < per_sm * sms ? want : per_sm * sms;
        dispatch_gather_bulk_kernel<<<grid, GB_WARPS * 32, gb_smem, st>>>(
            static_cast<const char *>(x), inv_perm, T, row_bytes, K, (int64_t)T * K,
            static_cast<char *>(x_perm), status, timeout_ns);
        count_launch();
        return cudaGetLastError();
    }
    const int chunks = d / 8;
    const int64_t total = (int64_t)T * chunks;
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (total + 255) / 256;
    const int grid = (int)(want < (int64_t)sms * 16 ? want : (int64_t)sms * 16);
    dispatch_gather_kernel<<<grid, 256, 0, st>>>(static_cast<const uint4 *>(x), inv_perm, T, chunks,
                                                 K, (int64_t)T * K, static_cast<uint4 *>(x_perm));
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_dispatch(const void *x, const int32_t *topk_idx, int T, int d, int E, int G,
                            int K, int32_t *counts, int32_t *offsets, int32_t *send,
                            int32_t *send_tok, int32_t *perm_token, int32_t *inv_perm,
                            void *x_perm, const DispatchWs &ws, int32_t *status, cudaStream_t st) {
    const int nblk = dispatch_nblk(T);
    cudaError_t err;
    if (T == 0) {
        // no copies: zero the outputs that still have entries
        if ((err = cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, st))) return err;
        if ((err = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), st))) return err;
        if ((err = cudaMemsetAsync(send, 0, sizeof(int32_t) * G * G, st))) return err;
        if (send_tok && (err = cudaMemsetAsync(send_tok, 0, sizeof(int32_t) * G * G, st))) return err;
        return cudaSuccess;
    }
    const size_t smem_count = sizeof(uint32_t) * (E * WORDS + 2 * G * G);
    const size_t smem_scatter = sizeof(uint32_t) * (E * WORDS + E + 1 + BLK / 32 + 2 * E);
    if (smem_count > 48 * 1024 &&
        (err = cudaFuncSetAttribute(dispatch_count_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_count)))
        return err;
    if (smem_scatter > 48 * 1024 &&
        (err = cudaFuncSetAttribute(dispatch_scatter_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_scatter)))
        return err;
    dispatch_count_kernel<<<nblk, BLK, smem_count, st>>>(topk_idx, T, E, G, K, ws.hist_t,
                                                         ws.send_part, ws.sendtok_part, status);
    count_launch();
    if ((err = cudaGetLastError())) return err;
    const int fused_scan = nblk <= SCAN_FUSE_MAX_BLOCKS;
    if (!fused_scan) {
        dispatch_scan_kernel<<<(E + 7) / 8, 256, 0, st>>>(ws.hist_t, nblk, E, G, ws.send_part,
                                                          ws.sendtok_part, ws.base_t, counts, send,
                                                          send_tok);
        count_launch();
        if ((err = cudaGetLastError())) return err;
    }
    dispatch_scatter_kernel<<<nblk, BLK, smem_scatter, st>>>(
        topk_idx, T, E, G, K, fused_scan, ws.hist_t, ws.send_part, ws.sendtok_part, counts,
        ws.base_t, send, send_tok, offsets, perm_token, inv_perm);
    count_launch();
    if ((err = cudaGetLastError())) return err;
    if (x_perm) return launch_permute(x, inv_perm, T, d, K, x_perm, st, status);
    return cudaSuccess;
}

}  // namespace moe
