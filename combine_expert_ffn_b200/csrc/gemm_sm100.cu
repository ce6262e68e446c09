// gemm_sm100.cu -- grouped expert FFN on the 5th-generation tensor cores.
//
// Per routed expert e with rows R_e = [offsets[e], offsets[e+1]) of x_perm
// and for the shared experts on all T rows of x:
//   GEMM1:  h = SiLU(X W_g^T) * (X W_u^T)     (SwiGLU fused in the epilogue)
//   GEMM2:  y = h W_d^T
// ("shared experts (always active) + fine-grained routed experts", "MoE +
// Expert-Parallel Overlap (Exp08)", Implemented; the pages' per token-expert
// cost is 6 d d_ff FLOPs, same page, Implemented / overlap simulator.)
//
// One persistent kernel per GEMM, one CTA per SM, 192 threads:
//   warp 0      TMA producer: A tile 128 x 64 and B tile 256 x 64 (bf16,
//               128-byte swizzle) per stage into a 4-stage smem ring
//   warp 1      TMEM owner (512 columns = two 128 x 256 fp32 accumulators)
//               and single-thread tcgen05.mma issuer (M=128, N=256, K=16)
//   warps 2..5  epilogue: tcgen05.ld -> SwiGLU or plain -> bf16 -> global
// GEMM1 has two more A-operand variants with extra warps: rows gathered from
// x (x[perm_token[r]], 4 warps of 16-byte cp.async copies) and the FP8
// payload widened to bf16 in shared memory (2 groups of 4 converter warps).
// The accumulator is double-buffered so the epilogue of tile i overlaps the
// mainloop of tile i+1.  (Token rows on the MMA's M side and weight rows on N:
// measured on B200, weights-stationary tiles with tokens on N -- 1-CTA or CTA
// pair -- lost 20-45% to TMA issue throughput despite doing less MMA work.)
// Tiles: for every expert, ceil(R_e/128) row tiles x
// the output column tiles; row tiles of one expert are adjacent in the tile
// order so the expert's weight tiles are read from HBM about once and served
// from L2 to its other row tiles.  Row tiles may run past the segment end
// into the next expert's rows (or past the buffer, where TMA fills zeros):
// those rows are computed and never stored.  Every wait is bounded; on
// running out the kernel records MOE_ERR_DEVICE_TIMEOUT, drains its own TMA
// loads and MMAs, frees TMEM and returns.
#include <cstring>

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "kernels.h"


// Paired row tiles (grouped_ffn_pair_kernel) for the gate/up GEMM and the
// down GEMM; 0 selects the single-tile kernel with double-buffered TMEM.  The
// gate/up GEMM also takes the paired kernel when the experts average at least
// MOE_PAIR_MIN_ROWS rows (most row tiles then come in pairs; measured on the
// skewed V3 workload, 1024 rows per expert on average: 21.4 vs 22.6 ms for the
// expert FFN, while at 256 rows per expert the single-tile kernel is faster).
#ifndef MOE_PAIR_GEMM1
#define MOE_PAIR_GEMM1 0
#endif
#ifndef MOE_PAIR_MIN_ROWS
#define MOE_PAIR_MIN_ROWS 512
#endif
#ifndef MOE_PAIR_GEMM2
#define MOE_PAIR_GEMM2 0
#endif

#ifndef MOE_GEMM_KB_GROUP
#define MOE_GEMM_KB_GROUP 1
#endif

// One-CTA kernel: a tile with at most 64 valid rows issues M = 64 MMAs (1 on,
// 0 off).  Its accumulator rows then sit in TMEM lanes (i % 16) + 32 (i / 16).
#ifndef MOE_GEMM_TAIL64
#define MOE_GEMM_TAIL64 1
#endif

// CTA-pair grouped GEMMs (tcgen05.mma.cta_group::2, packed weights only):
// 0 never (default), 1 always when the weights are packed.  Bit-identical to
// the one-CTA kernel, but not faster: measured +17 % at the V3 routing (256-row
// pair tiles pad 19 % more rows than 128-row tiles), +5 % at mid, +1 % at the
// skewed routing (no padding), +50 % for decode (half as many weight streams).
#ifndef MOE_GEMM_CTA2
#define MOE_GEMM_CTA2 0
#endif

namespace moe {
namespace gemm {

constexpr int KB_GROUP = MOE_GEMM_KB_GROUP;
constexpr int BM = 128;
constexpr int BK = 64;
constexpr int BN_ACC = 256;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN_ACC * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_THREADS = 192;
// Variants of GEMM1's routed A operand: TMA tiles of x_perm; rows gathered
// from x by four extra warps (16-byte cp.async copies); or the FP8 payload,
// TMA-loaded as bytes and widened to bf16 in place by converter warps.
enum { A_TMA = 0, A_GATHER = 1, A_FP8 = 2 };
constexpr int GATHER_WARPS = 4;
constexpr int GATHER_THREADS = GATHER_WARPS * 32;
// The FP8 variant runs two such groups of converter warps on alternate stages,
// so that one group's barriers and widening overlap the other's.
constexpr int CONV_GROUPS = 2;
template <int AMODE>
constexpr int extra_threads() {
    return AMODE == A_FP8 ? CONV_GROUPS * GATHER_THREADS : AMODE == A_GATHER ? GATHER_THREADS : 0;
}
constexpr int FP8_STAGE_OFF = A_BYTES / 2;  // FP8 bytes land in the upper half of the A stage
constexpr int TMEM_COLS = 512;
constexpr int MAX_E = 1024;
constexpr int STORE_BUF = 32 * 32 * 2;     // one warp's 32 rows x 32 columns of bf16
constexpr int SMEM_DYN = STAGES * STAGE_BYTES + 4 * 2 * STORE_BUF + 1024;

enum { EPI_SWIGLU = 0, EPI_STORE = 1 };

template <int EPI>
struct Cfg {
    static constexpr int BN_OUT = EPI == EPI_STORE ? 256 : 128;    // output columns per tile
    static constexpr int BN_MMA = 256;                              // MMA N
    static constexpr uint32_t TX = A_BYTES + BN_MMA * BK * 2;      // bytes per stage
};

struct Maps {
    CUtensorMap a_r;   // routed A  [rows_r, k_r]           box 64 x 128
    CUtensorMap a_s;   // shared A  [T, k_s]                box 64 x 128
    CUtensorMap b0_r;  // routed B  gate | down  3-D        box 64 x (128 | 256) x 1
    CUtensorMap b1_r;  // routed B  up (SwiGLU only)
    CUtensorMap b0_s;  // shared B  gate | down
    CUtensorMap b1_s;  // shared B  up
    CUtensorMap o_r;   // routed output [rows_r, n_out_r]    box 32 x 32, for full tiles
    CUtensorMap o_s;   // shared output [T, n_out_s]         box 32 x 32
    CUtensorMap a_q;   // routed FP8 payload [rows_r, k_r] bytes, box 64 x 128 (A_FP8)
    CUtensorMap bpk;   // CTA-pair kernel: the packed weights as rows of 128 bytes, box 64 x 128
};

struct Params {
    const int32_t *offsets;  // [E+1]
    const int32_t *perm_token;  // gather variant: routed row r of A is x[perm_token[r]]
    const void *x;           // gather variant: x [x_rows, k_r] bf16
    int x_rows;
    const float *x_scale;    // FP8 variant: [rows_r, k_r / 128] payload scales
    int E;
    int rows_r;              // rows of the routed A buffer (T*K)
    int T;                   // shared rows; 0 = no shared experts
    int n_out_r, n_out_s;    // output columns
    int k_r, k_s;            // reduction lengths
    int kseg_s;              // shared B is split along k into experts of this width
    __nv_bfloat16 *out_r;
    __nv_bfloat16 *out_s;
    int32_t *status;
    int64_t timeout_ns;
    int *tile_counter;       // paired kernel: next tile to hand out (zero at launch)
    // packed weights (pack.cu): the B tile (e, n, kb) is the 32 KB block
    // ((e * bp_nt_r + n) * k_r/64 + kb) of bp_r (routed) and (n * k_s/64 + kb) of
    // bp_s (shared); null: tensor-map loads of the row-major weights
    const uint8_t *bp_r, *bp_s;
    int bp_nt_r;
    // CTA-pair kernel: first 128-byte row of bp_r / bp_s in the map bpk
    int64_t bpk_row_r, bpk_row_s;
};

// The B tile of (tile, k block kb) from the packed weights: one 32 KB bulk copy.
template <int EPI>
__device__ __forceinline__ void load_packed_b(const Params &p, int e, int n0, int kb,
                                              uint32_t dst, uint32_t bar) {
    const int n = n0 / Cfg<EPI>::BN_OUT;
    const uint8_t *src = e >= 0
        ? p.bp_r + ((((size_t)e * p.bp_nt_r + n) * (p.k_r / BK) + kb) << 15)
        : p.bp_s + ((((size_t)n) * (p.k_s / BK) + kb) << 15);
    bulk_load(dst, src, 32768, bar);
}

struct Tile {
    int row0;        // first A row
    int rows_valid;  // rows to store
    int n0;          // first output column
    int e;           // expert (routed) or -1 (shared)
    int kblocks;
};

template <int EPI>
__device__ __forceinline__ Tile decode_tile(int idx, const int *tile_base, const int *seg,
                                            const int *segc, const Params &p, int ntr, int mt_s,
                                            int nt_s) {
    constexpr int BN_OUT = Cfg<EPI>::BN_OUT;
    Tile t;
    if (idx < ntr) {
        int lo = 0, hi = p.E;  // tile_base[lo] <= idx < tile_base[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (tile_base[mid] <= idx) lo = mid; else hi = mid;
        }
        const int cnt = segc[lo];
        const int mt = (cnt + BM - 1) / BM;
        const int local = idx - tile_base[lo];
        const int n = local / mt, m = local - n * mt;
        t.row0 = seg[lo] + m * BM;
        t.rows_valid = min(BM, cnt - m * BM);
        t.n0 = n * BN_OUT;
        t.e = lo;
        t.kblocks = p.k_r / BK;
    } else {
        const int local = idx - ntr;
        const int m = local / nt_s, n = local - m * nt_s;  // column tiles fastest
        t.row0 = m * BM;
        t.rows_valid = min(BM, p.T - m * BM);
        t.n0 = n * BN_OUT;
        t.e = -1;
        t.kblocks = p.k_s / BK;
    }
    return t;
}

// Bounded wait used while winding down: ignores the abort flag, so that
// copies and MMAs already in flight are waited for before the CTA exits.
__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity, int64_t timeout_ns,
                                           int32_t *status) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if ((int64_t)(globaltimer_ns() - t0) > timeout_ns) {
            record_status(status, MOE_ERR_DEVICE_TIMEOUT);
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ float silu_mul(float g, float u) {
    return g * __frcp_rn(1.0f + __expf(-g)) * u;
}

// Named barrier of converter group grp (ids 1 and 2; 0 is __syncthreads).
__device__ __forceinline__ void converters_sync(int grp) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "n"(GATHER_THREADS) : "memory");
}

template <int EPI, int AMODE>
__global__ void __launch_bounds__(NUM_THREADS + extra_threads<AMODE>(), 1)
grouped_ffn_gemm_kernel(const __grid_constant__ Maps maps, const Params p) {
    static_assert(AMODE == A_TMA || EPI == EPI_SWIGLU, "only GEMM1 has A-operand variants");
    constexpr bool GATHER = AMODE == A_GATHER;
    constexpr bool EXTRA = AMODE != A_TMA;  // extra warps write A stages
    constexpr int BN_OUT = Cfg<EPI>::BN_OUT;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[STAGES];
    __shared__ __align__(8) uint64_t empty_bar[STAGES];
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];
    __shared__ __align__(8) uint64_t done_bar;
    __shared__ __align__(8) uint64_t qfull_bar[STAGES];  // A_FP8: payload bytes of a stage landed
    __shared__ int conv_ok_s[CONV_GROUPS];
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    __shared__ int tile_base[MAX_E + 1];
    __shared__ int seg[MAX_E];
    __shared__ int segc[MAX_E];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t smem0 = smem_u32(smem);
    volatile int *abort_flag = &abort_s;

    // ---------------------------------------------------------- prologue
    if (warp == 0) {
        // tile_base[e] = sum over experts < e of (row tiles x column tiles)
        const int nt_r = (p.n_out_r + BN_OUT - 1) / BN_OUT;
        int carry = 0;
        for (int e0 = 0; e0 < p.E; e0 += 32) {
            const int e = e0 + lane;
            int lo = 0, cnt = 0;
            if (e < p.E) {
                lo = p.offsets[e];
                cnt = p.offsets[e + 1] - lo;
                // a segment outside [0, rows_r] or of negative length is
                // treated as empty and reported
                if (lo < 0 || cnt < 0 || lo + cnt > p.rows_r) {
                    record_status(p.status, MOE_ERR_DEVICE_FAULT);
                    lo = 0;
                    cnt = 0;
                }
                seg[e] = lo;
                segc[e] = cnt;
            }
            const int v = ((cnt + BM - 1) / BM) * nt_r;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += n;
            }
            if (e < p.E) tile_base[e] = carry + incl - v;
            carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0) {
            tile_base[p.E] = carry;
            tma_prefetch_desc(&maps.o_r);
            if (AMODE == A_TMA) tma_prefetch_desc(&maps.a_r);
            if (AMODE == A_FP8) tma_prefetch_desc(&maps.a_q);
            if (!p.bp_r) {
                tma_prefetch_desc(&maps.b0_r);
                if (EPI == EPI_SWIGLU) tma_prefetch_desc(&maps.b1_r);
            }
            if (p.T > 0) {
                tma_prefetch_desc(&maps.a_s);
                if (!p.bp_s) {
                    tma_prefetch_desc(&maps.b0_s);
                    if (EPI == EPI_SWIGLU) tma_prefetch_desc(&maps.b1_s);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            for (int s = 0; s < STAGES; ++s) {
                mbar_init(smem_u32(&full_bar[s]), 1 + (EXTRA ? GATHER_THREADS : 0));
                mbar_init(smem_u32(&qfull_bar[s]), 1);
                mbar_init(smem_u32(&empty_bar[s]), 1);
            }
            for (int b = 0; b < 2; ++b) {
                mbar_init(smem_u32(&tfull_bar[b]), 1);
                mbar_init(smem_u32(&tempty_bar[b]), 128);
            }
            mbar_init(smem_u32(&done_bar), 1);
            abort_s = 0;
            fence_barrier_init();
        }
        __syncwarp();
        tmem_alloc<TMEM_COLS>(smem_u32(&tmem_base_s));
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_s;

    const int ntr = tile_base[p.E];
    const int mt_s = p.T > 0 ? (p.T + BM - 1) / BM : 0;
    const int nt_s = p.T > 0 ? (p.n_out_s + BN_OUT - 1) / BN_OUT : 0;
    const int total = ntr + mt_s * nt_s;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        // B tiles, and A tiles except the routed ones of the gather variant
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t n_issued = 0;
            for (int idx = blockIdx.x; idx < total; idx += gridDim.x) {
                const Tile t = decode_tile<EPI>(idx, tile_base, seg, segc, p, ntr, mt_s, nt_s);
                const bool a_by_tma = AMODE == A_TMA || t.e < 0;
                bool ok = true;
                for (int kb = 0; kb < t.kblocks; ++kb) {
                    // KB_GROUP > 1: wait until the next KB_GROUP stages are free, so that
                    // the copies of adjacent k blocks (adjacent bytes of the same rows)
                    // are requested together
                    if (KB_GROUP > 1 && kb % KB_GROUP == 0) {
                        int st2 = stage;
                        uint32_t ph2 = phase;
                        for (int g = 0; g < KB_GROUP && kb + g < t.kblocks && ok; ++g) {
                            if (!mbar_wait_bounded(smem_u32(&empty_bar[st2]), ph2 ^ 1u, abort_flag,
                                                   p.status, p.timeout_ns))
                                ok = false;
                            if (++st2 == STAGES) { st2 = 0; ph2 ^= 1u; }
                        }
                        if (!ok) break;
                    }
                    if (!mbar_wait_bounded(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag,
                                           p.status, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full_bar[stage]);
                    const uint32_t a_dst = smem0 + stage * STAGE_BYTES;
                    const uint32_t b_dst = a_dst + A_BYTES;
                    const int k = kb * BK;
                    mbar_arrive_expect_tx(fb, a_by_tma ? Cfg<EPI>::TX : Cfg<EPI>::TX - A_BYTES);
                    if (AMODE == A_FP8) {  // converters wait for this barrier every stage
                        const uint32_t qb = smem_u32(&qfull_bar[stage]);
                        if (a_by_tma) {
                            mbar_arrive(qb);
                        } else {
                            mbar_arrive_expect_tx(qb, A_BYTES / 2);
                            tma_load_2d(a_dst + FP8_STAGE_OFF, &maps.a_q, qb, k, t.row0);
                        }
                    }
                    if (t.e >= 0) {
                        if (a_by_tma) tma_load_2d(a_dst, &maps.a_r, fb, k, t.row0);
                        if (p.bp_r) {
                            load_packed_b<EPI>(p, t.e, t.n0, kb, b_dst, fb);
                        } else if (EPI == EPI_SWIGLU) {
                            tma_load_3d(b_dst, &maps.b0_r, fb, k, t.n0, t.e);
                            tma_load_3d(b_dst + BN_ACC / 2 * BK * 2, &maps.b1_r, fb, k, t.n0, t.e);
                        } else {
                            tma_load_3d(b_dst, &maps.b0_r, fb, k, t.n0, t.e);
                        }
                    } else {
                        tma_load_2d(a_dst, &maps.a_s, fb, k, t.row0);
                        if (p.bp_s) {
                            load_packed_b<EPI>(p, -1, t.n0, kb, b_dst, fb);
                        } else if (EPI == EPI_SWIGLU) {
                            tma_load_3d(b_dst, &maps.b0_s, fb, k, t.n0, 0);
                            tma_load_3d(b_dst + BN_ACC / 2 * BK * 2, &maps.b1_s, fb, k, t.n0, 0);
                        } else {
                            const int s = k / p.kseg_s;
                            tma_load_3d(b_dst, &maps.b0_s, fb, k - s * p.kseg_s, t.n0, s);
                        }
                    }
                    ++n_issued;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
            }
            // wind down: every load issued into a stage has landed
            for (int s = 0; s < STAGES; ++s) {
                if (n_issued > (uint32_t)s) {
                    const uint32_t uses = (n_issued - 1 - s) / STAGES + 1;
                    drain_wait(smem_u32(&full_bar[s]), (uses - 1) & 1u, p.timeout_ns, p.status);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int idx = blockIdx.x; idx < total; idx += gridDim.x) {
                const Tile t = decode_tile<EPI>(idx, tile_base, seg, segc, p, ntr, mt_s, nt_s);
                if (!mbar_wait_bounded(smem_u32(&tempty_bar[acc]), acc_phase ^ 1u, abort_flag,
                                       p.status, p.timeout_ns))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN_ACC;
                // a tail tile of at most 64 rows: M = 64 MMAs over the first 64 A rows
                const uint32_t idesc = MOE_GEMM_TAIL64 && t.rows_valid <= BM / 2
                                           ? idesc_bf16_f32<BM / 2, Cfg<EPI>::BN_MMA>()
                                           : idesc_bf16_f32<BM, Cfg<EPI>::BN_MMA>();
                bool ok = true;
                for (int kb = 0; kb < t.kblocks; ++kb) {
                    if (!mbar_wait_bounded(smem_u32(&full_bar[stage]), phase, abort_flag, p.status,
                                           p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (EXTRA) fence_proxy_async();  // A rows written through the generic proxy
                    const uint32_t a_addr = smem0 + stage * STAGE_BYTES;
                    const uint64_t a_desc = smem_desc_sw128(a_addr);
                    const uint64_t b_desc = smem_desc_sw128(a_addr + A_BYTES);
#pragma unroll
                    for (int ks = 0; ks < BK / 16; ++ks)
                        tc_mma_bf16(d_tmem, a_desc + 2 * ks, b_desc + 2 * ks, idesc,
                                    (kb | ks) != 0 ? 1u : 0u);
                    tc_commit(smem_u32(&empty_bar[stage]));
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit(smem_u32(&tfull_bar[acc]));
                if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
            }
            // wind down: every MMA issued has completed
            tc_commit(smem_u32(&done_bar));
            drain_wait(smem_u32(&done_bar), 0, p.timeout_ns, p.status);
        }
        __syncwarp();
    } else if (AMODE == A_FP8 && warp >= NUM_THREADS / 32) {
        // ------------------------------------------------------ FP8 converters
        // Two groups of four warps take alternate stages.  In its stages,
        // thread g of a group widens the 8-byte chunk c = g % 8 of the rows
        // g / 8 + 16 j (j < 8): x_hat = bf16(E4M3^-1(q) * s), s the row's scale
        // of the 128-channel block, into the 128-byte-swizzled bf16 stage.  The
        // payload sits in the upper half of that stage, so every converter of
        // the group reads its bytes before any writes (named barrier).  Thread 0
        // of the group alone waits (bounded) for the payload and shares the
        // outcome.
        const int grp = (warp - NUM_THREADS / 32) / GATHER_WARPS;
        const int g = threadIdx.x - NUM_THREADS - grp * GATHER_THREADS;
        const int c = g & 7, r0 = g >> 3;
        const int nsb = p.k_r / 128;  // scales per row
        int stage = 0;
        uint32_t phase = 0, n_use = 0;
        bool ok = true;
        for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
            const Tile t = decode_tile<EPI>(idx, tile_base, seg, segc, p, ntr, mt_s, nt_s);
            const bool conv = t.e >= 0;
            float s_cur[8], s_next[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int r = r0 + 16 * j;
                s_cur[j] = 0.f;
                s_next[j] = conv && r < t.rows_valid ? p.x_scale[(size_t)(t.row0 + r) * nsb] : 0.f;
            }
            for (int kb = 0; kb < t.kblocks; ++kb, ++n_use) {
                if ((int)(n_use % CONV_GROUPS) != grp) {  // the other group's stage
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                    continue;
                }
                if (conv) {  // this group's stages step one 128-channel block each
                    const int nb = kb / 2 + 1;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int r = r0 + 16 * j;
                        s_cur[j] = s_next[j];
                        s_next[j] = nb < nsb && r < t.rows_valid
                                        ? p.x_scale[(size_t)(t.row0 + r) * nsb + nb] : 0.f;
                    }
                }
                if (g == 0)
                    conv_ok_s[grp] = mbar_wait_bounded(smem_u32(&qfull_bar[stage]), phase,
                                                       abort_flag, p.status, p.timeout_ns);
                converters_sync(grp);
                ok = *reinterpret_cast<volatile int *>(&conv_ok_s[grp]) != 0;
                if (!ok) break;  // every converter of the group read the same flag
                uint8_t *st = smem + stage * STAGE_BYTES;
                uint2 raw[8];
                if (conv) {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        raw[j] = *reinterpret_cast<const uint2 *>(st + FP8_STAGE_OFF +
                                                                  (r0 + 16 * j) * 64 + c * 8);
                }
                // every payload byte is in registers, and every converter of the
                // group has read the flag before thread 0 may write the next one
                converters_sync(grp);
                if (conv) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int r = r0 + 16 * j;
                        const uint32_t w2[2] = {raw[j].x, raw[j].y};
                        uint32_t o[4];
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
                                (__nv_fp8x2_storage_t)(w2[h >> 1] >> (16 * (h & 1))), __NV_E4M3);
                            const float2 f = __half22float2(__half2(hr));
                            o[h] = pack_bf16x2(__fmul_rn(f.x, s_cur[j]), __fmul_rn(f.y, s_cur[j]));
                        }
                        *reinterpret_cast<uint4 *>(st + r * (BK * 2) + ((c ^ (r & 7)) << 4)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                    fence_proxy_async();
                }
                mbar_arrive(smem_u32(&full_bar[stage]));
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
        }
    } else if (GATHER && warp >= NUM_THREADS / 32) {
        // ------------------------------------------------------ A-row gatherers
        // Thread g copies the 16-byte chunk c = g % 8 of the rows g / 8 + 16 j
        // (j < 8) of every routed A stage: x[perm_token[row0 + r]][k + 8c ..]
        // lands at r * 128 + ((c ^ (r % 8)) * 16), the 128-byte swizzle a TMA
        // tile load would produce.  Every stage -- copied or not -- gets one
        // arrival per gatherer on its full barrier, made by the copy hardware
        // once the thread's copies have landed; the MMA thread fences the
        // generic-proxy writes for the tensor core after its wait.
        const int g = threadIdx.x - NUM_THREADS;
        const int c = g & 7, r0 = g >> 3;
        const __nv_bfloat16 *xg = static_cast<const __nv_bfloat16 *>(p.x);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
            const Tile t = decode_tile<EPI>(idx, tile_base, seg, segc, p, ntr, mt_s, nt_s);
            const bool copy = t.e >= 0;
            const __nv_bfloat16 *src[8];
            if (copy) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int r = r0 + 16 * j;
                    int tok = 0;  // rows past the segment (never stored) read row 0
                    if (r < t.rows_valid) {
                        tok = p.perm_token[t.row0 + r];
                        if (tok < 0 || tok >= p.x_rows) {
                            record_status(p.status, MOE_ERR_DEVICE_FAULT);
                            tok = 0;
                        }
                    }
                    src[j] = xg + (size_t)tok * p.k_r + 8 * c;
                }
            }
            for (int kb = 0; kb < t.kblocks; ++kb) {
                if (!mbar_wait_bounded(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag,
                                       p.status, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                if (copy) {
                    const uint32_t a_dst = smem0 + stage * STAGE_BYTES;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int r = r0 + 16 * j;
                        cp_async_16(a_dst + r * (BK * 2) + ((c ^ (r & 7)) << 4), src[j] + kb * BK);
                    }
                }
                cp_async_arrive_noinc(smem_u32(&full_bar[stage]));
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
        }
        cp_async_wait_all();  // no copy into this CTA's stages outlives the thread
    } else {
        // ------------------------------------------------------ epilogue
        // A full tile (128 valid rows) leaves through TMA stores: each warp
        // stages its 32 rows x 32 columns (64-byte rows) in shared memory and
        // one lane stores the box, so global writes are whole 64-byte row
        // pieces.  Rows of a partial tile that belong to the next expert must
        // not be written, so partial tiles use masked direct stores.
        const int q = warp & 3;            // TMEM lane quarter this warp may access
        const uint32_t stage_buf0 = smem0 + STAGES * STAGE_BYTES + (warp - 2) * 2 * STORE_BUF;
        int sb = 0;                        // staging buffer toggle
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int idx = blockIdx.x; idx < total; idx += gridDim.x) {
            const Tile t = decode_tile<EPI>(idx, tile_base, seg, segc, p, ntr, mt_s, nt_s);
            if (!mbar_wait_bounded(smem_u32(&tfull_bar[acc]), acc_phase, abort_flag, p.status,
                                   p.timeout_ns))
                break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN_ACC;
            // accumulator row of this lane: lane of quarter q for M = 128; for an
            // M = 64 tail tile lanes 0..15 of the quarter hold rows 16 q .. 16 q + 15
            const bool m64 = MOE_GEMM_TAIL64 && t.rows_valid <= BM / 2;
            const int row = m64 ? q * 16 + (lane & 15) : q * 32 + lane;
            const bool shared = t.e < 0;
            const int n_out = shared ? p.n_out_s : p.n_out_r;
            __nv_bfloat16 *orow = (shared ? p.out_s : p.out_r) + (size_t)(t.row0 + row) * n_out;
            const CUtensorMap *omap = shared ? &maps.o_s : &maps.o_r;
            const bool full = t.rows_valid == BM;
            const bool row_ok = (!m64 || lane < 16) && row < t.rows_valid;
#pragma unroll 1
            for (int c = 0; c < BN_OUT; c += 32) {
                uint4 o[4];
                if (EPI == EPI_SWIGLU) {
                    uint32_t g[32], u[32];
                    tmem_ld32(taddr + c, g);
                    tmem_ld32(taddr + BN_ACC / 2 + c, u);
                    tc_wait_ld();
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        o[v].x = pack_bf16x2(silu_mul(__uint_as_float(g[8 * v + 0]), __uint_as_float(u[8 * v + 0])),
                                             silu_mul(__uint_as_float(g[8 * v + 1]), __uint_as_float(u[8 * v + 1])));
                        o[v].y = pack_bf16x2(silu_mul(__uint_as_float(g[8 * v + 2]), __uint_as_float(u[8 * v + 2])),
                                             silu_mul(__uint_as_float(g[8 * v + 3]), __uint_as_float(u[8 * v + 3])));
                        o[v].z = pack_bf16x2(silu_mul(__uint_as_float(g[8 * v + 4]), __uint_as_float(u[8 * v + 4])),
                                             silu_mul(__uint_as_float(g[8 * v + 5]), __uint_as_float(u[8 * v + 5])));
                        o[v].w = pack_bf16x2(silu_mul(__uint_as_float(g[8 * v + 6]), __uint_as_float(u[8 * v + 6])),
                                             silu_mul(__uint_as_float(g[8 * v + 7]), __uint_as_float(u[8 * v + 7])));
                    }
                } else {
                    uint32_t r[32];
                    tmem_ld32(taddr + c, r);
                    tc_wait_ld();
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        o[v].x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
                        o[v].y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
                        o[v].z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
                        o[v].w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
                    }
                }
                if (t.n0 + c >= n_out) continue;     // whole chunk past the last column
                if (full) {
                    // staging buffer sb: the store that last read it must be done
                    if (lane == 0) bulk_wait_group_read<1>();
                    __syncwarp();
                    const uint32_t buf = stage_buf0 + sb * STORE_BUF;
                    uint4 *sp = reinterpret_cast<uint4 *>(smem + (buf - smem0)) + lane * 4;
#pragma unroll
                    for (int v = 0; v < 4; ++v) sp[v] = o[v];
                    fence_proxy_async();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(omap, buf, t.n0 + c, t.row0 + q * 32);
                        bulk_commit_group();
                    }
                    sb ^= 1;
                } else if (row_ok) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + t.n0 + c);
#pragma unroll
                    for (int v = 0; v < 4; ++v) dst[v] = o[v];
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&tempty_bar[acc]));
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
        if (lane == 0) bulk_wait_group_all();  // every staged store has landed
        __syncwarp();
    }

    // ---------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc<TMEM_COLS>(tmem_base);
    }
}

// ---------------------------------------------------------------- paired row tiles
// The same grouped GEMM with two 128-row tiles of one expert (or of the shared
// rows) on every weight stage: per k step the MMA thread issues
// D0 += A0 B^T and D1 += A1 B^T into the two halves of TMEM, so each 32 KB
// weight tile loaded into shared memory feeds 2 x 128 rows.  Per SM that is
// 64 bytes of operands per MMA clock instead of 96, and a 3-stage ring of
// 64 KB stages covers twice the MMA time of the 4-stage ring above, which
// hides more of the L2 / HBM latency.  An expert with an odd number of row
// tiles ends with a single tile (one MMA per k step).  Both accumulators use
// all 512 TMEM columns, so there is no second accumulator for the next tile:
// 8 epilogue warps (two per TMEM lane quarter, each half of the columns) read
// both accumulators into registers (activated and rounded to bf16: 64 or 128
// registers a thread), release TMEM, and only then store, so the next tile's
// MMAs wait for the TMEM reads and the activation but not for the stores.
// Tiles are handed out dynamically: the producer warp takes the next index
// from a launch-wide atomic counter (zeroed on the stream before the launch)
// and passes it to the MMA thread and the epilogue warps through a small ring
// in shared memory, so CTAs that drew single tiles or ran slower take more
// tiles and none idles at the end while others still hold a backlog.
constexpr int P_STAGES = 3;
constexpr int P_STAGE_BYTES = 2 * A_BYTES + B_BYTES;     // 64 KB
constexpr int P_EPI_WARPS = 8;
constexpr int P_THREADS = 64 + P_EPI_WARPS * 32;         // 320
constexpr int P_SMEM_DYN = P_STAGES * P_STAGE_BYTES + P_EPI_WARPS * STORE_BUF + 1024;
constexpr int TQ = 4;  // tile indices handed from the producer to the other roles

struct PTile {
    int row0;     // first A row of the first tile (the second starts 128 rows later)
    int rv0, rv1; // rows to store of each tile (rv1 == 0: a single tile)
    int n0;       // first output column
    int e;        // expert (routed) or -1 (shared)
    int kblocks;
};

// Tile idx: routed experts first, each with ceil(ceil(rows/128)/2) row pairs x
// the column tiles (row pairs fastest, so consecutive tiles share the weight
// tile), then the shared rows in pairs x the column tiles (columns fastest).
template <int EPI>
__device__ __forceinline__ PTile decode_pair(int idx, const int *tile_base, const int *seg,
                                             const int *segc, const Params &p, int ntr,
                                             int nt_s) {
    constexpr int BN_OUT = Cfg<EPI>::BN_OUT;
    PTile t;
    int rows, g;
    if (idx < ntr) {
        int lo = 0, hi = p.E;  // tile_base[lo] <= idx < tile_base[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (tile_base[mid] <= idx) lo = mid; else hi = mid;
        }
        rows = segc[lo];
        const int mg = ((rows + BM - 1) / BM + 1) / 2;
        const int local = idx - tile_base[lo];
        const int n = local / mg;
        g = local - n * mg;
        t.row0 = seg[lo] + g * 2 * BM;
        t.n0 = n * BN_OUT;
        t.e = lo;
        t.kblocks = p.k_r / BK;
    } else {
        const int local = idx - ntr;
        g = local / nt_s;
        const int n = local - g * nt_s;
        rows = p.T;
        t.row0 = g * 2 * BM;
        t.n0 = n * BN_OUT;
        t.e = -1;
        t.kblocks = p.k_s / BK;
    }
    const int left = rows - g * 2 * BM;
    t.rv0 = min(BM, left);
    t.rv1 = max(0, min(BM, left - BM));
    return t;
}

template <int EPI>
__global__ void __launch_bounds__(P_THREADS, 1)
grouped_ffn_pair_kernel(const __grid_constant__ Maps maps, const Params p) {
    constexpr int BN_OUT = Cfg<EPI>::BN_OUT;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[P_STAGES];
    __shared__ __align__(8) uint64_t empty_bar[P_STAGES];
    __shared__ __align__(8) uint64_t tfull_bar, tempty_bar, done_bar;
    __shared__ __align__(8) uint64_t tq_full[TQ], tq_empty[TQ];
    __shared__ int tile_q[TQ];
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    __shared__ int tile_base[MAX_E + 1];
    __shared__ int seg[MAX_E];
    __shared__ int segc[MAX_E];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t smem0 = smem_u32(smem);
    volatile int *abort_flag = &abort_s;

    // ---------------------------------------------------------- prologue
    if (warp == 0) {
        const int nt_r = (p.n_out_r + BN_OUT - 1) / BN_OUT;
        int carry = 0;
        for (int e0 = 0; e0 < p.E; e0 += 32) {
            const int e = e0 + lane;
            int lo = 0, cnt = 0;
            if (e < p.E) {
                lo = p.offsets[e];
                cnt = p.offsets[e + 1] - lo;
                if (lo < 0 || cnt < 0 || lo + cnt > p.rows_r) {
                    record_status(p.status, MOE_ERR_DEVICE_FAULT);
                    lo = 0;
                    cnt = 0;
                }
                seg[e] = lo;
                segc[e] = cnt;
            }
            const int v = (((cnt + BM - 1) / BM + 1) / 2) * nt_r;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += n;
            }
            if (e < p.E) tile_base[e] = carry + incl - v;
            carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0) {
            tile_base[p.E] = carry;
            tma_prefetch_desc(&maps.o_r);
            tma_prefetch_desc(&maps.a_r);
            if (!p.bp_r) {
                tma_prefetch_desc(&maps.b0_r);
                if (EPI == EPI_SWIGLU) tma_prefetch_desc(&maps.b1_r);
            }
            if (p.T > 0) {
                tma_prefetch_desc(&maps.a_s);
                if (!p.bp_s) {
                    tma_prefetch_desc(&maps.b0_s);
                    if (EPI == EPI_SWIGLU) tma_prefetch_desc(&maps.b1_s);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            for (int s = 0; s < P_STAGES; ++s) {
                mbar_init(smem_u32(&full_bar[s]), 1);
                mbar_init(smem_u32(&empty_bar[s]), 1);
            }
            mbar_init(smem_u32(&tfull_bar), 1);
            mbar_init(smem_u32(&tempty_bar), P_EPI_WARPS);
            mbar_init(smem_u32(&done_bar), 1);
            for (int s = 0; s < TQ; ++s) {
                mbar_init(smem_u32(&tq_full[s]), 1);
                mbar_init(smem_u32(&tq_empty[s]), 1 + P_EPI_WARPS);
            }
            abort_s = 0;
            fence_barrier_init();
        }
        __syncwarp();
        tmem_alloc<TMEM_COLS>(smem_u32(&tmem_base_s));
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_s;

    const int ntr = tile_base[p.E];
    const int mg_s = p.T > 0 ? ((p.T + BM - 1) / BM + 1) / 2 : 0;
    const int nt_s = p.T > 0 ? (p.n_out_s + BN_OUT - 1) / BN_OUT : 0;
    const int total = ntr + mg_s * nt_s;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0, qs = 0;
            uint32_t phase = 0, n_issued = 0, qph = 0;
            for (;;) {
                // hand out the next tile: fetch it from the launch-wide counter and
                // publish it to the MMA thread and the epilogue warps
                if (!mbar_wait_bounded(smem_u32(&tq_empty[qs]), qph ^ 1u, abort_flag, p.status,
                                       p.timeout_ns))
                    break;
                const int idx = atomicAdd(p.tile_counter, 1);
                tile_q[qs] = idx;
                mbar_arrive(smem_u32(&tq_full[qs]));
                if (++qs == TQ) { qs = 0; qph ^= 1u; }
                if (idx >= total) break;
                const PTile t = decode_pair<EPI>(idx, tile_base, seg, segc, p, ntr, nt_s);
                const bool two = t.rv1 > 0;
                const uint32_t tx = Cfg<EPI>::TX + (two ? A_BYTES : 0);
                bool ok = true;
                for (int kb = 0; kb < t.kblocks; ++kb) {
                    if (!mbar_wait_bounded(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag,
                                           p.status, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full_bar[stage]);
                    const uint32_t a0 = smem0 + stage * P_STAGE_BYTES;
                    const uint32_t b_dst = a0 + 2 * A_BYTES;
                    const int k = kb * BK;
                    mbar_arrive_expect_tx(fb, tx);
                    if (t.e >= 0) {
                        tma_load_2d(a0, &maps.a_r, fb, k, t.row0);
                        if (two) tma_load_2d(a0 + A_BYTES, &maps.a_r, fb, k, t.row0 + BM);
                        if (p.bp_r) {
                            load_packed_b<EPI>(p, t.e, t.n0, kb, b_dst, fb);
                        } else if (EPI == EPI_SWIGLU) {
                            tma_load_3d(b_dst, &maps.b0_r, fb, k, t.n0, t.e);
                            tma_load_3d(b_dst + BN_ACC / 2 * BK * 2, &maps.b1_r, fb, k, t.n0, t.e);
                        } else {
                            tma_load_3d(b_dst, &maps.b0_r, fb, k, t.n0, t.e);
                        }
                    } else {
                        tma_load_2d(a0, &maps.a_s, fb, k, t.row0);
                        if (two) tma_load_2d(a0 + A_BYTES, &maps.a_s, fb, k, t.row0 + BM);
                        if (p.bp_s) {
                            load_packed_b<EPI>(p, -1, t.n0, kb, b_dst, fb);
                        } else if (EPI == EPI_SWIGLU) {
                            tma_load_3d(b_dst, &maps.b0_s, fb, k, t.n0, 0);
                            tma_load_3d(b_dst + BN_ACC / 2 * BK * 2, &maps.b1_s, fb, k, t.n0, 0);
                        } else {
                            const int sidx = k / p.kseg_s;
                            tma_load_3d(b_dst, &maps.b0_s, fb, k - sidx * p.kseg_s, t.n0, sidx);
                        }
                    }
                    ++n_issued;
                    if (++stage == P_STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
            }
            for (int s = 0; s < P_STAGES; ++s) {
                if (n_issued > (uint32_t)s) {
                    const uint32_t uses = (n_issued - 1 - s) / P_STAGES + 1;
                    drain_wait(smem_u32(&full_bar[s]), (uses - 1) & 1u, p.timeout_ns, p.status);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0, qs = 0;
            uint32_t phase = 0, tphase = 0, qph = 0;
            constexpr uint32_t idesc = idesc_bf16_f32<BM, Cfg<EPI>::BN_MMA>();
            for (;;) {
                if (!mbar_wait_bounded(smem_u32(&tq_full[qs]), qph, abort_flag, p.status,
                                       p.timeout_ns))
                    break;
                const int idx = tile_q[qs];
                mbar_arrive(smem_u32(&tq_empty[qs]));
                if (++qs == TQ) { qs = 0; qph ^= 1u; }
                if (idx >= total) break;
                const PTile t = decode_pair<EPI>(idx, tile_base, seg, segc, p, ntr, nt_s);
                const bool two = t.rv1 > 0;
                if (!mbar_wait_bounded(smem_u32(&tempty_bar), tphase ^ 1u, abort_flag, p.status,
                                       p.timeout_ns))
                    break;
                tc_fence_after();
                bool ok = true;
                for (int kb = 0; kb < t.kblocks; ++kb) {
                    if (!mbar_wait_bounded(smem_u32(&full_bar[stage]), phase, abort_flag, p.status,
                                           p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem0 + stage * P_STAGE_BYTES;
                    const uint64_t a0_desc = smem_desc_sw128(a0);
                    const uint64_t a1_desc = smem_desc_sw128(a0 + A_BYTES);
                    const uint64_t b_desc = smem_desc_sw128(a0 + 2 * A_BYTES);
#pragma unroll
                    for (int ks = 0; ks < BK / 16; ++ks) {
                        const uint32_t accum = (kb | ks) != 0 ? 1u : 0u;
                        tc_mma_bf16(tmem_base, a0_desc + 2 * ks, b_desc + 2 * ks, idesc, accum);
                        if (two)
                            tc_mma_bf16(tmem_base + BN_ACC, a1_desc + 2 * ks, b_desc + 2 * ks, idesc,
                                        accum);
                    }
                    tc_commit(smem_u32(&empty_bar[stage]));
                    if (++stage == P_STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit(smem_u32(&tfull_bar));
                tphase ^= 1u;
            }
            tc_commit(smem_u32(&done_bar));
            drain_wait(smem_u32(&done_bar), 0, p.timeout_ns, p.status);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue
        // Warp w drains TMEM lanes 32*(w%4).. (its 32 rows of each tile) for
        // half of the tile's output columns: full tiles leave through TMA
        // stores of 32 x 32 boxes staged in this warp's buffer, partial tiles
        // through masked direct stores (rows past rv belong to the next
        // expert or to no one).
        const int q = warp & 3;
        const int hh = (warp - 2) >> 2;                 // column half
        const int row = q * 32 + lane;
        constexpr int HALF = BN_OUT / 2;                // output columns per warp
        const uint32_t buf = smem0 + P_STAGES * P_STAGE_BYTES + (warp - 2) * STORE_BUF;
        uint4 *sp = reinterpret_cast<uint4 *>(smem + (buf - smem0)) + lane * 4;
        uint32_t tphase = 0, qph = 0;
        int qs = 0;
        for (;;) {
            int idx = 0, ok = 1;
            if (lane == 0) {
                ok = mbar_wait_bounded(smem_u32(&tq_full[qs]), qph, abort_flag, p.status,
                                       p.timeout_ns);
                if (ok) {
                    idx = tile_q[qs];
                    mbar_arrive(smem_u32(&tq_empty[qs]));
                }
            }
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            idx = __shfl_sync(0xFFFFFFFFu, idx, 0);
            if (!ok) break;
            if (++qs == TQ) { qs = 0; qph ^= 1u; }
            if (idx >= total) break;
            const PTile t = decode_pair<EPI>(idx, tile_base, seg, segc, p, ntr, nt_s);
            if (!mbar_wait_bounded(smem_u32(&tfull_bar), tphase, abort_flag, p.status,
                                   p.timeout_ns))
                break;
            tc_fence_after();
            const bool shared = t.e < 0;
            const int n_out = shared ? p.n_out_s : p.n_out_r;
            const CUtensorMap *omap = shared ? &maps.o_s : &maps.o_r;
            __nv_bfloat16 *obase = shared ? p.out_s : p.out_r;
            // 1. both accumulators into registers (this warp's rows, its half of the
            //    columns, already activated and rounded to bf16), then TMEM is
            //    released: the next tile's MMAs overlap the stores below
            constexpr int NCH = HALF / 32;  // 32-column chunks per tile and warp
            uint4 keep[2][NCH][4];
#pragma unroll
            for (int ti = 0; ti < 2; ++ti) {
                const int rv = ti == 0 ? t.rv0 : t.rv1;
                const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + ti * BN_ACC;
#pragma unroll
                for (int cc = 0; cc < NCH; ++cc) {
                    const int c = hh * HALF + cc * 32;
                    uint4 *o = keep[ti][cc];
                    if (rv <= 0) {
#pragma unroll
                        for (int v = 0; v < 4; ++v) o[v] = make_uint4(0u, 0u, 0u, 0u);
                    } else if (EPI == EPI_SWIGLU) {
                        uint32_t g[32], u[32];
                        tmem_ld32(taddr + c, g);
                        tmem_ld32(taddr + BN_ACC / 2 + c, u);
                        tc_wait_ld();
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            o[v].x = pack_bf16x2(silu_mul(__uint_as_float(g[8 * v + 0]), __uint_as_float(u[8 * v + 0])),
                                                 silu_mul(__uint_as_float(g[8 * v + 1]), __uint_as_float(u[8 * v + 1])));
                            o[v].y = pack_bf16x2(silu_mul(__uint_as_float(g[8 * v + 2]), __uint_as_float(u[8 * v + 2])),
                                                 silu_mul(__uint_as_float(g[8 * v + 3]), __uint_as_float(u[8 * v + 3])));
                            o[v].z = pack_bf16x2(silu_mul(__uint_as_float(g[8 * v + 4]), __uint_as_float(u[8 * v + 4])),
                                                 silu_mul(__uint_as_float(g[8 * v + 5]), __uint_as_float(u[8 * v + 5])));
                            o[v].w = pack_bf16x2(silu_mul(__uint_as_float(g[8 * v + 6]), __uint_as_float(u[8 * v + 6])),
                                                 silu_mul(__uint_as_float(g[8 * v + 7]), __uint_as_float(u[8 * v + 7])));
                        }
                    } else {
                        uint32_t r[32];
                        tmem_ld32(taddr + c, r);
                        tc_wait_ld();
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            o[v].x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
                            o[v].y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
                            o[v].z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
                            o[v].w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&tempty_bar));
            tphase ^= 1u;
            // 2. the stores
#pragma unroll
            for (int ti = 0; ti < 2; ++ti) {
                const int rv = ti == 0 ? t.rv0 : t.rv1;
                if (rv <= 0) continue;
                const int rbase = t.row0 + ti * BM;
                const bool full = rv == BM;
                const bool row_ok = row < rv;
                __nv_bfloat16 *orow = obase + (size_t)(rbase + row) * n_out;
#pragma unroll
                for (int cc = 0; cc < NCH; ++cc) {
                    const int c = hh * HALF + cc * 32;
                    const uint4 *o = keep[ti][cc];
                    if (t.n0 + c >= n_out) continue;  // whole chunk past the last column
                    if (full) {
                        // the staging buffer: the store that last read it must be done
                        if (lane == 0) bulk_wait_group_read<0>();
                        __syncwarp();
#pragma unroll
                        for (int v = 0; v < 4; ++v) sp[v] = o[v];
                        fence_proxy_async();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(omap, buf, t.n0 + c, rbase + q * 32);
                            bulk_commit_group();
                        }
                    } else if (row_ok) {
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + t.n0 + c);
#pragma unroll
                        for (int v = 0; v < 4; ++v) dst[v] = o[v];
                    }
                }
            }
        }
        if (lane == 0) bulk_wait_group_all();
        __syncwarp();
    }

    // ---------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc<TMEM_COLS>(tmem_base);
    }
}

// ---------------------------------------------------------------- CTA pairs
// The grouped GEMM on pairs of SMs (a cluster of 2 CTAs and
// tcgen05.mma.cta_group::2): a pair tile is 256 token rows of one expert (or
// of the shared rows) x 256 accumulator columns.  CTA r of the pair holds
// rows 128 r .. 128 r + 127 of A and rows 128 r .. of the 256-row weight tile
// (its half of the packed 32 KB tile: one contiguous 16 KB), so per SM a k
// block brings 32 KB into shared memory instead of 48 KB for the same MMA
// work; each CTA's TMEM holds the accumulator of its own 128 rows, double
// buffered, so the epilogue overlaps the next tile as in the one-CTA kernel.
// The leader (rank 0) issues the MMAs.  Every load of both CTAs completes on
// the leader's full barrier of its stage; the leader's commits arrive on the
// empty and TMEM-full barriers of both CTAs (tcgen05.commit to both CTAs of
// the pair), and both CTAs' epilogue warps arrive on the leader's TMEM-empty
// barrier.  An
// expert's last pair tile may hold fewer than 256 valid rows: rows past the
// segment are computed from whatever the loads bring and never stored.
// Packed weights only.
constexpr int C2_STAGES = 6;
constexpr int C2_STAGE_BYTES = A_BYTES + B_BYTES / 2;             // 32 KB per CTA
constexpr int C2_THREADS = 192;
constexpr int C2_SMEM_DYN = C2_STAGES * C2_STAGE_BYTES + 4 * 2 * STORE_BUF + 1024;
constexpr int C2_ROWS = 2 * BM;                                    // rows per pair tile

struct C2Tile {
    int row0;        // first A row of the pair tile
    int rows_valid;  // valid rows of the pair tile (may exceed 128, at most 256)
    int n0;          // first output column
    int e;           // expert or -1 (shared)
    int kblocks;
};

template <int EPI>
__device__ __forceinline__ C2Tile decode_c2(int idx, const int *tile_base, const int *seg,
                                            const int *segc, const Params &p, int ntr,
                                            int nt_s) {
    constexpr int BN_OUT = Cfg<EPI>::BN_OUT;
    C2Tile t;
    if (idx < ntr) {
        int lo = 0, hi = p.E;  // tile_base[lo] <= idx < tile_base[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (tile_base[mid] <= idx) lo = mid; else hi = mid;
        }
        const int cnt = segc[lo];
        const int mt = (cnt + C2_ROWS - 1) / C2_ROWS;
        const int local = idx - tile_base[lo];
        const int n = local / mt, m = local - n * mt;
        t.row0 = seg[lo] + m * C2_ROWS;
        t.rows_valid = min(C2_ROWS, cnt - m * C2_ROWS);
        t.n0 = n * BN_OUT;
        t.e = lo;
        t.kblocks = p.k_r / BK;
    } else {
        const int local = idx - ntr;
        const int m = local / nt_s, n = local - m * nt_s;
        t.row0 = m * C2_ROWS;
        t.rows_valid = min(C2_ROWS, p.T - m * C2_ROWS);
        t.n0 = n * BN_OUT;
        t.e = -1;
        t.kblocks = p.k_s / BK;
    }
    return t;
}

template <int EPI>
__global__ void __launch_bounds__(C2_THREADS, 1)
grouped_ffn_cta2_kernel(const __grid_constant__ Maps maps, const Params p) {
    constexpr int BN_OUT = Cfg<EPI>::BN_OUT;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[C2_STAGES];   // used in the leader
    __shared__ __align__(8) uint64_t empty_bar[C2_STAGES];
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];          // used in the leader
    __shared__ __align__(8) uint64_t done_bar;
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    __shared__ int tile_base[MAX_E + 1];
    __shared__ int seg[MAX_E];
    __shared__ int segc[MAX_E];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t smem0 = smem_u32(smem);
    volatile int *abort_flag = &abort_s;

    // ---------------------------------------------------------- prologue
    if (warp == 0) {
        const int nt_r = (p.n_out_r + BN_OUT - 1) / BN_OUT;
        int carry = 0;
        for (int e0 = 0; e0 < p.E; e0 += 32) {
            const int e = e0 + lane;
            int lo = 0, cnt = 0;
            if (e < p.E) {
                lo = p.offsets[e];
                cnt = p.offsets[e + 1] - lo;
                if (lo < 0 || cnt < 0 || lo + cnt > p.rows_r) {
                    record_status(p.status, MOE_ERR_DEVICE_FAULT);
                    lo = 0;
                    cnt = 0;
                }
                seg[e] = lo;
                segc[e] = cnt;
            }
            const int v = ((cnt + C2_ROWS - 1) / C2_ROWS) * nt_r;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += n;
            }
            if (e < p.E) tile_base[e] = carry + incl - v;
            carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0) {
            tile_base[p.E] = carry;
            tma_prefetch_desc(&maps.o_r);
            tma_prefetch_desc(&maps.a_r);
            tma_prefetch_desc(&maps.bpk);
            if (p.T > 0) tma_prefetch_desc(&maps.a_s);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            for (int s = 0; s < C2_STAGES; ++s) {
                mbar_init(smem_u32(&full_bar[s]), 1);
                mbar_init(smem_u32(&empty_bar[s]), 1);
            }
            for (int b = 0; b < 2; ++b) {
                mbar_init(smem_u32(&tfull_bar[b]), 1);
                mbar_init(smem_u32(&tempty_bar[b]), 2 * 4);  // 4 epilogue warps per CTA
            }
            mbar_init(smem_u32(&done_bar), 1);
            abort_s = 0;
            fence_barrier_init();
        }
        __syncwarp();
        tmem_alloc_pair<TMEM_COLS>(smem_u32(&tmem_base_s));
        tc_fence_before();
    }
    __syncthreads();
    // both CTAs' barriers are initialised and both TMEM allocations done
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_s;

    const int ntr = tile_base[p.E];
    const int mt_s = p.T > 0 ? (p.T + C2_ROWS - 1) / C2_ROWS : 0;
    const int nt_s = p.T > 0 ? (p.n_out_s + BN_OUT - 1) / BN_OUT : 0;
    const int total = ntr + mt_s * nt_s;
    const int pair_id = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t n_issued = 0;
            for (int idx = pair_id; idx < total; idx += n_pairs) {
                const C2Tile t = decode_c2<EPI>(idx, tile_base, seg, segc, p, ntr, nt_s);
                const int kb_total = t.e >= 0 ? p.k_r / BK : p.k_s / BK;
                // first 128-byte row of this CTA's half of the (n, kb = 0) weight tile
                const int64_t brow0 =
                    (t.e >= 0 ? p.bpk_row_r + ((int64_t)t.e * p.bp_nt_r + t.n0 / BN_OUT) * kb_total * 256
                              : p.bpk_row_s + (int64_t)(t.n0 / BN_OUT) * kb_total * 256) +
                    rank * BM;
                bool ok = true;
                for (int kb = 0; kb < t.kblocks; ++kb) {
                    if (!mbar_wait_bounded(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag,
                                           p.status, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = mapa_shared(smem_u32(&full_bar[stage]), 0);
                    const uint32_t a_dst = smem0 + stage * C2_STAGE_BYTES;
                    const uint32_t b_dst = a_dst + A_BYTES;
                    if (leader) mbar_arrive_expect_tx(smem_u32(&full_bar[stage]), 2 * C2_STAGE_BYTES);
                    const CUtensorMap *am = t.e >= 0 ? &maps.a_r : &maps.a_s;
                    tma_load_2d_pair(a_dst, am, fb, kb * BK, t.row0 + (int)rank * BM);
                    tma_load_2d_pair(b_dst, &maps.bpk, fb, 0, (int32_t)(brow0 + (int64_t)kb * 256));
                    ++n_issued;
                    if (++stage == C2_STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
            }
            // wind down (leader): every load of both CTAs has landed
            if (leader) {
                for (int s = 0; s < C2_STAGES; ++s) {
                    if (n_issued > (uint32_t)s) {
                        const uint32_t uses = (n_issued - 1 - s) / C2_STAGES + 1;
                        drain_wait(smem_u32(&full_bar[s]), (uses - 1) & 1u, p.timeout_ns, p.status);
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer (leader)
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            constexpr uint32_t idesc = idesc_bf16_f32<C2_ROWS, Cfg<EPI>::BN_MMA>();
            for (int idx = pair_id; idx < total; idx += n_pairs) {
                const C2Tile t = decode_c2<EPI>(idx, tile_base, seg, segc, p, ntr, nt_s);
                if (!mbar_wait_bounded(smem_u32(&tempty_bar[acc]), acc_phase ^ 1u, abort_flag,
                                       p.status, p.timeout_ns))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN_ACC;
                bool ok = true;
                for (int kb = 0; kb < t.kblocks; ++kb) {
                    if (!mbar_wait_bounded(smem_u32(&full_bar[stage]), phase, abort_flag, p.status,
                                           p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem0 + stage * C2_STAGE_BYTES;
                    const uint64_t a_desc = smem_desc_sw128(a_addr);
                    const uint64_t b_desc = smem_desc_sw128(a_addr + A_BYTES);
#pragma unroll
                    for (int ks = 0; ks < BK / 16; ++ks)
                        tc_mma_bf16_pair(d_tmem, a_desc + 2 * ks, b_desc + 2 * ks, idesc,
                                         (kb | ks) != 0 ? 1u : 0u);
                    tc_commit_pair_both(smem_u32(&empty_bar[stage]));
                    if (++stage == C2_STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit_pair_both(smem_u32(&tfull_bar[acc]));
                if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
            }
            // wind down: every MMA issued has completed (both CTAs' TMEM written)
            tc_commit_pair(smem_u32(&done_bar));
            drain_wait(smem_u32(&done_bar), 0, p.timeout_ns, p.status);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue (both CTAs)
        // as in the one-CTA kernel, for this CTA's 128 rows of the pair tile
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const uint32_t stage_buf0 = smem0 + C2_STAGES * C2_STAGE_BYTES + (warp - 2) * 2 * STORE_BUF;
        int sb = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int idx = pair_id; idx < total; idx += n_pairs) {
            const C2Tile t = decode_c2<EPI>(idx, tile_base, seg, segc, p, ntr, nt_s);
            if (!mbar_wait_bounded(smem_u32(&tfull_bar[acc]), acc_phase, abort_flag, p.status,
                                   p.timeout_ns))
                break;
            tc_fence_after();
            const int rv = min(BM, t.rows_valid - (int)rank * BM);  // this CTA's valid rows
            const int row0 = t.row0 + (int)rank * BM;
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN_ACC;
            const bool shared = t.e < 0;
            const int n_out = shared ? p.n_out_s : p.n_out_r;
            __nv_bfloat16 *orow = (shared ? p.out_s : p.out_r) + (size_t)(row0 + row) * n_out;
            const CUtensorMap *omap = shared ? &maps.o_s : &maps.o_r;
            const bool full = rv == BM;
            const bool row_ok = row < rv;
#pragma unroll 1
            for (int c = 0; c < BN_OUT && rv > 0; c += 32) {
                uint4 o[4];
                if (EPI == EPI_SWIGLU) {
                    uint32_t g[32], u[32];
                    tmem_ld32(taddr + c, g);
                    tmem_ld32(taddr + BN_ACC / 2 + c, u);
                    tc_wait_ld();
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        o[v].x = pack_bf16x2(silu_mul(__uint_as_float(g[8 * v + 0]), __uint_as_float(u[8 * v + 0])),
                                             silu_mul(__uint_as_float(g[8 * v + 1]), __uint_as_float(u[8 * v + 1])));
                        o[v].y = pack_bf16x2(silu_mul(__uint_as_float(g[8 * v + 2]), __uint_as_float(u[8 * v + 2])),
                                             silu_mul(__uint_as_float(g[8 * v + 3]), __uint_as_float(u[8 * v + 3])));
                        o[v].z = pack_bf16x2(silu_mul(__uint_as_float(g[8 * v + 4]), __uint_as_float(u[8 * v + 4])),
                                             silu_mul(__uint_as_float(g[8 * v + 5]), __uint_as_float(u[8 * v + 5])));
                        o[v].w = pack_bf16x2(silu_mul(__uint_as_float(g[8 * v + 6]), __uint_as_float(u[8 * v + 6])),
                                             silu_mul(__uint_as_float(g[8 * v + 7]), __uint_as_float(u[8 * v + 7])));
                    }
                } else {
                    uint32_t r[32];
                    tmem_ld32(taddr + c, r);
                    tc_wait_ld();
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        o[v].x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
                        o[v].y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
                        o[v].z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
                        o[v].w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
                    }
                }
                if (t.n0 + c >= n_out) continue;     // whole chunk past the last column
                if (full) {
                    if (lane == 0) bulk_wait_group_read<1>();
                    __syncwarp();
                    const uint32_t buf = stage_buf0 + sb * STORE_BUF;
                    uint4 *sp = reinterpret_cast<uint4 *>(smem + (buf - smem0)) + lane * 4;
#pragma unroll
                    for (int v = 0; v < 4; ++v) sp[v] = o[v];
                    fence_proxy_async();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(omap, buf, t.n0 + c, row0 + q * 32);
                        bulk_commit_group();
                    }
                    sb ^= 1;
                } else if (row_ok) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + t.n0 + c);
#pragma unroll
                    for (int v = 0; v < 4; ++v) dst[v] = o[v];
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty_bar[acc]), 0));
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
        if (lane == 0) bulk_wait_group_all();  // every staged store has landed
        __syncwarp();
    }

    // ---------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    // the leader's MMAs into this CTA's TMEM and every load into this CTA's
    // shared memory are done before either CTA frees TMEM or exits
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair<TMEM_COLS>(tmem_base);
    }
}

// Bounded-wait self-test: one thread waits on a barrier that never completes.
__global__ void bounded_wait_selftest_kernel(int32_t *status, int64_t timeout_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_s;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_s = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_bounded(smem_u32(&bar), 0, &abort_s, status, timeout_ns);
    __syncthreads();
}

// ---------------------------------------------------------------- host side
namespace {
// 2-D bf16 map over [rows, cols] row-major, box 64 (cols) x box_rows.
bool map_2d(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    return tensor_map_2d_bf16(m, base, rows, cols, BK, box_rows);
}

// 3-D bf16 map over [n_mat, rows, cols], box 64 (cols) x box_rows x 1.
bool map_3d(CUtensorMap *m, const void *base, uint64_t n_mat, uint64_t rows, uint64_t cols,
            uint32_t box_rows) {
    return tensor_map_3d_bf16(m, base, n_mat, rows, cols, BK, box_rows);
}

int sm_count() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
    return sms;
}

template <int EPI>
cudaError_t launch_pair(const Maps &maps, const Params &p, cudaStream_t st) {
    cudaError_t err = cudaFuncSetAttribute(grouped_ffn_pair_kernel<EPI>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM_DYN);
    if (err != cudaSuccess) return err;
    grouped_ffn_pair_kernel<EPI><<<sm_count(), P_THREADS, P_SMEM_DYN, st>>>(maps, p);
    count_launch();
    return cudaGetLastError();
}

template <int EPI>
cudaError_t launch_cta2(const Maps &maps, const Params &p, cudaStream_t st) {
    auto kern = grouped_ffn_cta2_kernel<EPI>;
    cudaError_t err =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C2_SMEM_DYN);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(C2_THREADS, 1, 1);
    cfg.dynamicSmemBytes = C2_SMEM_DYN;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // one wave of pairs: as many clusters as fit at once, at most one CTA per SM
    int pairs = sm_count() / 2;
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    int fit = 0;
    if (cudaOccupancyMaxActiveClusters(&fit, kern, &cfg) == cudaSuccess && fit > 0 && fit < pairs)
        pairs = fit;
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    err = cudaLaunchKernelEx(&cfg, kern, maps, p);
    count_launch();
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

template <int EPI, int AMODE>
cudaError_t launch_one(const Maps &maps, const Params &p, cudaStream_t st) {
    cudaError_t err = cudaFuncSetAttribute(grouped_ffn_gemm_kernel<EPI, AMODE>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_DYN);
    if (err != cudaSuccess) return err;
    grouped_ffn_gemm_kernel<EPI, AMODE>
        <<<sm_count(), NUM_THREADS + extra_threads<AMODE>(), SMEM_DYN, st>>>(maps, p);
    count_launch();
    return cudaGetLastError();
}
}  // namespace
}  // namespace gemm

cudaError_t launch_expert_ffn(const FfnArgs &a, cudaStream_t st) {
    using namespace gemm;
    if (!tensor_maps_available()) return cudaErrorNotSupported;
    const uint64_t rows_r = (uint64_t)a.T * a.K;
    const bool has_shared = a.n_shared > 0 && a.T > 0;
    const int ffs = a.n_shared * a.d_ff_shared;
    if (rows_r == 0) return cudaSuccess;
    // tile counters of the paired kernels: words 16 and 17 of the status block
    int *counters = reinterpret_cast<int *>(a.status) + 16;
    const bool pair1 = MOE_PAIR_GEMM1 || rows_r >= (uint64_t)MOE_PAIR_MIN_ROWS * a.E;
    if (pair1 || MOE_PAIR_GEMM2) {
        cudaError_t e0 = cudaMemsetAsync(counters, 0, 2 * sizeof(int), st);
        if (e0 != cudaSuccess) return e0;
    }

    // GEMM1: h = SwiGLU(x_perm) per expert; h_shared = SwiGLU(x) for the shared experts
    Maps m1;
    std::memset(&m1, 0, sizeof(m1));
    const bool gather = a.perm_token != nullptr;
    const bool packed = a.packed != nullptr;
    PackedLayout PL{};
    if (packed) PL = packed_layout(a.E, a.d, a.d_ff, a.n_shared, a.d_ff_shared);
    const uint8_t *pk = static_cast<const uint8_t *>(a.packed);
    // with packed weights the B maps stay unused (zero) and are never touched
    bool ok = packed || (map_3d(&m1.b0_r, a.w_gate, a.E, a.d_ff, a.d, BN_ACC / 2) &&
                         map_3d(&m1.b1_r, a.w_up, a.E, a.d_ff, a.d, BN_ACC / 2));
    // routed A: x_perm by tiled loads, x rows gathered by the gatherer warps, or the
    // FP8 payload by byte tiles (a_r then only stands in for the unused map)
    const bool fp8 = a.x_perm_q != nullptr;
    if (fp8)
        ok = ok && tensor_map_2d_u8(&m1.a_q, a.x_perm_q, rows_r, a.d, BK, BM) &&
             map_2d(&m1.a_r, a.x, a.T, a.d, BM);
    else
        ok = ok && map_2d(&m1.a_r, gather ? a.x : a.x_perm, gather ? a.T : rows_r, a.d, BM);
    if (!fp8) m1.a_q = m1.a_r;
    if (has_shared)
        ok = ok && map_2d(&m1.a_s, a.x, a.T, a.d, BM) &&
             (packed || (map_3d(&m1.b0_s, a.ws_gate, 1, ffs, a.d, BN_ACC / 2) &&
                         map_3d(&m1.b1_s, a.ws_up, 1, ffs, a.d, BN_ACC / 2)));
    else
        m1.a_s = m1.a_r, m1.b0_s = m1.b0_r, m1.b1_s = m1.b1_r;
    // output maps for the full-tile TMA stores (box 32 x 32, no swizzle)
    ok = ok && tensor_map_2d_bf16(&m1.o_r, a.h, rows_r, a.d_ff, 32, 32, 0);
    if (has_shared)
        ok = ok && tensor_map_2d_bf16(&m1.o_s, a.h_shared, a.T, ffs, 32, 32, 0);
    else
        m1.o_s = m1.o_r;
    if (!ok) return cudaErrorInvalidValue;
    Params p1{};
    p1.offsets = a.offsets;
    p1.perm_token = a.perm_token;
    p1.x = a.x;
    p1.x_rows = a.T;
    p1.x_scale = a.x_scale;
    p1.E = a.E;
    p1.rows_r = (int)rows_r;
    p1.T = has_shared ? a.T : 0;
    p1.n_out_r = a.d_ff;
    p1.n_out_s = ffs;
    p1.k_r = a.d;
    p1.k_s = a.d;
    p1.kseg_s = a.d;
    p1.out_r = static_cast<__nv_bfloat16 *>(a.h);
    p1.out_s = static_cast<__nv_bfloat16 *>(a.h_shared);
    p1.status = a.status;
    p1.timeout_ns = a.timeout_ns;
    p1.tile_counter = counters;
    if (packed) {
        p1.bp_r = pk + PL.gu;
        p1.bp_s = has_shared ? pk + PL.gu_s : nullptr;
        p1.bp_nt_r = PL.nt1;
    }
    // the CTA-pair kernels read the packed weights through one 2-D map of 128-byte rows
    const bool cta2 = MOE_GEMM_CTA2 && packed && !fp8 && !gather;
    if (cta2) {
        if (!tensor_map_2d_bf16(&m1.bpk, pk, PL.total / 128, BK, BK, BM, 0))
            return cudaErrorInvalidValue;
        p1.bpk_row_r = (int64_t)(PL.gu / 128);
        p1.bpk_row_s = (int64_t)(PL.gu_s / 128);
    }
    cudaError_t err = fp8      ? launch_one<EPI_SWIGLU, A_FP8>(m1, p1, st)
                      : gather ? launch_one<EPI_SWIGLU, A_GATHER>(m1, p1, st)
                      : cta2   ? launch_cta2<EPI_SWIGLU>(m1, p1, st)
                      : pair1  ? launch_pair<EPI_SWIGLU>(m1, p1, st)
                               : launch_one<EPI_SWIGLU, A_TMA>(m1, p1, st);
    if (err != cudaSuccess) return err;

    // GEMM2: y_perm = h W_d^T per expert; y_shared = h_shared Ws_d^T (k split per shared expert)
    Maps m2;
    std::memset(&m2, 0, sizeof(m2));
    ok = map_2d(&m2.a_r, a.h, rows_r, a.d_ff, BM) &&
         (packed || map_3d(&m2.b0_r, a.w_down, a.E, a.d, a.d_ff, BN_ACC));
    if (has_shared)
        ok = ok && map_2d(&m2.a_s, a.h_shared, a.T, ffs, BM) &&
             (packed || map_3d(&m2.b0_s, a.ws_down, a.n_shared, a.d, a.d_ff_shared, BN_ACC));
    else
        m2.a_s = m2.a_r, m2.b0_s = m2.b0_r;
    m2.b1_r = m2.b0_r;
    m2.a_q = m2.a_r;
    m2.b1_s = m2.b0_s;
    ok = ok && tensor_map_2d_bf16(&m2.o_r, a.y_perm, rows_r, a.d, 32, 32, 0);
    if (has_shared)
        ok = ok && tensor_map_2d_bf16(&m2.o_s, a.y_shared, a.T, a.d, 32, 32, 0);
    else
        m2.o_s = m2.o_r;
    if (!ok) return cudaErrorInvalidValue;
    Params p2 = p1;
    p2.perm_token = nullptr;
    p2.x_scale = nullptr;
    p2.n_out_r = a.d;
    p2.n_out_s = a.d;
    p2.k_r = a.d_ff;
    p2.k_s = ffs;
    p2.kseg_s = a.d_ff_shared;
    p2.out_r = static_cast<__nv_bfloat16 *>(a.y_perm);
    p2.out_s = static_cast<__nv_bfloat16 *>(a.y_shared);
    p2.tile_counter = counters + 1;
    if (packed) {
        p2.bp_r = pk + PL.down;
        p2.bp_s = has_shared ? pk + PL.down_s : nullptr;
        p2.bp_nt_r = PL.nt2;
    }
    if (cta2) {
        m2.bpk = m1.bpk;
        p2.bpk_row_r = (int64_t)(PL.down / 128);
        p2.bpk_row_s = (int64_t)(PL.down_s / 128);
        return launch_cta2<EPI_STORE>(m2, p2, st);
    }
    return MOE_PAIR_GEMM2 ? launch_pair<EPI_STORE>(m2, p2, st)
                          : launch_one<EPI_STORE, A_TMA>(m2, p2, st);
}

cudaError_t launch_bounded_wait_selftest(int64_t timeout_ns, int32_t *status, cudaStream_t st) {
    gemm::bounded_wait_selftest_kernel<<<1, 32, 0, st>>>(status, timeout_ns);
    count_launch();
    return cudaGetLastError();
}

}  // namespace moe
