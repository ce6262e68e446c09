// router_fused.cu -- router affinities and node-limited top-K in one kernel.
//
//   s_i = f(x . e_i + o_i),  b_i = s_i + bias_i
//   keep the M groups (of G contiguous experts) with the largest sum of their
//   top-(K/M) b; take the K largest b inside them; w_j = s_j / sum_j s_j
// (top-k gating over expert affinities with per-expert bias balancing, "MoE +
// Expert-Parallel Overlap (Exp08)", Implemented; a token's experts in at most
// M groups, "moe-node-limited-routing", opening definition.  f is
// DeepSeek-V3's sigmoid or the V4 sqrt(softplus).)
//
// For E <= 256 one CTA holds a 128-token tile against ALL experts (MMA
// M = 128, N = E rounded up to 16), so a token's affinities never leave the
// chip: the logits go from TMEM to registers to shared memory, the selection
// threads turn them into affinities in their registers, and only topk_idx /
// topk_w (and, when asked for, the affinities) are written.  The fp32 weights are split into three exact bf16 parts (router
// split kernel in router_tc.cu); the 12 MMAs of each 64-wide k block (or of
// PROMO consecutive k blocks) land in a fresh TMEM buffer whose values the
// epilogue adds into IEEE fp32 registers, which keeps the affinities within a
// few 1e-7 of the double-precision definition.
//
// The reduction over d is split over a cluster of C CTAs (C = 1, 2, 4 or 8,
// enough for tiles x C to fill the SMs, at least four k blocks each).  After
// its k range, CTA r owns the 128/C token rows [r*128/C, (r+1)*128/C) of the
// tile: every CTA of the cluster writes its partial logits of those rows into
// r's shared memory (distributed shared memory), and r adds the C partials in
// rank order, so the result does not depend on timing.
//
// One CTA, 320 threads:
//   warp 0      TMA producer: x tile (128 x 64) into a 3-stage A ring, each
//               weight part (N x 64) into a B ring of up to 8 stages
//   warp 1      TMEM owner (2 buffers x 256 columns), single-thread MMA issuer
//   warps 2..9  epilogue: warp w reads TMEM lanes 32*(w%4).. and columns
//               128*((w-2)/4) .. +128 (two warps per lane quarter), adds each
//               k block into fp32 registers; then the cluster reduction and,
//               with a thread per (token, group), the affinity function and
//               the selection in registers, warp shuffles between the token's
//               groups
// Every mbarrier wait is bounded; on running out the kernel records
// MOE_ERR_DEVICE_TIMEOUT, drains its own copies and MMAs and still meets its
// cluster barriers, so no CTA of the cluster is left waiting.
#include <cooperative_groups.h>

#include "kernels.h"

namespace moe {
namespace rfused {

namespace cg = cooperative_groups;

#ifndef MOE_ROUTER_PROMO
#define MOE_ROUTER_PROMO 1
#endif

constexpr int BM = 128, BK = 64, PARTS = 3;
// k blocks whose MMAs accumulate in one TMEM buffer before the epilogue adds
// the buffer into its fp32 registers
constexpr int PROMO = MOE_ROUTER_PROMO;
constexpr int A_STAGES = 3;
constexpr int A_BYTES = BM * BK * 2;          // 16 KB
constexpr int B_RING_BYTES = 160 * 1024;      // B ring budget
constexpr int MAX_B_STAGES = 8;
constexpr int NUM_THREADS = 320;
constexpr int EPI_THREADS = 256;
constexpr int ACC_COLS = 256;                 // TMEM columns per accumulator buffer
constexpr int TMEM_COLS = 512;

struct Maps {
    CUtensorMap x;      // [T, d]      box 64 x 128
    CUtensorMap parts;  // [3, E, d]   box 64 x BN x 1
};

struct Params {
    int T, E, d, G, K, M;
    int BN;            // MMA N = E rounded up to 16
    int b_stages;      // B ring stages
    int C;             // CTAs per cluster (k splits)
    int affinity;      // 0 sigmoid, 1 sqrt(softplus)
    const float *off;  // [E] or null
    const float *bias; // [E] or null
    float *scores;     // [T, E] or null
    int32_t *topk_idx; // [T, K]
    float *topk_w;     // [T, K]
    int32_t *status;
    int64_t timeout_ns;
};

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

// The affinity function, KIND a compile-time constant so that each instance
// holds one formula (a runtime branch between the two got both evaluated per
// element, measured).
template <int KIND>
__device__ __forceinline__ float affinity_fn(float L) {
    if (KIND == 1) {
        const float sp = L > 0.f ? L + log1pf(expf(-L)) : log1pf(expf(L));
        return sqrtf(sp);
    }
    // sigmoid: hardware exp2 and reciprocal (a few ulp each), a few 1e-7 from
    // the definition, far inside the affinities' 1e-5 bar.  (The IEEE-rounded
    // reciprocal costs about ten times as much here, measured.)
    return __fdividef(1.0f, 1.0f + __expf(-L));
}

// Selection key: orderable(b) in the high word, ~index in the low word, so the
// largest key is the largest b with ties to the lower index.
__device__ __forceinline__ uint64_t sel_key(float b, int i) {
    return ((uint64_t)orderable(b) << 32) | (uint32_t)(~(uint32_t)i);
}
__device__ __forceinline__ int key_index(uint64_t k) { return (int)(~(uint32_t)k); }

// 32 lanes x 16 consecutive fp32 columns: thread i receives row (lane base + i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// Named barrier over the 256 epilogue threads (id 1; 0 is __syncthreads).
__device__ __forceinline__ void epi_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory");
}

// Largest of 32 keys whose slot is below n and whose key is below `below`
// (0 if none): independent masks, then a depth-5 tree, so the 32 compares
// overlap instead of forming one dependent chain.
__device__ __forceinline__ uint64_t tree_best(const uint64_t (&k)[32], int n, uint64_t below) {
    uint64_t m[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) {
        const uint64_t a = (q < n && k[q] < below) ? k[q] : 0ull;
        const uint64_t b = (q + 16 < n && k[q + 16] < below) ? k[q + 16] : 0ull;
        m[q] = a > b ? a : b;
    }
#pragma unroll
    for (int w = 8; w > 0; w >>= 1)
#pragma unroll
        for (int q = 0; q < w; ++q) m[q] = m[q] > m[q + w] ? m[q] : m[q + w];
    return m[0];
}

// The biased affinity a selection key was made from (orderable() inverted;
// -0 comes back as +0, which adds and compares the same).
__device__ __forceinline__ float key_value(uint64_t k) {
    const uint32_t o = (uint32_t)(k >> 32);
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

// Affinities and node-limited top-K of the R token rows this CTA owns, from the
// C partial logits red[r][row][col] (r = cluster rank).  Thread (token, group
// g): the token's G groups sit in G consecutive lanes of an epilogue warp, 32
// / G tokens per warp.  A thread adds its group's gsz <= 32 logits over the C
// partials in rank order, adds the offset, applies the affinity function and
// keeps the selection key of b = s + bias per expert in registers; then
//   group score  the sum of the group's K/M best b, added in pick order;
//   kept groups  the M best group keys (a group is kept when fewer than M of
//                the token's groups have a larger key);
//   top-K        K rounds of "largest key below the last pick" over the kept
//                groups' lanes (tree inside a lane, shuffles across lanes);
//                the token's first lane recomputes each pick's unbiased s
//                from its logits for the gate.
// Keys are orderable(b) << 32 | ~index, so ties go to the lower index.
template <int C, int KIND>
__device__ __forceinline__ void select_rows(const Params &p, const float *red, int rs, int R,
                                            int m0, int rank, int ew, int lane,
                                            const float *bias_s, const float *off_s,
                                            bool aborted) {
    const int E = p.E, G = p.G, K = p.K, M = p.M;
    const int gsz = E / G, kpg = K / M;
    const int tpw = 32 / G;                         // tokens per warp
    const int sub = lane / G, g = lane - (lane / G) * G;
    const bool pow2 = (G & (G - 1)) == 0;
    for (int t0 = 0; t0 < R; t0 += 8 * tpw) {
        const int tl = t0 + ew * tpw + sub;
        const bool valid = sub < tpw && tl < R;
        const int t = m0 + rank * R + tl;
        const float *rg = red + (size_t)(valid ? tl : 0) * rs + g * gsz;
        uint64_t kv[32];
        float *so = (valid && p.scores && !aborted && t < p.T)
                        ? p.scores + (size_t)t * E + g * gsz : nullptr;
#pragma unroll
        for (int q = 0; q < 32; ++q) {
            kv[q] = 0ull;
            if (q < gsz) {
                float L = rg[q];
#pragma unroll
                for (int r = 1; r < C; ++r) L = __fadd_rn(L, rg[(size_t)r * R * rs + q]);
                if (p.off) L += off_s[g * gsz + q];
                const float sq = affinity_fn<KIND>(L);
                kv[q] = sel_key(__fadd_rn(sq, bias_s[g * gsz + q]), g * gsz + q);
                if (so) so[q] = sq;
            }
        }
        // group score: the sum of the group's K/M best b, in pick order
        uint64_t prev = ~0ull;
        float gsum = 0.f;
        for (int r = 0; r < kpg; ++r) {
            const uint64_t best = tree_best(kv, gsz, prev);
            const float bb = key_value(best);
            prev = best;
            gsum = r == 0 ? bb : __fadd_rn(gsum, bb);
        }
        const uint64_t gkey = sel_key(gsum, g);
        // kept: fewer than M of the token's groups have a larger key
        int above = 0;
        for (int q = 0; q < G; ++q) {
            const uint64_t o = __shfl_sync(0xFFFFFFFFu, gkey, sub * G + q < 32 ? sub * G + q : 0);
            above += o > gkey;
        }
        const bool kept = valid && above < M;
        // top-K over the kept groups, in pick order
        const bool writer = valid && g == 0 && t < p.T && !aborted;
        uint64_t last = ~0ull;
        float denom = 0.f;
        float sv[32];  // the picks' unbiased affinities, slot order (K <= 32)
        for (int r = 0; r < K; ++r) {
            uint64_t best = kept ? tree_best(kv, gsz, last) : 0ull;
            if (pow2) {  // the token's lanes are an aligned power of two
                for (int off = G >> 1; off > 0; off >>= 1) {
                    const uint64_t o = __shfl_xor_sync(0xFFFFFFFFu, best, off);
                    best = o > best ? o : best;
                }
            } else {
                uint64_t mx = best;
                for (int q = 0; q < G; ++q) {
                    const uint64_t o =
                        __shfl_sync(0xFFFFFFFFu, best, sub * G + q < 32 ? sub * G + q : 0);
                    mx = o > mx ? o : mx;
                }
                best = mx;
            }
            last = best;
            if (writer) {
                int e = key_index(best);
                e = e < 0 ? 0 : (e >= E ? E - 1 : e);
                // the pick's unbiased affinity, recomputed from its logits exactly as
                // its owner lane computed it
                const float *re = red + (size_t)tl * rs + e;
                float L = re[0];
#pragma unroll
                for (int c = 1; c < C; ++c) L = __fadd_rn(L, re[(size_t)c * R * rs]);
                if (p.off) L += off_s[e];
                const float bs = affinity_fn<KIND>(L);
                p.topk_idx[(size_t)t * K + r] = e;
                sv[r] = bs;
                denom = __fadd_rn(denom, bs);
            }
        }
        // gates over the chosen unbiased affinities, in slot order
        if (writer) {
            for (int r = 0; r < K; ++r) p.topk_w[(size_t)t * K + r] = __fdiv_rn(sv[r], denom);
        }
    }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
router_select_kernel(const __grid_constant__ Maps maps, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t afull[A_STAGES], aempty[A_STAGES];
    __shared__ __align__(8) uint64_t bfull[MAX_B_STAGES], bempty[MAX_B_STAGES];
    __shared__ __align__(8) uint64_t accfull[2], accempty[2];
    __shared__ __align__(8) uint64_t done_bar;
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    __shared__ float bias_s[256], off_s[256];

    cg::cluster_group cluster = cg::this_cluster();
    const int C = p.C;
    const int rank = C > 1 ? (int)cluster.block_rank() : 0;
    const int tile = blockIdx.x / C;
    const int m0 = tile * BM;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // 1024-byte aligned base, derived by an offset from the __shared__ array so
    // that accesses through it stay shared-memory accesses
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t smem0 = smem_u32(smem);
    const uint32_t b_ring0 = smem0 + A_STAGES * A_BYTES;
    const uint32_t b_bytes = (uint32_t)p.BN * BK * 2;
    volatile int *abort_flag = &abort_s;

    const int kblocks = p.d / BK;
    const int kb0 = (int)((int64_t)kblocks * rank / C);
    const int kb1 = (int)((int64_t)kblocks * (rank + 1) / C);

    for (int i = threadIdx.x; i < p.E; i += NUM_THREADS) {
        bias_s[i] = p.bias ? p.bias[i] : 0.0f;
        off_s[i] = p.off ? p.off[i] : 0.0f;
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&maps.x);
        tma_prefetch_desc(&maps.parts);
    } else if (warp == 1) {
        if (lane == 0) {
            for (int s = 0; s < A_STAGES; ++s) {
                mbar_init(smem_u32(&afull[s]), 1);
                mbar_init(smem_u32(&aempty[s]), 1);
            }
            for (int s = 0; s < p.b_stages; ++s) {
                mbar_init(smem_u32(&bfull[s]), 1);
                mbar_init(smem_u32(&bempty[s]), 1);
            }
            for (int b = 0; b < 2; ++b) {
                mbar_init(smem_u32(&accfull[b]), 1);
                mbar_init(smem_u32(&accempty[b]), EPI_THREADS / 32);
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

    // epilogue thread geometry (warps 2..9)
    const int q = warp & 3;                           // TMEM lane quarter
    const int half = (warp - 2) >> 2;                 // column half
    const int row = q * 32 + lane;                    // tile row of this thread
    const int col0 = half * 128;
    float acc[128];
#pragma unroll
    for (int c = 0; c < 128; ++c) acc[c] = 0.f;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            int as = 0, bs = 0;
            uint32_t aph = 0, bph = 0, a_issued = 0, b_issued = 0;
            bool ok = true;
            for (int kb = kb0; kb < kb1 && ok; ++kb) {
                if (!mbar_wait_bounded(smem_u32(&aempty[as]), aph ^ 1u, abort_flag, p.status,
                                       p.timeout_ns)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(smem_u32(&afull[as]), A_BYTES);
                tma_load_2d(smem0 + as * A_BYTES, &maps.x, smem_u32(&afull[as]), kb * BK, m0);
                ++a_issued;
                if (++as == A_STAGES) { as = 0; aph ^= 1u; }
                for (int part = PARTS - 1; part >= 0; --part) {
                    if (!mbar_wait_bounded(smem_u32(&bempty[bs]), bph ^ 1u, abort_flag, p.status,
                                           p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(smem_u32(&bfull[bs]), b_bytes);
                    tma_load_3d(b_ring0 + bs * b_bytes, &maps.parts, smem_u32(&bfull[bs]), kb * BK,
                                0, part);
                    ++b_issued;
                    if (++bs == p.b_stages) { bs = 0; bph ^= 1u; }
                }
            }
            // wind down: every load issued into a stage has landed
            for (int s = 0; s < A_STAGES; ++s)
                if (a_issued > (uint32_t)s)
                    drain_wait(smem_u32(&afull[s]), ((a_issued - 1 - s) / A_STAGES) & 1u,
                               p.timeout_ns, p.status);
            for (int s = 0; s < p.b_stages; ++s)
                if (b_issued > (uint32_t)s)
                    drain_wait(smem_u32(&bfull[s]), ((b_issued - 1 - s) / p.b_stages) & 1u,
                               p.timeout_ns, p.status);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int as = 0, bs = 0, buf = 0;
            uint32_t aph = 0, bph = 0, cph = 0;
            const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                   ((uint32_t)(p.BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
            bool ok = true;
            for (int kb = kb0; kb < kb1 && ok; ++kb) {
                const bool first = (kb - kb0) % PROMO == 0;
                const bool last = (kb - kb0) % PROMO == PROMO - 1 || kb + 1 == kb1;
                if ((first && !mbar_wait_bounded(smem_u32(&accempty[buf]), cph ^ 1u, abort_flag,
                                                 p.status, p.timeout_ns)) ||
                    !mbar_wait_bounded(smem_u32(&afull[as]), aph, abort_flag, p.status,
                                       p.timeout_ns)) {
                    ok = false;
                    break;
                }
                const uint64_t a_desc = smem_desc_sw128(smem0 + as * A_BYTES);
                const uint32_t d_tmem = tmem_base + buf * ACC_COLS;
                // smallest part first: the fresh accumulator is smallest while
                // the smallest products are added
                for (int part = PARTS - 1; part >= 0; --part) {
                    if (!mbar_wait_bounded(smem_u32(&bfull[bs]), bph, abort_flag, p.status,
                                           p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t b_desc = smem_desc_sw128(b_ring0 + bs * b_bytes);
#pragma unroll
                    for (int ks = 0; ks < BK / 16; ++ks)
                        tc_mma_bf16(d_tmem, a_desc + 2 * ks, b_desc + 2 * ks, idesc,
                                    (first && part == PARTS - 1 && ks == 0) ? 0u : 1u);
                    tc_commit(smem_u32(&bempty[bs]));
                    if (++bs == p.b_stages) { bs = 0; bph ^= 1u; }
                }
                if (!ok) break;
                tc_commit(smem_u32(&aempty[as]));
                if (++as == A_STAGES) { as = 0; aph ^= 1u; }
                if (last) {
                    tc_commit(smem_u32(&accfull[buf]));
                    if (++buf == 2) { buf = 0; cph ^= 1u; }
                }
            }
            tc_commit(smem_u32(&done_bar));
            drain_wait(smem_u32(&done_bar), 0, p.timeout_ns, p.status);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue: k blocks
        int buf = 0;
        uint32_t cph = 0;
        const bool has_cols = col0 < p.BN;
        for (int kb = kb0; kb < kb1; kb += PROMO) {
            if (!mbar_wait_bounded(smem_u32(&accfull[buf]), cph, abort_flag, p.status,
                                   p.timeout_ns))
                break;
            tc_fence_after();
            if (has_cols) {
                const uint32_t taddr =
                    tmem_base + ((uint32_t)(q * 32) << 16) + buf * ACC_COLS + col0;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    if (col0 + ch * 16 < p.BN) {
                        uint32_t v[16];
                        tmem_ld16(taddr + ch * 16, v);
                        tc_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            acc[ch * 16 + j] = __fadd_rn(acc[ch * 16 + j], __uint_as_float(v[j]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&accempty[buf]));
            if (++buf == 2) { buf = 0; cph ^= 1u; }
        }
    }

    // ---------------------------------------------------------- cluster reduction
    // Ring buffers are free once every CTA of the cluster has passed here (its
    // copies landed, its MMAs done).  Each epilogue thread stores its partial
    // logits into red[rank][row - owner*R][col] of the CTA that owns the row
    // (through distributed shared memory when that is another CTA).
    tc_fence_before();
    __syncthreads();
    const int R = BM / C;                 // token rows owned by each CTA of the cluster
    const int rs = p.BN + 4;              // floats per row of red
    float *red = reinterpret_cast<float *>(smem);  // [C][R][rs]
    if (C > 1) cluster.sync();
    if (warp >= 2 && col0 < p.BN) {
        const int owner = row / R;
        float *base = owner == rank ? red : cluster.map_shared_rank(red, owner);
        float *dst = base + ((size_t)rank * R + (row - owner * R)) * rs + col0;
#pragma unroll
        for (int c = 0; c < 128; c += 4)
            if (col0 + c < p.BN)
                *reinterpret_cast<float4 *>(dst + c) =
                    make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
    }
    if (C > 1) cluster.sync();

    // ---------------------------------------------------------- affinities and selection
    if (warp >= 2) {
        epi_sync();
        const bool aborted = *abort_flag != 0;
        const int ew = warp - 2;
        if (p.affinity == 1) {
            switch (C) {
            case 1: select_rows<1, 1>(p, red, rs, R, m0, rank, ew, lane, bias_s, off_s, aborted); break;
            case 2: select_rows<2, 1>(p, red, rs, R, m0, rank, ew, lane, bias_s, off_s, aborted); break;
            case 4: select_rows<4, 1>(p, red, rs, R, m0, rank, ew, lane, bias_s, off_s, aborted); break;
            default: select_rows<8, 1>(p, red, rs, R, m0, rank, ew, lane, bias_s, off_s, aborted); break;
            }
        } else {
            switch (C) {
            case 1: select_rows<1, 0>(p, red, rs, R, m0, rank, ew, lane, bias_s, off_s, aborted); break;
            case 2: select_rows<2, 0>(p, red, rs, R, m0, rank, ew, lane, bias_s, off_s, aborted); break;
            case 4: select_rows<4, 0>(p, red, rs, R, m0, rank, ew, lane, bias_s, off_s, aborted); break;
            default: select_rows<8, 0>(p, red, rs, R, m0, rank, ew, lane, bias_s, off_s, aborted); break;
            }
        }
    }

    // ---------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc<TMEM_COLS>(tmem_base);
    }
}

}  // namespace rfused

bool router_fused_supported(int E, int G, int K) {
    return E <= 256 && G <= 32 && E / G <= 32 && K <= 32;
}

int router_fused_cluster(int T, int d) {
    const int tiles = (T + rfused::BM - 1) / rfused::BM;
    const int kblocks = d / rfused::BK;
    int c = 1;
    while (c < 8 && tiles * c * 2 <= 148 && kblocks / (c * 2) >= 4) c *= 2;
    return c;
}

cudaError_t launch_router_select_fused(const void *x, const void *e_split, const float *off,
                                       const float *bias, int T, int d, int E, int G, int K,
                                       int M, int affinity, float *scores, int32_t *topk_idx,
                                       float *topk_w, int32_t *status, int64_t timeout_ns,
                                       cudaStream_t st) {
    using namespace rfused;
    if (T == 0) return cudaSuccess;
    const int BN = (E + 15) / 16 * 16;
    const int C = router_fused_cluster(T, d);
    const size_t b_bytes = (size_t)BN * BK * 2;
    int b_stages = (int)(B_RING_BYTES / b_bytes);
    if (b_stages > MAX_B_STAGES) b_stages = MAX_B_STAGES;
    const size_t ring = (size_t)A_STAGES * A_BYTES + b_stages * b_bytes;
    // after the k loop the same bytes hold the received partials, then the
    // affinity rows, group keys and candidate lists of the selection
    const size_t post = (size_t)BM * (BN + 4) * 4;
    size_t dyn = ring > post ? ring : post;
    dyn += 1024;
    Maps m;
    if (!tensor_map_2d_bf16(&m.x, x, T, d, BK, BM) ||
        !tensor_map_3d_bf16(&m.parts, e_split, PARTS, E, d, BK, BN))
        return cudaErrorInvalidValue;
    Params p{T, E, d, G, K, M, BN, b_stages, C, affinity, off, bias, scores, topk_idx, topk_w,
             status, timeout_ns};
    cudaError_t err = cudaFuncSetAttribute(router_select_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
    if (err != cudaSuccess) return err;
    const int tiles = (T + BM - 1) / BM;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(tiles * C);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = dyn;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, router_select_kernel, m, p);
    count_launch();
    return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
