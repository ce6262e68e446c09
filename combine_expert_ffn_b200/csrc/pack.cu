// pack.cu -- expert weights in the grouped GEMM's tile order.
//
// The grouped GEMM streams every expert weight from HBM about once per step
// (at V3 sizes 22.5 GB, each byte used by only ~2.5 row tiles of tokens), so
// how fast those bytes arrive decides its speed.  In the row-major layout a
// weight tile of 256 rows x 64 columns is 256 pieces of 128 bytes, 2*d bytes
// apart.  Packed, every such tile is one contiguous 32 KB block that already
// holds the 128-byte-swizzled image the MMA reads from shared memory, so the
// GEMM fetches it with a single bulk copy and the DRAM sees long sequential
// reads.  Packing is a one-time transform of static parameters (at model
// load); the packed FFN computes exactly what the row-major one does.
//
// Tile (o, n, kb), 32 KB, at ((o * NT + n) * KB + kb) * 32 KB of its region;
// row r (0..255) of the tile, 16-byte chunk c (0..7) of its 64 columns, is at
// r * 128 + ((c ^ (r % 8)) * 16).  Regions, in this order:
//   gate/up, routed  o = expert, n < ceil(d_ff/128), kb < d/64: rows 0..127
//                    gate rows n*128.., rows 128..255 up rows n*128..
//   down, routed     o = expert, n < ceil(d/256), kb < d_ff/64: rows n*256..
//                    of W_down[e] ([d, d_ff]), columns kb*64..
//   gate/up, shared  as routed, one "expert" of n_shared*d_ff_shared rows
//   down, shared     rows n*256.. of the shared down projections, columns
//                    kb*64.. of their concatenation along d_ff_shared
// Rows past the matrix are zero.
#include "kernels.h"

namespace moe {

namespace {

constexpr int TILE = 32768;
constexpr int CHUNKS = TILE / 16;  // 16-byte chunks per tile

struct PackRegion {
    int mode;          // 0 gate/up, 1 down (routed, or shared with seg > 0)
    int n_outer;       // experts (1 for the shared region)
    int nt, kb;        // column tiles, k blocks
    int rows;          // valid rows of the matrix (d_ff, d, or n_shared*d_ff_shared)
    int cols;          // row length in elements of the source matrix
    int seg;           // shared down: columns per shared expert (0 otherwise)
    int n_seg_rows;    // shared down: rows (d) of each shared expert's matrix
    const uint4 *a;    // gate or down
    const uint4 *b;    // up (gate/up only)
    uint4 *dst;
};

__global__ void __launch_bounds__(256)
pack_kernel(PackRegion R, int64_t total_chunks) {
    for (int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; q < total_chunks;
         q += (int64_t)gridDim.x * blockDim.x) {
        const int64_t tile = q / CHUNKS;
        const int w = (int)(q - tile * CHUNKS);
        const int r = w >> 3, pos = w & 7;
        const int c = pos ^ (r & 7);  // source chunk held at this position
        const int kb = (int)(tile % R.kb);
        const int64_t on = tile / R.kb;
        const int n = (int)(on % R.nt);
        const int o = (int)(on / R.nt);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        const int64_t col = (int64_t)kb * 64 + c * 8;  // first element of the chunk
        if (R.mode == 0) {
            const int half = r >> 7;
            const int row = n * 128 + (r & 127);
            if (row < R.rows) {
                const uint4 *src = half ? R.b : R.a;
                v = src[(((int64_t)o * R.rows + row) * R.cols + col) / 8];
            }
        } else {
            const int row = n * 256 + r;
            if (row < R.rows) {
                if (R.seg > 0) {  // shared down: segment s of the concatenated k
                    const int64_t s = col / R.seg, kk = col - s * R.seg;
                    v = R.a[((s * R.n_seg_rows + row) * R.seg + kk) / 8];
                } else {
                    v = R.a[(((int64_t)o * R.rows + row) * R.cols + col) / 8];
                }
            }
        }
        R.dst[q] = v;
    }
}

cudaError_t launch_region(const PackRegion &R, cudaStream_t st) {
    const int64_t tiles = (int64_t)R.n_outer * R.nt * R.kb;
    const int64_t total = tiles * CHUNKS;
    if (total == 0) return cudaSuccess;
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (total + 255) / 256;
    const int grid = (int)(want < (int64_t)sms * 16 ? want : (int64_t)sms * 16);
    pack_kernel<<<grid, 256, 0, st>>>(R, total);
    count_launch();
    return cudaGetLastError();
}

}  // namespace

PackedLayout packed_layout(int E, int d, int d_ff, int n_shared, int d_ff_shared) {
    PackedLayout L{};
    L.nt1 = (d_ff + 127) / 128;
    L.kb1 = d / 64;
    L.nt2 = (d + 255) / 256;
    L.kb2 = d_ff / 64;
    const int ffs = n_shared * d_ff_shared;
    L.nt1s = ffs > 0 ? (ffs + 127) / 128 : 0;
    L.kb2s = ffs / 64;
    size_t off = 0;
    L.gu = off;
    off += (size_t)E * L.nt1 * L.kb1 * TILE;
    L.down = off;
    off += (size_t)E * L.nt2 * L.kb2 * TILE;
    L.gu_s = off;
    off += (size_t)L.nt1s * L.kb1 * TILE;
    L.down_s = off;
    off += ffs > 0 ? (size_t)L.nt2 * L.kb2s * TILE : 0;
    L.total = off;
    return L;
}

cudaError_t launch_pack_weights(int E, int d, int d_ff, int n_shared, int d_ff_shared,
                                const void *w_gate, const void *w_up, const void *w_down,
                                const void *ws_gate, const void *ws_up, const void *ws_down,
                                void *packed, cudaStream_t st) {
    const PackedLayout L = packed_layout(E, d, d_ff, n_shared, d_ff_shared);
    char *base = static_cast<char *>(packed);
    PackRegion g{0, E, L.nt1, L.kb1, d_ff, d, 0, 0, static_cast<const uint4 *>(w_gate),
                 static_cast<const uint4 *>(w_up), reinterpret_cast<uint4 *>(base + L.gu)};
    cudaError_t err = launch_region(g, st);
    if (err != cudaSuccess) return err;
    PackRegion dn{1, E, L.nt2, L.kb2, d, d_ff, 0, 0, static_cast<const uint4 *>(w_down), nullptr,
                  reinterpret_cast<uint4 *>(base + L.down)};
    if ((err = launch_region(dn, st)) != cudaSuccess) return err;
    const int ffs = n_shared * d_ff_shared;
    if (ffs == 0) return cudaSuccess;
    PackRegion gs{0, 1, L.nt1s, L.kb1, ffs, d, 0, 0, static_cast<const uint4 *>(ws_gate),
                  static_cast<const uint4 *>(ws_up), reinterpret_cast<uint4 *>(base + L.gu_s)};
    if ((err = launch_region(gs, st)) != cudaSuccess) return err;
    PackRegion ds{1, 1, L.nt2, L.kb2s, d, ffs, d_ff_shared, d, static_cast<const uint4 *>(ws_down),
                  nullptr, reinterpret_cast<uint4 *>(base + L.down_s)};
    return launch_region(ds, st);
}

}  // namespace moe
