// Float32 forward for stem-like layers (Cin <= 3, one group, K*K <= 9, Cout a
// multiple of 32 up to 128) on tcgen05 tensor cores with split tf32 operands,
// as in fwd_f32_tc.cu:
//
//   Col * W^T  ~=  Col_hi * W_hi^T + Col_hi * W_lo^T + Col_lo * W_hi^T,
//
// x_hi the nearest tf32 value of x and x_lo = x - x_hi. Such a layer moves far
// more bytes (offsets, mask, and above all the float32 output) than it does
// arithmetic. Two kernels, both one CTA per SM over an equal share of the
// output rows (whole groups of 8):
//
//   * stem_row_kernel (Cout 32 or 64): one thread per output row of a wave of
//     three 128-row tiles, the input band staged once per wave, each tile's
//     MMAs, read-back and stores independent of the other tiles (described
//     above the kernel);
//   * stem_persistent_kernel (wider outputs), in tiles of up to 128 pixels
//     with two A buffers and two TMEM accumulators:
//       - warps 4-15 (three threads per tile row, each a third of the taps):
//         load the next tile's offsets and mask into registers, gather the
//         current tile's modulated samples (bilinear, a neighbour outside the
//         map contributing zero), split them and write both parts into the
//         tile's A buffer; one of them issues the tile's twelve kind::tf32 MMAs;
//       - warps 0-3: read the previous tile's accumulator from TMEM, add the
//         bias, write the rows into a swizzled staging tile and hand it to TMA
//         tensor stores, which drain while the next tiles are gathered.
#include "kernels.h"
#include "tc_ptx.cuh"
#include "fwd_common.cuh"

namespace dcn {
namespace {

constexpr int S_BM = 128;          // output pixels per tile (UMMA M)
constexpr int S_KP = 32;           // padded contraction depth: one 128-byte swizzle row of float32
constexpr int S_PARTS = 3;         // gather threads per tile row
constexpr int S_TAPS_PER_PART = 3;
constexpr int S_MAX_TAPS = 9;
constexpr int S_EPI_THREADS = 128;                 // warps 0-3
constexpr int S_GATHER0 = S_EPI_THREADS;           // first gather thread
constexpr int S_THREADS = S_EPI_THREADS + S_PARTS * S_BM;
constexpr int S_MAX_COUT = 128;
constexpr uint32_t S_TILE = S_BM * 128;            // one [128 x 32] float32 swizzled tile (16 KB)
constexpr int BAR_GATHER = 1, BAR_EPI = 2;         // named barriers (0 is __syncthreads)

struct StemArgs {
    Shape s;
    const float* x;
    const float* off;
    const float* mask;
    const float* w;
    const float* bias;
    unsigned* status;
    int tiles;           // ceil(P / 128)
    int w_bulk;          // weights 16-byte aligned and a whole number of 16-byte units
    uint32_t a_off, st_off, b_off, w_off, bias_off, bar_off;
    int acc_cols;        // columns per accumulator (Cout)
    int tmem_cols;
};

__device__ __forceinline__ uint32_t sw_off(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

template <int CIN>
__global__ void __launch_bounds__(S_THREADS, 1)
    stem_persistent_kernel(const __grid_constant__ CUtensorMap tmap_y, const __grid_constant__ CUtensorMap tmap_y8,
                           const StemArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const Shape& s = a.s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int KC = s.K2 * CIN;
    const uint32_t bsz = (uint32_t)s.Cout * 128;   // one B tile (hi or lo)
    float* s_w = reinterpret_cast<float*>(smem + a.w_off);
    float* s_bias = reinterpret_cast<float*>(smem + a.bias_off);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.bar_off);
    uint64_t* wbar = bars;              // raw weights landed
    uint64_t* mma_bar = bars + 1;       // [2] the MMAs of the tile in buffer b completed
    uint64_t* acc_empty = bars + 3;     // [2] the epilogue read accumulator b
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 5);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
    const uint32_t wbytes = (uint32_t)s.Cout * KC * 4;
    // This CTA's output pixels: an equal share [rbeg, rend) of the P rows of y,
    // cut at multiples of 8 rows, walked in tiles of up to 128 rows.
    const long long p8 = (s.P + 7) / 8;
    const int rbeg = (int)(8 * (p8 * blockIdx.x / gridDim.x));
    const int rend = blockIdx.x + 1 == gridDim.x ? s.P : (int)(8 * (p8 * (blockIdx.x + 1) / gridDim.x));
    const int ntl = rend > rbeg ? (rend - rbeg + S_BM - 1) / S_BM : 0;
    auto tile_end = [&](int i) { return min(rbeg + (i + 1) * S_BM, rend); };

    if (tid == 0) {
        ptx::mbar_init(ptx::smem_u32(wbar), 1);
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(ptx::smem_u32(&mma_bar[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&acc_empty[i]), 4);
        }
        *s_abort = 0;
        ptx::fence_mbar_init();
        if (a.w_bulk) {
            ptx::mbar_arrive_expect_tx(ptx::smem_u32(wbar), wbytes);
            for (uint32_t o = 0; o < wbytes; o += 16384u)
                ptx::bulk_load(ptx::smem_u32(smem + a.w_off) + o, reinterpret_cast<const uint8_t*>(a.w) + o,
                               min(16384u, wbytes - o), ptx::smem_u32(wbar));
        }
    }
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(s_tmem), (uint32_t)a.tmem_cols);
        ptx::tmem_relinquish();
    }
    for (int i = tid; i < s.Cout; i += S_THREADS) s_bias[i] = a.bias ? __ldg(a.bias + i) : 0.f;

    // ---- gather threads: this thread's row and taps, and the first tile's offsets in flight
    const int gt = tid - S_GATHER0;
    const int row = gt & (S_BM - 1), part = gt >> 7;
    const int tp_lo = s.K2 * part / S_PARTS, tp_hi = s.K2 * (part + 1) / S_PARTS;
    const int plane = s.Ho * s.Wo;
    // offsets and mask of tile-local row `row` of this CTA's i-th tile, for this thread's taps
    // (two register sets in turn: a tile's values are requested while the tile before it is gathered)
    float S0[3 * S_TAPS_PER_PART], S1[3 * S_TAPS_PER_PART];
    auto fetch = [&](int i, float (&v)[3 * S_TAPS_PER_PART]) {
        const int p = rbeg + i * S_BM + row;
        const bool pv = i < ntl && p < tile_end(i);
        int bb = 0, pix = 0;
        if (pv) {
            bb = p / plane;
            pix = p - bb * plane;
        }
        const float* offp = a.off + (size_t)bb * 2 * s.K2 * plane + pix;
        const float* mp = a.mask ? a.mask + (size_t)bb * s.K2 * plane + pix : nullptr;
#pragma unroll
        for (int j = 0; j < S_TAPS_PER_PART; ++j) {
            const int t = tp_lo + j;
            v[3 * j] = v[3 * j + 1] = 0.f;
            v[3 * j + 2] = 1.f;
            if (pv && t < tp_hi) {
                v[3 * j] = __ldg(offp + (size_t)(2 * t) * plane);
                v[3 * j + 1] = __ldg(offp + (size_t)(2 * t + 1) * plane);
                if (mp) v[3 * j + 2] = __ldg(mp + (size_t)t * plane);
            }
        }
    };
    if (gt >= 0) {
        fetch(0, S0);
        fetch(1, S1);
    }

    // ---- weights into the two B tiles: row n = output channel, k = tap*Cin + c, zero for k >= KC
    __syncthreads();  // barriers initialised, TMEM allocated, bias staged
    bool ok = true;
    if (a.w_bulk) ok = ptx::mbar_wait(ptx::smem_u32(wbar), 0, s_abort, a.status, WAIT_LIMIT);
    uint8_t* sB = smem + a.b_off;
    for (int e = tid; e < s.Cout * (S_KP / 4); e += S_THREADS) {
        const int n = e >> 3, c = e & 7;
        float v[4], hi[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = 4 * c + j;
            v[j] = k >= KC ? 0.f : (a.w_bulk ? s_w[n * KC + k] : __ldg(a.w + (size_t)n * KC + k));
            hi[j] = ptx::to_tf32(v[j]);
            lo[j] = v[j] - hi[j];
        }
        const uint32_t o = ptx::smem_u32(sB) + sw_off(n, c);
        ptx::sts_v4(o, make_uint4(__float_as_uint(hi[0]), __float_as_uint(hi[1]), __float_as_uint(hi[2]),
                                  __float_as_uint(hi[3])));
        ptx::sts_v4(o + bsz, make_uint4(__float_as_uint(lo[0]), __float_as_uint(lo[1]), __float_as_uint(lo[2]),
                                        __float_as_uint(lo[3])));
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (gt >= 0) {
        // ------------------------------------------------------------ gather --
        const float* xb0 = a.x;
        // tile i of this CTA from the offsets in `cur`
        auto gather_tile = [&](int i, const float (&cur)[3 * S_TAPS_PER_PART]) {
            const int buf = i & 1;
            const uint32_t arow = ptx::smem_u32(smem + a.a_off) + (uint32_t)buf * 2 * S_TILE + (uint32_t)row * 128;
            // the MMAs of tile i - 2 have read this A buffer (a thread that gives up still
            // reaches the barrier below, where all decide together)
            const bool w_ok = i < 2 || ptx::mbar_wait(ptx::smem_u32(&mma_bar[buf]), ((i >> 1) - 1) & 1, s_abort,
                                                      a.status, WAIT_LIMIT);
            const int p = rbeg + i * S_BM + row;
            const bool pv = w_ok && p < tile_end(i);
            int bb = 0, oy = 0, ox = 0;
            if (pv) {
                bb = p / plane;
                const int pix = p - bb * plane;
                const int ho = pix / s.Wo, wo = pix - ho * s.Wo;
                oy = ho * s.stride - s.pad;
                ox = wo * s.stride - s.pad;
            }
            const float* xb = xb0 + (size_t)bb * s.H * s.W * CIN;
#pragma unroll
            for (int j = 0; j < S_TAPS_PER_PART; ++j) {
                const int t = tp_lo + j;
                if (t >= tp_hi) break;
                float col[CIN];
#pragma unroll
                for (int c = 0; c < CIN; ++c) col[c] = 0.f;
                if (pv) {
                    const int ti = t / s.K, tj = t - ti * s.K;
                    int y0, x0;
                    float ly, lx;
                    split_coord(oy + ti * s.dil, cur[3 * j], y0, ly);
                    split_coord(ox + tj * s.dil, cur[3 * j + 1], x0, lx);
                    float wt[4], v[4][CIN];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int r = y0 + (q >> 1), cc = x0 + (q & 1);
                        wt[q] = 0.f;
#pragma unroll
                        for (int c = 0; c < CIN; ++c) v[q][c] = 0.f;
                        if (!inside(s, r, cc)) continue;
                        wt[q] = ((q >> 1) ? ly : 1.f - ly) * ((q & 1) ? lx : 1.f - lx) * cur[3 * j + 2];
                        const float* pc = xb + ((size_t)r * s.W + cc) * CIN;
#pragma unroll
                        for (int c = 0; c < CIN; ++c) v[q][c] = __ldg(pc + c);
                    }
#pragma unroll
                    for (int c = 0; c < CIN; ++c)
                        col[c] = wt[0] * v[0][c] + wt[1] * v[1][c] + wt[2] * v[2][c] + wt[3] * v[3][c];
                }
#pragma unroll
                for (int c = 0; c < CIN; ++c) {
                    const int k = t * CIN + c;
                    const float hi = ptx::to_tf32(col[c]);
                    const uint32_t o = arow + ((((k >> 2) ^ (row & 7)) << 4) | ((k & 3) << 2));
                    ptx::sts_f32(o, hi);
                    ptx::sts_f32(o + S_TILE, col[c] - hi);
                }
            }
            if (part == S_PARTS - 1) {
                for (int k = KC; k < S_KP; ++k) {
                    const uint32_t o = arow + ((((k >> 2) ^ (row & 7)) << 4) | ((k & 3) << 2));
                    ptx::sts_f32(o, 0.f);
                    ptx::sts_f32(o + S_TILE, 0.f);
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            if (ptx::bar_or_named(BAR_GATHER, S_PARTS * S_BM, !w_ok || *s_abort)) {
                ok = false;
                return;
            }
            if (gt == 0) {
                // accumulator `buf` was read by the epilogue of tile i - 2
                if (i >= 2 && !ptx::mbar_wait(ptx::smem_u32(&acc_empty[buf]), ((i >> 1) - 1) & 1, s_abort, a.status,
                                              WAIT_LIMIT)) {
                    ok = false;
                } else {
                    ptx::tc_fence_after();
                    const uint32_t idesc = ptx::idesc_tf32_f32(S_BM, s.Cout);
                    const uint32_t a0 = arow - (uint32_t)row * 128, b0 = ptx::smem_u32(sB);
                    const uint32_t d = tmem + (uint32_t)(buf * a.acc_cols);
                    // small terms first; each K step of 8 tf32 is 32 bytes along the swizzled row
#pragma unroll
                    for (int kk = 0; kk < S_KP / 8; ++kk)
                        ptx::mma_tf32(d, ptx::sw128_desc(a0 + S_TILE + kk * 32), ptx::sw128_desc(b0 + kk * 32), idesc,
                                      kk > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < S_KP / 8; ++kk)
                        ptx::mma_tf32(d, ptx::sw128_desc(a0 + kk * 32), ptx::sw128_desc(b0 + bsz + kk * 32), idesc,
                                      1u);
#pragma unroll
                    for (int kk = 0; kk < S_KP / 8; ++kk)
                        ptx::mma_tf32(d, ptx::sw128_desc(a0 + kk * 32), ptx::sw128_desc(b0 + kk * 32), idesc, 1u);
                    ptx::mma_commit(ptx::smem_u32(&mma_bar[buf]));
                }
            }
        };
        for (int i = 0; i < ntl && ok; i += 2) {
            gather_tile(i, S0);
            fetch(i + 2, S0);
            if (i + 1 < ntl && ok) {
                gather_tile(i + 1, S1);
                fetch(i + 3, S1);
            }
        }
    } else {
        // ---------------------------------------------------------- epilogue --
        const uint32_t taddr0 = tmem + ((uint32_t)(warp * 32) << 16);
        const uint32_t stg = ptx::smem_u32(smem + a.st_off);
        for (int i = 0; i < ntl && ok; ++i) {
            const int buf = i & 1;
            const bool w_ok = ptx::mbar_wait(ptx::smem_u32(&mma_bar[buf]), (i >> 1) & 1, s_abort, a.status, WAIT_LIMIT);
            ptx::tc_fence_after();
            // the previous tile's stores have finished reading the staging tile
            if (tid == 0) ptx::bulk_wait_group_read0();
            if (ptx::bar_or_named(BAR_EPI, S_EPI_THREADS, !w_ok || *s_abort)) {  // one decision for all four warps
                ok = false;
                break;
            }
            for (int cb = 0; cb < s.Cout / 32; ++cb) {
                float v[32];
                ptx::tmem_ld32(taddr0 + (uint32_t)(buf * a.acc_cols) + cb * 32, v);
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] += s_bias[cb * 32 + j];
                const uint32_t o = stg + cb * S_TILE;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    ptx::sts_v4(o + sw_off(tid, c), make_uint4(__float_as_uint(v[4 * c]), __float_as_uint(v[4 * c + 1]),
                                                               __float_as_uint(v[4 * c + 2]),
                                                               __float_as_uint(v[4 * c + 3])));
            }
            // accumulator `buf` is free for the tile after next
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&acc_empty[buf]));
            ptx::fence_proxy_async_smem();
            ptx::bar_sync_named(BAR_EPI, S_EPI_THREADS);
            if (tid == 0) {
                // a whole tile in 128-row boxes; a CTA's shorter last tile in 8-row boxes
                // (its share ends on a multiple of 8 rows, or at the end of y)
                const int p0 = rbeg + i * S_BM, nrow = tile_end(i) - p0;
                for (int cb = 0; cb < s.Cout / 32; ++cb) {
                    if (nrow == S_BM) {
                        ptx::tma_store_2d(&tmap_y, stg + cb * S_TILE, cb * 32, p0);
                    } else {
                        for (int r8 = 0; r8 < nrow; r8 += 8)
                            ptx::tma_store_2d(&tmap_y8, stg + cb * S_TILE + (uint32_t)r8 * 128, cb * 32, p0 + r8);
                    }
                }
                ptx::bulk_commit_group();
            }
        }
        if (tid == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");  // stores complete
    }

    // ------------------------------------------------------------ teardown --
    ptx::tc_fence_before();
    __syncthreads();
    if (!ok && tid == 0) {
        // MMAs may still be in flight: let them finish (bounded) before TMEM is released
        volatile int dummy = 0;
        for (int b = 0; b < 2; ++b) {
            const int last = ((ntl - 1 - b) >= 0) ? (ntl - 1 - b) : -1;
            if (last >= 0) ptx::mbar_wait(ptx::smem_u32(&mma_bar[last & 1]), (last >> 1) & 1, &dummy, nullptr,
                                          WAIT_LIMIT);
        }
    }
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, (uint32_t)a.tmem_cols);
    }
}

// ---------------------------------------------------------------------------
// Row-per-thread stem kernel (Cout 32 or 64). One CTA per SM walks an equal
// share of y's rows (whole groups of 8) in waves of up to three 128-row tiles,
// one thread per row of a wave:
//   1. one thread starts the wave's copies: the input rows its samples reach
//      when no offset moves them by more than R_MARGIN rows (one bulk copy of
//      contiguous rows) and, per tile, the offsets and mask (2-D TMA boxes of
//      128 pixels x every plane of the image); the threads read the weights
//      and the bias; the rows are then repacked into the band, one float4 per
//      pixel (channels, then zero), with R_MARGIN zero columns on either side
//      and zero rows outside the map, so a sample inside it needs no bounds
//      test and no clamping;
//   2. the thread blends its row's K*K samples (bilinear, times the mask) from
//      the band (from global memory, with the bounds tests, for a sample
//      outside it), appends a 1 in column K*K*Cin (the bias row of B), splits
//      every value into its tf32 part and the remainder, and writes the row of
//      the tile's two A tiles with 16-byte stores;
//   3. the tile's four warps meet at their own named barrier; one thread issues
//      the tile's twelve MMAs into the tile's TMEM accumulator; the four warps
//      read it back (their lane quarter) into the tile's A memory as a swizzled
//      staging tile, which leaves by TMA tensor stores (a whole tile) or by
//      coalesced 16-byte stores of the four warps (a shorter one).
// No step of a tile waits for another tile. Where the copies cannot be used
// (unaligned rows or planes, a wave or tile across two images) the threads
// load the same values themselves.
constexpr int R_THREADS = 384;
constexpr int R_TILES = 3;
constexpr int R_ROWS = R_TILES * S_BM;
constexpr int R_MAX_COUT = 64;
constexpr int R_MARGIN = 2;  // band rows beyond the taps' reach, and zero columns on either side of a band row
constexpr uint32_t R_BAND_MAX = 64 * 1024;                         // bytes of band (float4 per pixel)
constexpr int R_BAND_PER_THREAD = (int)(R_BAND_MAX / 16 + R_THREADS - 1) / R_THREADS;

struct RowArgs {
    Shape s;
    const float* x;
    const float* off;
    const float* mask;
    const float* w;
    const float* bias;
    float* y;
    unsigned* status;
    uint32_t b_off, band_off, od_off, bar_off;  // shared memory: A tiles at 0, B (hi, lo), band, offsets, barriers
    int tmem_cols;
    int band_bulk;  // x 16-byte aligned and a map row a whole number of 16-byte units: rows by bulk copy
    int od_tma;     // offsets (and mask) 16-byte aligned and Ho*Wo a multiple of 4: 2-D TMA boxes
};

// A wave of rows [r0, r0 + nr) and its band rows [yb0, yb0 + nbr) of image b.
struct RowWave {
    int r0, nr, b, yb0, nbr;
    bool band, one_image;
};

// A sample of the row kernel with a neighbour outside the staged band: the
// four neighbours from global memory with the bounds tests (a neighbour outside
// the map contributes zero). Out of line: it is rare, and the gather loop stays small.
template <int CIN>
__device__ __noinline__ float3 row_sample_slow(const Shape& s, const float* xb, int y0, int x0, float ly, float lx,
                                               float m, const float* x, unsigned* status) {
    bool yin0 = y0 >= 0 && y0 < s.H, yin1 = y0 + 1 >= 0 && y0 + 1 < s.H;
    const bool xin0 = x0 >= 0 && x0 < s.W, xin1 = x0 + 1 >= 0 && x0 + 1 < s.W;
    // clamped neighbour coordinates: a neighbour outside the map reads a valid
    // pixel and is zeroed by its weight and the select below
    int yc0 = min(max(y0, 0), s.H - 1), yc1 = min(max(y0 + 1, 0), s.H - 1);
    int xc0 = min(max(x0, 0), s.W - 1), xc1 = min(max(x0 + 1, 0), s.W - 1);
#ifdef DCN_CHECKED
    {  // range-checked build: the neighbours read lie inside x
        const size_t xbytes = (size_t)s.B * s.H * s.W * CIN * 4;
        const int cy[4] = {yc0, yc0, yc1, yc1}, cx[4] = {xc0, xc1, xc0, xc1};
        bool okg = true;
        for (int q = 0; q < 4; ++q)
            okg = okg && ptx::in_range(xb + ((size_t)cy[q] * s.W + cx[q]) * CIN, CIN * 4, x, xbytes, status);
        if (!okg) {  // skip the sample's neighbours: read pixel 0, add nothing
            yin0 = yin1 = false;
            yc0 = yc1 = xc0 = xc1 = 0;
        }
    }
#else
    (void)x;
    (void)status;
#endif
    const float w00 = (yin0 && xin0) ? (1.f - ly) * (1.f - lx) * m : 0.f;
    const float w01 = (yin0 && xin1) ? (1.f - ly) * lx * m : 0.f;
    const float w10 = (yin1 && xin0) ? ly * (1.f - lx) * m : 0.f;
    const float w11 = (yin1 && xin1) ? ly * lx * m : 0.f;
    const float* p0 = xb + (size_t)yc0 * s.W * CIN;
    const float* p1 = xb + (size_t)yc1 * s.W * CIN;
    float v[3] = {0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < CIN; ++c) {
        const float u0 = (yin0 && xin0) ? __ldg(p0 + xc0 * CIN + c) : 0.f;
        const float u1 = (yin0 && xin1) ? __ldg(p0 + xc1 * CIN + c) : 0.f;
        const float u2 = (yin1 && xin0) ? __ldg(p1 + xc0 * CIN + c) : 0.f;
        const float u3 = (yin1 && xin1) ? __ldg(p1 + xc1 * CIN + c) : 0.f;
        v[c] = w00 * u0 + w01 * u1 + w10 * u2 + w11 * u3;
    }
    return make_float3(v[0], v[1], v[2]);
}

template <int CIN>
__global__ void __launch_bounds__(R_THREADS, 1)
    stem_row_kernel(const __grid_constant__ CUtensorMap tmap_y, const __grid_constant__ CUtensorMap tmap_off,
                    const __grid_constant__ CUtensorMap tmap_mask, const RowArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const Shape& s = a.s;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int tile = warp >> 2;   // this thread's tile of a wave; its row of the tile is also its TMEM lane
    const int rl = tid & (S_BM - 1);
    const int K2 = s.K2, KC = K2 * CIN;
    const int plane = s.Ho * s.Wo;
    const int BW = s.W + 2 * R_MARGIN;  // band row: the map's columns and R_MARGIN zero columns on either side
    const int nch = (a.mask ? 3 : 2) * K2;
    const int ts = 3 * S_MAX_TAPS * S_BM;  // floats of a tile's offsets: [plane][128 rows]
    const long long p8 = (s.P + 7) / 8;
    const int rbeg = (int)(8 * (p8 * blockIdx.x / gridDim.x));
    const int rend = blockIdx.x + 1 == gridDim.x ? s.P : (int)(8 * (p8 * (blockIdx.x + 1) / gridDim.x));
    const int waves = rend > rbeg ? (rend - rbeg + R_ROWS - 1) / R_ROWS : 0;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.bar_off);
    uint64_t* mma_bar = bars;                 // [R_TILES] the MMAs of tile j completed
    uint64_t* od_bar = bars + R_TILES;        // [R_TILES] tile j's offsets landed
    uint64_t* band_bar = bars + 2 * R_TILES;  // the wave's input rows landed
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2 * R_TILES + 1);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
    const uint32_t abase = ptx::smem_u32(smem);
    const uint32_t band_u = ptx::smem_u32(smem + a.band_off);
    const uint32_t od_u = ptx::smem_u32(smem + a.od_off);
    float* s_od = reinterpret_cast<float*>(smem + a.od_off);

    auto wave_of = [&](int wv) {
        RowWave V;
        V.r0 = rbeg + wv * R_ROWS;
        V.nr = min(R_ROWS, rend - V.r0);
        V.b = V.r0 / plane;
        V.one_image = V.b == (V.r0 + V.nr - 1) / plane;
        const int ho0 = (V.r0 - V.b * plane) / s.Wo, ho1 = (V.r0 + V.nr - 1 - V.b * plane) / s.Wo;
        V.yb0 = ho0 * s.stride - s.pad - R_MARGIN;
        const int yb1 = ho1 * s.stride - s.pad + (s.K - 1) * s.dil + R_MARGIN;
        V.nbr = yb1 - V.yb0 + 1;
        V.band = V.one_image && (long long)V.nbr * BW * 16 <= (long long)R_BAND_MAX;
        return V;
    };
    auto rows_of = [&](const RowWave& V, int j) { return min(S_BM, V.nr - j * S_BM); };
    // one thread: the wave's bulk copies (input rows into the A tiles' memory, offsets per tile)
    auto stage_copies = [&](const RowWave& V) {
        ptx::fence_proxy_async_smem();  // the threads' last accesses of that memory come first
        if (V.band && a.band_bulk) {
            const int ylo = max(V.yb0, 0), yhi = min(V.yb0 + V.nbr - 1, s.H - 1);
            if (yhi >= ylo) {
                const uint32_t bytes = (uint32_t)(yhi - ylo + 1) * s.W * CIN * 4;
                ptx::mbar_arrive_expect_tx(ptx::smem_u32(band_bar), bytes);
                ptx::bulk_load(abase, a.x + ((size_t)V.b * s.H + ylo) * s.W * CIN, bytes, ptx::smem_u32(band_bar));
            } else {
                ptx::mbar_arrive(ptx::smem_u32(band_bar));
            }
        }
        if (V.one_image && a.od_tma) {
            const int pix0 = V.r0 - V.b * plane;
            for (int j = 0; j < R_TILES; ++j) {
                if (rows_of(V, j) <= 0) continue;
                const uint32_t dst = od_u + (uint32_t)(j * ts) * 4u;
                ptx::mbar_arrive_expect_tx(ptx::smem_u32(&od_bar[j]), (uint32_t)(nch * S_BM * 4));
                ptx::tma_load_2d(dst, &tmap_off, ptx::smem_u32(&od_bar[j]), pix0 + j * S_BM, V.b * 2 * K2);
                if (a.mask)
                    ptx::tma_load_2d(dst + (uint32_t)(2 * K2 * S_BM * 4), &tmap_mask, ptx::smem_u32(&od_bar[j]),
                                     pix0 + j * S_BM, V.b * K2);
            }
        }
    };
    // every thread: what the copies do not cover (its row's offsets; the band by plain loads)
    float bv[R_BAND_PER_THREAD][CIN];
    auto band_load = [&](const RowWave& V) {
        const float* xb = a.x + (size_t)V.b * s.H * s.W * CIN;
#pragma unroll
        for (int i = 0; i < R_BAND_PER_THREAD; ++i) {
            const int e = tid + i * R_THREADS;
#pragma unroll
            for (int c = 0; c < CIN; ++c) bv[i][c] = 0.f;
            if (e < V.nbr * BW) {
                const int r = e / BW, yy = V.yb0 + r, xx = e - r * BW - R_MARGIN;
                if (yy >= 0 && yy < s.H && xx >= 0 && xx < s.W) {
                    const float* px = xb + ((size_t)yy * s.W + xx) * CIN;
#pragma unroll
                    for (int c = 0; c < CIN; ++c) bv[i][c] = __ldg(px + c);
                }
            }
        }
    };
    auto band_store = [&](const RowWave& V) {
#pragma unroll
        for (int i = 0; i < R_BAND_PER_THREAD; ++i) {
            const int e = tid + i * R_THREADS;
            if (e < V.nbr * BW)
                ptx::sts_v4(band_u + (uint32_t)e * 16u,
                            make_uint4(__float_as_uint(bv[i][0]), __float_as_uint(CIN > 1 ? bv[i][CIN > 1 ? 1 : 0] : 0.f),
                                       __float_as_uint(CIN > 2 ? bv[i][CIN > 2 ? 2 : 0] : 0.f), 0u));
        }
    };
    // the rows copied into the A tiles' memory -> the band (float4 per pixel, zero border)
    auto band_repack = [&](const RowWave& V) {
        const int ylo = max(V.yb0, 0), yhi = min(V.yb0 + V.nbr - 1, s.H - 1);
        const int dr = R_THREADS / BW, dc = R_THREADS - dr * BW;
        int r = tid / BW, c = tid - r * BW;
        for (int e = tid; e < V.nbr * BW; e += R_THREADS) {
            const int yy = V.yb0 + r, xx = c - R_MARGIN;
            float v[3] = {0.f, 0.f, 0.f};
            if (yy >= ylo && yy <= yhi && xx >= 0 && xx < s.W) {
                const uint32_t src = abase + (uint32_t)(((yy - ylo) * s.W + xx) * CIN) * 4u;
#pragma unroll
                for (int q = 0; q < CIN; ++q) v[q] = ptx::lds_f32(src + 4u * q);
            }
            ptx::sts_v4(band_u + (uint32_t)e * 16u,
                        make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]), 0u));
            c += dc;
            r += dr;
            if (c >= BW) {
                c -= BW;
                ++r;
            }
        }
    };
    // this thread's row offsets into its tile's offset block (where no TMA box brings them)
    auto od_load = [&](const RowWave& V) {
        if (tid >= V.nr) return;
        const int p = V.r0 + tid, bb = p / plane, pix = p - bb * plane;
        const float* offp = a.off + (size_t)bb * 2 * K2 * plane + pix;
        const float* mp = a.mask ? a.mask + (size_t)bb * K2 * plane + pix : nullptr;
        float* dst = s_od + tile * ts + rl;
        for (int t = 0; t < 2 * K2; ++t) dst[t * S_BM] = __ldg(offp + (size_t)t * plane);
        if (mp)
            for (int t = 0; t < K2; ++t) dst[(2 * K2 + t) * S_BM] = __ldg(mp + (size_t)t * plane);
    };

    // ---- setup: the first wave's copies, the weights (B rows: weight k of output channel n for
    // k < K*K*Cin, its bias at k = K*K*Cin, zero beyond), TMEM
    RowWave V = wave_of(0);
    if (tid == 0) {
        for (int j = 0; j < R_TILES; ++j) {
            ptx::mbar_init(ptx::smem_u32(&mma_bar[j]), 1);
            ptx::mbar_init(ptx::smem_u32(&od_bar[j]), 1);
        }
        ptx::mbar_init(ptx::smem_u32(band_bar), 1);
        *s_abort = 0;
        ptx::fence_mbar_init();
        if (waves > 0) stage_copies(V);
    }
    constexpr int WCH = (R_MAX_COUT * (S_KP / 4) + R_THREADS - 1) / R_THREADS;
    float wr[WCH][4];
#pragma unroll
    for (int i = 0; i < WCH; ++i) {
        const int e = tid + i * R_THREADS, n = e >> 3, c = e & 7;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = 4 * c + j;
            float v = 0.f;
            if (n < s.Cout) {
                if (k < KC) v = __ldg(a.w + (size_t)n * KC + k);
                else if (k == KC && a.bias) v = __ldg(a.bias + n);
            }
            wr[i][j] = v;
        }
    }
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(s_tmem), (uint32_t)a.tmem_cols);
        ptx::tmem_relinquish();
    }
    // phases of band_bar, and of this thread's tile's od_bar, waited for (a wait that gives up
    // records the timeout in the status word and raises the abort flag, read at the next wave)
    int band_uses = 0, od_uses = 0;
    if (waves > 0) {
        if (!(V.one_image && a.od_tma)) od_load(V);
        if (V.band && !a.band_bulk) band_load(V);
    }
    const uint32_t sB = ptx::smem_u32(smem + a.b_off), bsz = (uint32_t)s.Cout * 128;
#pragma unroll
    for (int i = 0; i < WCH; ++i) {
        const int e = tid + i * R_THREADS, n = e >> 3, c = e & 7;
        if (n < s.Cout) {
            float hi[4], lo[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                hi[j] = ptx::to_tf32(wr[i][j]);
                lo[j] = wr[i][j] - hi[j];
            }
            ptx::sts_v4(sB + sw_off(n, c), make_uint4(__float_as_uint(hi[0]), __float_as_uint(hi[1]),
                                                      __float_as_uint(hi[2]), __float_as_uint(hi[3])));
            ptx::sts_v4(sB + bsz + sw_off(n, c), make_uint4(__float_as_uint(lo[0]), __float_as_uint(lo[1]),
                                                            __float_as_uint(lo[2]), __float_as_uint(lo[3])));
        }
    }
    __syncthreads();  // barriers initialised before any thread waits on them
    if (waves > 0 && V.band) {
        if (a.band_bulk) {
            ptx::mbar_wait(ptx::smem_u32(band_bar), band_uses & 1, s_abort, a.status, WAIT_LIMIT);
            ++band_uses;
            band_repack(V);
        } else {
            band_store(V);
        }
    }
    ptx::fence_proxy_async_smem();  // B tiles visible to the tensor cores
    ptx::tc_fence_before();
    __syncthreads();  // TMEM allocated, B tiles, the band and the threads' offsets written
    ptx::tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t arow = abase + (uint32_t)tile * 2 * S_TILE + (uint32_t)rl * 128;
    const uint32_t stg = abase + (uint32_t)tile * 2 * S_TILE;  // the tile's A memory, reused as output staging
    int mma_iss = 0, mma_wt = 0;  // this tile's MMA commits issued, and waited for
#ifdef DCN_CHECKED
    const uint8_t* band_p = smem + a.band_off;
#endif

    for (int wv = 0; wv < waves; ++wv) {
        if (wv > 0) {
            V = wave_of(wv);
            if (rl == 0) ptx::bulk_wait_group_read0();  // the last wave's stores have read their staging
            ptx::tc_fence_before();
            __syncthreads();  // every thread is done with the band, the offsets, the A tiles and the accumulators
            if (*s_abort) break;
            if (tid == 0) stage_copies(V);
            if (!(V.one_image && a.od_tma)) od_load(V);
            if (V.band) {
                if (a.band_bulk) {
                    ptx::mbar_wait(ptx::smem_u32(band_bar), band_uses & 1, s_abort, a.status, WAIT_LIMIT);
                    ++band_uses;
                    band_repack(V);
                } else {
                    band_load(V);
                    band_store(V);
                }
            }
            __syncthreads();
            ptx::tc_fence_after();
        }
        const int trows = rows_of(V, tile);
        if (trows > 0 && V.one_image && a.od_tma) {
            ptx::mbar_wait(ptx::smem_u32(&od_bar[tile]), od_uses & 1, s_abort, a.status, WAIT_LIMIT);
            ++od_uses;
        }
        if (tid < V.nr) {
            const int p = V.r0 + tid, bb = p / plane, pix = p - bb * plane;
            const int ho = pix / s.Wo, wo = pix - ho * s.Wo;
            const int oy = ho * s.stride - s.pad, ox = wo * s.stride - s.pad;
            const float* xb = a.x + (size_t)bb * s.H * s.W * CIN;
            const uint32_t odr = od_u + (uint32_t)(tile * ts + rl) * 4u;
            float col[S_KP];
#pragma unroll
            for (int k = 0; k < S_KP; ++k) col[k] = k == KC ? 1.f : 0.f;
            int ti = 0, tj = 0;
#pragma unroll
            for (int t = 0; t < S_MAX_TAPS; ++t) {
                if (t < K2) {
                    int y0, x0;
                    float ly, lx;
                    split_coord(oy + ti * s.dil, ptx::lds_f32(odr + (uint32_t)(2 * t * S_BM) * 4u), y0, ly);
                    split_coord(ox + tj * s.dil, ptx::lds_f32(odr + (uint32_t)((2 * t + 1) * S_BM) * 4u), x0, lx);
                    const float m = a.mask ? ptx::lds_f32(odr + (uint32_t)((2 * K2 + t) * S_BM) * 4u) : 1.f;
                    float v[CIN];
                    bool fast = V.band && (unsigned)(y0 - V.yb0) < (unsigned)(V.nbr - 1) &&
                                (unsigned)(x0 + R_MARGIN) < (unsigned)(BW - 1);
#ifdef DCN_CHECKED
                    if (fast) {  // range-checked build: the four band pixels lie inside the wave's band
                        const uint8_t* q = band_p + ((size_t)(y0 - V.yb0) * BW + x0 + R_MARGIN) * 16;
                        fast = ptx::in_range(q, 32, band_p, (size_t)V.nbr * BW * 16, a.status) &&
                               ptx::in_range(q + (size_t)BW * 16, 32, band_p, (size_t)V.nbr * BW * 16, a.status);
                    }
#endif
                    if (fast) {
                        // every neighbour inside the band (zero outside the map): no tests, no clamping
                        const uint32_t q = band_u + (uint32_t)((y0 - V.yb0) * BW + x0 + R_MARGIN) * 16u;
                        const uint4 c00 = ptx::lds_v4(q), c01 = ptx::lds_v4(q + 16u);
                        const uint4 c10 = ptx::lds_v4(q + (uint32_t)BW * 16u), c11 = ptx::lds_v4(q + (uint32_t)BW * 16u + 16u);
                        const float hy0 = (1.f - ly) * m, hy1 = ly * m;
                        const float w00 = hy0 * (1.f - lx), w01 = hy0 * lx, w10 = hy1 * (1.f - lx), w11 = hy1 * lx;
                        const uint32_t u00[3] = {c00.x, c00.y, c00.z}, u01[3] = {c01.x, c01.y, c01.z};
                        const uint32_t u10[3] = {c10.x, c10.y, c10.z}, u11[3] = {c11.x, c11.y, c11.z};
#pragma unroll
                        for (int c = 0; c < CIN; ++c)
                            v[c] = w00 * __uint_as_float(u00[c]) + w01 * __uint_as_float(u01[c]) +
                                   w10 * __uint_as_float(u10[c]) + w11 * __uint_as_float(u11[c]);
                    } else {
                        const float3 u = row_sample_slow<CIN>(s, xb, y0, x0, ly, lx, m, a.x, a.status);
                        v[0] = u.x;
                        if (CIN > 1) v[CIN > 1 ? 1 : 0] = u.y;
                        if (CIN > 2) v[CIN > 2 ? 2 : 0] = u.z;
                    }
#pragma unroll
                    for (int c = 0; c < CIN; ++c) col[t * CIN + c] = v[c];
                }
                if (++tj == s.K) {
                    tj = 0;
                    ++ti;
                }
            }
            // the row of both A tiles: tf32 parts and remainders, 16 bytes at a time
#pragma unroll
            for (int c = 0; c < S_KP / 4; ++c) {
                float hi[4], lo[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    hi[j] = ptx::to_tf32(col[4 * c + j]);
                    lo[j] = col[4 * c + j] - hi[j];
                }
                const uint32_t o = arow + (uint32_t)((c ^ (rl & 7)) << 4);
                ptx::sts_v4(o, make_uint4(__float_as_uint(hi[0]), __float_as_uint(hi[1]), __float_as_uint(hi[2]),
                                          __float_as_uint(hi[3])));
                ptx::sts_v4(o + S_TILE, make_uint4(__float_as_uint(lo[0]), __float_as_uint(lo[1]),
                                                   __float_as_uint(lo[2]), __float_as_uint(lo[3])));
            }
        }
        if (trows <= 0) continue;  // uniform over the tile's four warps
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        ptx::bar_sync_named(1 + tile, S_BM);
        if (rl == 0) {
            ptx::tc_fence_after();
            const uint32_t idesc = ptx::idesc_tf32_f32(S_BM, s.Cout);
            const uint32_t a0 = stg, d = tmem + (uint32_t)(tile * s.Cout);
            // small terms first; each K step of 8 tf32 is 32 bytes along the swizzled row
#pragma unroll
            for (int kk = 0; kk < S_KP / 8; ++kk)
                ptx::mma_tf32(d, ptx::sw128_desc(a0 + S_TILE + kk * 32), ptx::sw128_desc(sB + kk * 32), idesc,
                              kk > 0 ? 1u : 0u);
#pragma unroll
            for (int kk = 0; kk < S_KP / 8; ++kk)
                ptx::mma_tf32(d, ptx::sw128_desc(a0 + kk * 32), ptx::sw128_desc(sB + bsz + kk * 32), idesc, 1u);
#pragma unroll
            for (int kk = 0; kk < S_KP / 8; ++kk)
                ptx::mma_tf32(d, ptx::sw128_desc(a0 + kk * 32), ptx::sw128_desc(sB + kk * 32), idesc, 1u);
            ptx::mma_commit(ptx::smem_u32(&mma_bar[tile]));
        }
        ++mma_iss;
        const bool mok = __all_sync(0xffffffffu, ptx::mbar_wait(ptx::smem_u32(&mma_bar[tile]), mma_wt & 1, s_abort,
                                                                a.status, WAIT_LIMIT));
        if (mok) ++mma_wt;
        ptx::tc_fence_after();
        if (mok) {
            // accumulator rows of this warp's lane quarter -> staging (the A tiles, free once the MMAs completed)
            uint32_t r0[32], r1[32];
            const uint32_t ta = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(tile * s.Cout);
            ptx::tmem_ld32_issue(ta, r0);
            if (s.Cout > 32) ptx::tmem_ld32_issue(ta + 32u, r1);
            ptx::tmem_wait_ld(r0);
            if (s.Cout > 32) ptx::tmem_wait_ld(r1);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                ptx::sts_v4(stg + sw_off(rl, i), make_uint4(r0[4 * i], r0[4 * i + 1], r0[4 * i + 2], r0[4 * i + 3]));
            if (s.Cout > 32) {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    ptx::sts_v4(stg + S_TILE + sw_off(rl, i),
                                make_uint4(r1[4 * i], r1[4 * i + 1], r1[4 * i + 2], r1[4 * i + 3]));
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        ptx::bar_sync_named(1 + tile, S_BM);
        const int p0 = V.r0 + tile * S_BM;
        if (trows == S_BM) {
            if (rl == 0) {  // a whole tile: TMA tensor stores of 32-column boxes
                for (int cb = 0; cb < s.Cout / 32; ++cb) ptx::tma_store_2d(&tmap_y, stg + (uint32_t)cb * S_TILE, cb * 32, p0);
                ptx::bulk_commit_group();
            }
        } else {
            // a shorter tile (the end of the CTA's rows): 16-byte pieces of the staging tile, each
            // warp writing whole rows of y
            const int nq = s.Cout / 4;  // 16-byte pieces per row: 8 or 16
            const int lq = nq == 16 ? 4 : 3;
            for (int f = rl; f < trows * nq; f += S_BM) {
                const int r = f >> lq, q = f & (nq - 1);
                const uint4 v = ptx::lds_v4(stg + (uint32_t)(q >> 3) * S_TILE + sw_off(r, q & 7));
                *reinterpret_cast<uint4*>(a.y + (size_t)(p0 + r) * s.Cout + 4 * q) = v;
            }
        }
    }
    if (rl == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");  // stores complete

    // ------------------------------------------------------------ teardown --
    ptx::tc_fence_before();
    __syncthreads();
    if (*s_abort && rl == 0 && mma_iss > mma_wt) {
        // MMAs may still be in flight: let them finish (bounded) before TMEM is released
        volatile int dummy = 0;
        ptx::mbar_wait(ptx::smem_u32(&mma_bar[tile]), (mma_iss - 1) & 1, &dummy, nullptr, WAIT_LIMIT);
    }
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, (uint32_t)a.tmem_cols);
    }
}

struct RowPlan {
    uint32_t b_off, band_off, od_off, bar_off, smem_bytes;
    int tmem_cols;
};

RowPlan make_row_plan(const Shape& s) {
    RowPlan pl;
    pl.b_off = (uint32_t)R_TILES * 2 * S_TILE;  // A tiles (hi, lo) of the wave's tiles at 0
    pl.band_off = pl.b_off + 2u * (uint32_t)s.Cout * 128;
    pl.od_off = pl.band_off + R_BAND_MAX;
    pl.bar_off = pl.od_off + (uint32_t)R_TILES * 3 * S_MAX_TAPS * S_BM * 4;
    pl.smem_bytes = pl.bar_off + 64 + 1024;
    int cols = 32;
    while (cols < R_TILES * s.Cout) cols *= 2;
    pl.tmem_cols = cols;
    return pl;
}

template <int CIN>
cudaError_t launch_row(const Shape& s, const StemArgs& a0, float* y, const CUtensorMap& map, cudaStream_t st) {
    const RowPlan pl = make_row_plan(s);
    const int plane = s.Ho * s.Wo;
    const bool od_tma = (reinterpret_cast<uintptr_t>(a0.off) & 15) == 0 &&
                        (!a0.mask || (reinterpret_cast<uintptr_t>(a0.mask) & 15) == 0) && plane % 4 == 0;
    // offsets [B * 2K^2 planes][Ho*Wo] and mask [B * K^2 planes][Ho*Wo] as 2-D float32 tensors,
    // boxes of 128 pixels x every plane of one image
    CUtensorMap map_off{}, map_mask{};
    if (od_tma) {
        auto encode = get_encode();
        if (!encode) return cudaErrorNotSupported;
        cuuint64_t dims[2] = {(cuuint64_t)plane, (cuuint64_t)s.B * 2 * s.K2};
        cuuint64_t strides[1] = {(cuuint64_t)plane * 4};
        cuuint32_t box[2] = {(cuuint32_t)S_BM, (cuuint32_t)(2 * s.K2)};
        cuuint32_t estr[2] = {1, 1};
        if (encode(&map_off, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(a0.off), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
        map_mask = map_off;
        if (a0.mask) {
            cuuint64_t mdims[2] = {(cuuint64_t)plane, (cuuint64_t)s.B * s.K2};
            cuuint32_t mbox[2] = {(cuuint32_t)S_BM, (cuuint32_t)s.K2};
            if (encode(&map_mask, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(a0.mask), mdims, strides,
                       mbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return cudaErrorInvalidValue;
        }
    }
    static DeviceFlags attr;
    cudaError_t e = max_dynamic_smem_once((const void*)stem_row_kernel<CIN>, 227 * 1024, attr);
    if (e != cudaSuccess) return e;
    RowArgs ra;
    ra.s = s;
    ra.x = a0.x;
    ra.off = a0.off;
    ra.mask = a0.mask;
    ra.w = a0.w;
    ra.bias = a0.bias;
    ra.y = y;
    ra.status = a0.status;
    ra.b_off = pl.b_off;
    ra.band_off = pl.band_off;
    ra.od_off = pl.od_off;
    ra.bar_off = pl.bar_off;
    ra.tmem_cols = pl.tmem_cols;
    ra.band_bulk = ((reinterpret_cast<uintptr_t>(a0.x) & 15) == 0 && ((size_t)s.W * CIN * 4) % 16 == 0) ? 1 : 0;
    ra.od_tma = od_tma ? 1 : 0;
    const int grid = (int)std::min<long long>(num_sms(), ((long long)s.P + 7) / 8);
    stem_row_kernel<CIN><<<grid, R_THREADS, pl.smem_bytes, st>>>(map, map_off, map_mask, ra);
    return cudaGetLastError();
}

struct StemPlan {
    uint32_t a_off, st_off, b_off, w_off, bias_off, bar_off, smem_bytes;
    int tmem_cols;
};

StemPlan make_stem_plan(const Shape& s) {
    StemPlan pl;
    pl.a_off = 0;                                              // two buffers of (hi, lo) A tiles
    pl.st_off = 4 * S_TILE;                                    // output staging: Cout / 32 tiles
    pl.b_off = pl.st_off + (uint32_t)(s.Cout / 32) * S_TILE;   // B hi, lo
    pl.w_off = pl.b_off + 2u * (uint32_t)s.Cout * 128;
    pl.bias_off = pl.w_off + (((uint32_t)s.Cout * s.K2 * s.Cin * 4 + 15) & ~15u);
    pl.bar_off = pl.bias_off + (uint32_t)s.Cout * 4;
    pl.smem_bytes = pl.bar_off + 64 + 1024;
    int cols = 32;
    while (cols < 2 * s.Cout) cols *= 2;
    pl.tmem_cols = cols;
    return pl;
}

template <int CIN>
cudaError_t launch_stem(const Shape& s, const float* x, const float* off, const float* mask, const float* w,
                        const float* bias, float* y, unsigned* status, cudaStream_t st) {
    const StemPlan pl = make_stem_plan(s);
    auto encode = get_encode();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap map;
    cuuint64_t dims[2] = {(cuuint64_t)s.Cout, (cuuint64_t)s.P};
    cuuint64_t strides[1] = {(cuuint64_t)s.Cout * 4};
    cuuint32_t box[2] = {32, (cuuint32_t)S_BM};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, y, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    CUtensorMap map8;  // the same, in boxes of 8 rows
    cuuint32_t box8[2] = {32, 8};
    r = encode(&map8, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, y, dims, strides, box8, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    StemArgs a;
    a.s = s;
    a.x = x;
    a.off = off;
    a.mask = mask;
    a.w = w;
    a.bias = bias;
    a.status = status;
    a.tiles = (s.P + S_BM - 1) / S_BM;
    a.w_bulk = ((reinterpret_cast<uintptr_t>(w) & 15) == 0 && ((size_t)s.Cout * s.K2 * s.Cin * 4) % 16 == 0) ? 1 : 0;
    a.a_off = pl.a_off;
    a.st_off = pl.st_off;
    a.b_off = pl.b_off;
    a.w_off = pl.w_off;
    a.bias_off = pl.bias_off;
    a.bar_off = pl.bar_off;
    a.acc_cols = s.Cout;
    a.tmem_cols = pl.tmem_cols;
    if (s.Cout <= R_MAX_COUT) return launch_row<CIN>(s, a, y, map, st);
    static DeviceFlags attr;
    cudaError_t e = max_dynamic_smem_once((const void*)stem_persistent_kernel<CIN>, 227 * 1024, attr);
    if (e != cudaSuccess) return e;
    // one CTA per SM, each an equal share of the rows (a whole number of 8-row groups)
    const int grid = (int)std::min<long long>(num_sms(), ((long long)s.P + 7) / 8);
    stem_persistent_kernel<CIN><<<grid, S_THREADS, pl.smem_bytes, st>>>(map, map8, a);
    return cudaGetLastError();
}

}  // namespace

// Cin <= 3 with one group, K*K <= 9, Cout a multiple of 32 up to 128, and index
// ranges within 32 bits (y 16-byte aligned: TMA stores).
bool fwd_f32_stem_supported(const Shape& s) {
    if (s.Cin > 3 || s.G != 1 || s.K2 > S_MAX_TAPS || s.K2 * s.Cin > S_KP) return false;
    if (s.Cout % 32 || s.Cout < 32 || s.Cout > S_MAX_COUT) return false;
    if ((long long)s.B * 2 * s.K2 * s.Ho * s.Wo >= (1LL << 31) || (long long)s.B * s.H * s.W * s.Cin >= (1LL << 31))
        return false;
    return make_stem_plan(s).smem_bytes <= 227 * 1024;
}

cudaError_t fwd_f32_stem(const Shape& s, const void* x, const void* off, const void* mask, const void* w,
                         const void* bias, void* y, unsigned* status, cudaStream_t st) {
    const float *xf = (const float*)x, *of = (const float*)off, *mf = (const float*)mask, *wf = (const float*)w,
                *bf = (const float*)bias;
    float* yf = (float*)y;
    switch (s.Cin) {
        case 1: return launch_stem<1>(s, xf, of, mf, wf, bf, yf, status, st);
        case 2: return launch_stem<2>(s, xf, of, mf, wf, bf, yf, status, st);
        default: return launch_stem<3>(s, xf, of, mf, wf, bf, yf, status, st);
    }
}

}  // namespace dcn
