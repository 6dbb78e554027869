// Persistent float32 forward for stem-like layers (Cin <= 3, one group,
// K*K <= 9, Cout a multiple of 32 up to 128) on tcgen05 tensor cores with split
// tf32 operands, as in fwd_f32_tc.cu:
//
//   Col * W^T  ~=  Col_hi * W_hi^T + Col_hi * W_lo^T + Col_lo * W_hi^T,
//
// x_hi the nearest tf32 value of x and x_lo = x - x_hi. Such a layer moves far
// more bytes (offsets, mask, and above all the float32 output) than it does
// arithmetic, so the kernel is laid out to keep reads and writes in flight
// together: one CTA per SM walks an equal share of the output rows (whole
// groups of 8), in tiles of up to 128 pixels, with two A buffers and two TMEM
// accumulators.
//
//   * warps 4-15 (three threads per tile row, each a third of the taps): load
//     the next tile's offsets and mask into registers, gather the current
//     tile's modulated samples (bilinear, a neighbour outside the map
//     contributing zero), split them and write both parts into the tile's A
//     buffer; one of them issues the tile's twelve kind::tf32 MMAs;
//   * warps 0-3: read the previous tile's accumulator from TMEM, add the bias,
//     write the rows into a swizzled staging tile and hand it to TMA tensor
//     stores, which drain while the next tiles are gathered.
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

// ------------------------------------------------------------------------
// Bulk-synchronous variant for narrow outputs (Cout <= 64). With 148 CTAs a
// 224x224 layer gives each CTA under three tiles, too few for a tile-by-tile
// pipeline to reach a steady state: every tile would pay the full latency of
// its offsets, its neighbours and its stores. Here all 16 warps work on one
// round of up to three tiles at once:
//
//   1. one thread loads the round's offsets and mask with 2-D TMA boxes (128
//      pixels x all offset or mask planes of one image: one box per tile and
//      tensor, where one copy per plane would queue dozens of small copies on
//      the copy engine) and bulk-copies the band of input rows the round's
//      samples can reach into shared memory; when a round spans two images or
//      is misaligned, the threads load the offsets themselves;
//   2. each thread blends its samples, reading neighbours from the band (or
//      from global memory for a neighbour outside it), and writes the split
//      tf32 parts into the round's A tiles;
//   3. one thread issues the MMAs of all tiles of the round (one accumulator
//      per tile in TMEM);
//   4. every warp reads 16 accumulator columns of its lane quarter for each
//      tile, adds the bias, writes them into the staging tiles (which reuse the
//      A tiles' shared memory) and one thread starts the TMA stores, which
//      drain while the next round (if any) is gathered.
constexpr int B_THREADS = 512;
constexpr int B_TILES = 3;                                        // tiles per round
constexpr int B_ROWS = B_TILES * S_BM;                           // rows per round
constexpr int B_MAX_COUT = 64;
constexpr uint32_t B_BAND_MAX = 48 * 1024;                       // bytes of input rows staged per round
constexpr int B_MAX_CH = 3 * S_MAX_TAPS;                          // offset and mask planes of a sample
constexpr int B_BAND_MARGIN = 2;                                  // rows beyond the taps' reach

// 16 consecutive f32 columns of this thread's TMEM lane (32x32b shape, x16).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

struct BspArgs {
    StemArgs st;
    uint32_t band_off, od_off;
    int band_ok;  // x 16-byte aligned and a row of the map a whole number of 16-byte units
    int od_ok;    // offsets (and mask) 16-byte aligned and Ho*Wo a multiple of 4
};

template <int CIN>
__global__ void __launch_bounds__(B_THREADS, 1)
    stem_bsp_kernel(const __grid_constant__ CUtensorMap tmap_y, const __grid_constant__ CUtensorMap tmap_y8,
                    const __grid_constant__ CUtensorMap tmap_off, const __grid_constant__ CUtensorMap tmap_mask,
                    const BspArgs ba) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const StemArgs& a = ba.st;
    const Shape& s = a.s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int KC = s.K2 * CIN;
    const uint32_t bsz = (uint32_t)s.Cout * 128;  // one B tile (hi or lo)
    const int ncb = s.Cout / 32;                   // 32-column blocks of y
    float* s_w = reinterpret_cast<float*>(smem + a.w_off);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.bar_off);
    uint64_t* wbar = bars;         // raw weights landed
    uint64_t* band_bar = bars + 1;  // a round's input band landed
    uint64_t* mma_bar = bars + 2;   // [B_TILES] the MMAs of tile slot e completed
    uint64_t* od_bar = bars + 2 + B_TILES;  // a round's offsets and mask landed
    // per tile: [channel][128 rows], channels dy, dx of each tap then the mask of each tap
    float* s_od = reinterpret_cast<float*>(smem + ba.od_off);
    const int ts = 3 * s.K2 * S_BM;  // floats per tile
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 3 + B_TILES);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
    const uint32_t wbytes = (uint32_t)s.Cout * KC * 4;
    // this CTA's rows: an equal share of y's rows, cut at multiples of 8
    const long long p8 = (s.P + 7) / 8;
    const int rbeg = (int)(8 * (p8 * blockIdx.x / gridDim.x));
    const int rend = blockIdx.x + 1 == gridDim.x ? s.P : (int)(8 * (p8 * (blockIdx.x + 1) / gridDim.x));
    const int rounds = rend > rbeg ? (rend - rbeg + B_ROWS - 1) / B_ROWS : 0;
    const int plane = s.Ho * s.Wo;
    const int nch = (a.mask ? 3 : 2) * s.K2;

    // a round's rows, and the input rows its samples reach when no offset moves
    // them by more than the margin (within one image; otherwise no band)
    struct Round {
        int r0, nr, nt, b_first, b_last, yb0, yb1, pix0;
        bool use_band, od_bulk;
    };
    auto round_of = [&](int rd) {
        Round R;
        R.r0 = rbeg + rd * B_ROWS;
        R.nr = min(B_ROWS, rend - R.r0);
        R.nt = (R.nr + S_BM - 1) / S_BM;
        R.b_first = R.r0 / plane;
        R.b_last = (R.r0 + R.nr - 1) / plane;
        R.yb0 = 0;
        R.yb1 = -1;
        if (ba.band_ok && R.b_first == R.b_last) {
            const int ho0 = (R.r0 - R.b_first * plane) / s.Wo, ho1 = (R.r0 + R.nr - 1 - R.b_first * plane) / s.Wo;
            R.yb0 = max(0, ho0 * s.stride - s.pad - B_BAND_MARGIN);
            R.yb1 = min(s.H - 1, ho1 * s.stride - s.pad + (s.K - 1) * s.dil + 1 + B_BAND_MARGIN);
            if ((long long)(R.yb1 - R.yb0 + 1) * s.W * CIN * 4 > (long long)B_BAND_MAX) R.yb1 = R.yb0 - 1;
        }
        R.use_band = R.yb1 >= R.yb0;
        R.pix0 = R.r0 - R.b_first * plane;
        R.od_bulk = ba.od_ok && R.b_first == R.b_last && (R.pix0 & 3) == 0;
        return R;
    };
    // one thread: the band copy and the offset/mask boxes of a round
    auto stage_copies = [&](const Round& R) {
        if (R.use_band) {
            const uint32_t bytes = (uint32_t)(R.yb1 - R.yb0 + 1) * s.W * CIN * 4;
            const uint8_t* src = reinterpret_cast<const uint8_t*>(a.x + ((size_t)R.b_first * s.H + R.yb0) * s.W * CIN);
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive_expect_tx(ptx::smem_u32(band_bar), bytes);
            ptx::bulk_load(ptx::smem_u32(smem + ba.band_off), src, bytes, ptx::smem_u32(band_bar));
        }
        if (R.od_bulk) {
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive_expect_tx(ptx::smem_u32(od_bar), (uint32_t)(R.nt * nch * S_BM * 4));
            for (int tl = 0; tl < R.nt; ++tl) {
                const uint32_t dst = ptx::smem_u32(s_od + tl * ts);
                ptx::tma_load_2d(dst, &tmap_off, ptx::smem_u32(od_bar), R.pix0 + tl * S_BM, R.b_first * 2 * s.K2);
                if (a.mask)
                    ptx::tma_load_2d(dst + (uint32_t)(2 * s.K2 * S_BM * 4), &tmap_mask, ptx::smem_u32(od_bar),
                                     R.pix0 + tl * S_BM, R.b_first * s.K2);
            }
        }
    };

    if (tid == 0) {
        ptx::mbar_init(ptx::smem_u32(wbar), 1);
        ptx::mbar_init(ptx::smem_u32(band_bar), 1);
        for (int e = 0; e < B_TILES; ++e) ptx::mbar_init(ptx::smem_u32(&mma_bar[e]), 1);
        ptx::mbar_init(ptx::smem_u32(od_bar), 1);
        *s_abort = 0;
        ptx::fence_mbar_init();
        // round 0's inputs first: nothing else of the kernel needs to be ready for them
        if (rounds > 0) stage_copies(round_of(0));
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
    // epilogue role: lane quarter q of every tile, 16 columns starting at 16 * cq
    const int q = warp & 3, cq = warp >> 2;
    const bool epi = 16 * cq < s.Cout;
    // this lane's bias value (lane j of a warp holds column 16 * cq + (j & 15)), requested early
    const float bias_reg = (epi && a.bias) ? __ldg(a.bias + 16 * cq + (lane & 15)) : 0.f;
    __syncthreads();  // barriers initialised, TMEM allocated
    ptx::tc_fence_after();
    const uint32_t tmem = *s_tmem;
    bool ok = true;
    uint8_t* sB = smem + a.b_off;
    int band_uses = 0, od_uses = 0;
    int mma_iss[B_TILES] = {}, mma_wt[B_TILES] = {};  // per tile slot: MMA commits issued, and waited for
    const uint32_t abase = ptx::smem_u32(smem + a.a_off);
    for (int rd = 0; rd < rounds; ++rd) {
        const Round R = round_of(rd);
        const int r0 = R.r0, nr = R.nr, nt = R.nt, yb0 = R.yb0, yb1 = R.yb1;
        const bool use_band = R.use_band, od_bulk = R.od_bulk;
        // the previous round's stores have read the staging tiles (the A tiles' memory)
        // and every thread is done with the band and the offsets
        if (rd > 0) {
            if (tid == 0) ptx::bulk_wait_group_read0();
            __syncthreads();
            if (tid == 0) stage_copies(R);
        }
        if (!od_bulk) {  // the threads load the offsets themselves
            for (int e = tid; e < nch * nr; e += B_THREADS) {
                const int ch = e / nr, r = e - ch * nr;
                const int p = r0 + r, bb = p / plane, pix = p - bb * plane;
                s_od[(r >> 7) * ts + ch * S_BM + (r & (S_BM - 1))] =
                    ch < 2 * s.K2 ? __ldg(a.off + ((size_t)bb * 2 * s.K2 + ch) * plane + pix)
                                  : __ldg(a.mask + ((size_t)bb * s.K2 + (ch - 2 * s.K2)) * plane + pix);
            }
        }
        if (rd == 0) {
            // weights into the two B tiles: row n = output channel, k = tap*Cin + c, zero for k >= KC
            if (a.w_bulk) ok = ptx::mbar_wait(ptx::smem_u32(wbar), 0, s_abort, a.status, WAIT_LIMIT) && ok;
            for (int e = tid; e < s.Cout * (S_KP / 4); e += B_THREADS) {
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
                ptx::sts_v4(o + bsz, make_uint4(__float_as_uint(lo[0]), __float_as_uint(lo[1]),
                                                __float_as_uint(lo[2]), __float_as_uint(lo[3])));
            }
        }
        if (od_bulk) ok = ptx::mbar_wait(ptx::smem_u32(od_bar), od_uses & 1, s_abort, a.status, WAIT_LIMIT) && ok;
        od_uses += od_bulk ? 1 : 0;
        if (use_band) ok = ptx::mbar_wait(ptx::smem_u32(band_bar), band_uses & 1, s_abort, a.status, WAIT_LIMIT) && ok;
        band_uses += use_band ? 1 : 0;
        __syncthreads();  // s_od written by the threads (fallback) is visible
        // Tiles are gathered one after another; tile tl's MMAs run while tile tl + 1
        // is gathered, and its epilogue and stores follow that gather, so the
        // output of a round leaves while the round is still being computed.
        // Thread -> row rl of each tile, taps t = (g + tile) mod 4 + 4i (2 or 3 per tile).
        const int rl = tid & (S_BM - 1), g = tid >> 7;
        const uint32_t od_u = ptx::smem_u32(s_od), band_u = ptx::smem_u32(smem + ba.band_off);
        for (int tl = 0; tl <= nt; ++tl) {
            if (tl < nt) {
                const int r = tl * S_BM + rl;
                const uint32_t arow = abase + (uint32_t)tl * 2 * S_TILE + (uint32_t)rl * 128;
                if (r < nr) {
                    const int p = r0 + r, bb = p / plane, pix = p - bb * plane;
                    const int ho = pix / s.Wo, wo = pix - ho * s.Wo;
                    const int oy = ho * s.stride - s.pad, ox = wo * s.stride - s.pad;
                    const float* xb = a.x + (size_t)bb * s.H * s.W * CIN;
                for (int t = (g + tl) & 3; t < s.K2; t += 4) {
                    const int ti = t / s.K, tj = t - ti * s.K;
                    const uint32_t od_t = od_u + (uint32_t)(tl * ts + rl) * 4;
                    const float dy = ptx::lds_f32(od_t + (uint32_t)(2 * t * S_BM) * 4);
                    const float dx = ptx::lds_f32(od_t + (uint32_t)((2 * t + 1) * S_BM) * 4);
                    const float mk = a.mask ? ptx::lds_f32(od_t + (uint32_t)((2 * s.K2 + t) * S_BM) * 4) : 1.f;
                    int y0, x0;
                    float ly, lx;
                    split_coord(oy + ti * s.dil, dy, y0, ly);
                    split_coord(ox + tj * s.dil, dx, x0, lx);
                    bool yin0 = y0 >= 0 && y0 < s.H, yin1 = y0 + 1 >= 0 && y0 + 1 < s.H;
                    const bool xin0 = x0 >= 0 && x0 < s.W, xin1 = x0 + 1 >= 0 && x0 + 1 < s.W;
                    const float w00 = (yin0 && xin0) ? (1.f - ly) * (1.f - lx) * mk : 0.f;
                    const float w01 = (yin0 && xin1) ? (1.f - ly) * lx * mk : 0.f;
                    const float w10 = (yin1 && xin0) ? ly * (1.f - lx) * mk : 0.f;
                    const float w11 = (yin1 && xin1) ? ly * lx * mk : 0.f;
                    // clamped neighbour coordinates: a neighbour outside the map reads a valid
                    // pixel and is zeroed by its weight and the select below
                    int yc0 = min(max(y0, 0), s.H - 1), yc1 = min(max(y0 + 1, 0), s.H - 1);
                    int xc0 = min(max(x0, 0), s.W - 1), xc1 = min(max(x0 + 1, 0), s.W - 1);
                    float v[4][CIN];
                    bool in_band = use_band && yc0 >= yb0 && yc1 <= yb1;
#ifdef DCN_CHECKED
                    {  // range-checked build: the band rows read lie inside the staged band, and the
                       // neighbours read from global memory inside x
                        const size_t band_bytes = use_band ? (size_t)(yb1 - yb0 + 1) * s.W * CIN * 4 : 0;
                        const float* bandp = reinterpret_cast<const float*>(smem + ba.band_off);
                        const size_t xbytes = (size_t)s.B * s.H * s.W * CIN * 4;
                        const int cy[4] = {yc0, yc0, yc1, yc1}, cx[4] = {xc0, xc1, xc0, xc1};
                        bool ok_band = true, ok_glob = true;
                        for (int q = 0; q < 4; ++q) {
                            if (in_band)
                                ok_band = ok_band && ptx::in_range(bandp + ((size_t)(cy[q] - yb0) * s.W + cx[q]) * CIN,
                                                                   CIN * 4, bandp, band_bytes, a.status);
                            else
                                ok_glob = ok_glob && ptx::in_range(xb + ((size_t)cy[q] * s.W + cx[q]) * CIN, CIN * 4,
                                                                   a.x, xbytes, a.status);
                        }
                        if (!ok_band || !ok_glob) {  // skip the sample's neighbours: read pixel 0, add nothing
                            yin0 = yin1 = false;
                            in_band = false;
                            yc0 = yc1 = xc0 = xc1 = 0;
                        }
                    }
#endif
                    if (in_band) {
                        const uint32_t r0a = band_u + (uint32_t)(((yc0 - yb0) * s.W) * CIN) * 4;
                        const uint32_t r1a = band_u + (uint32_t)(((yc1 - yb0) * s.W) * CIN) * 4;
#pragma unroll
                        for (int c = 0; c < CIN; ++c) {
                            v[0][c] = ptx::lds_f32(r0a + (uint32_t)(xc0 * CIN + c) * 4);
                            v[1][c] = ptx::lds_f32(r0a + (uint32_t)(xc1 * CIN + c) * 4);
                            v[2][c] = ptx::lds_f32(r1a + (uint32_t)(xc0 * CIN + c) * 4);
                            v[3][c] = ptx::lds_f32(r1a + (uint32_t)(xc1 * CIN + c) * 4);
                        }
                    } else {
                        const float* p0 = xb + (size_t)yc0 * s.W * CIN;
                        const float* p1 = xb + (size_t)yc1 * s.W * CIN;
#pragma unroll
                        for (int c = 0; c < CIN; ++c) {
                            v[0][c] = __ldg(p0 + xc0 * CIN + c);
                            v[1][c] = __ldg(p0 + xc1 * CIN + c);
                            v[2][c] = __ldg(p1 + xc0 * CIN + c);
                            v[3][c] = __ldg(p1 + xc1 * CIN + c);
                        }
                    }
#pragma unroll
                    for (int c = 0; c < CIN; ++c) {
                        const float u0 = (yin0 && xin0) ? v[0][c] : 0.f, u1 = (yin0 && xin1) ? v[1][c] : 0.f;
                        const float u2 = (yin1 && xin0) ? v[2][c] : 0.f, u3 = (yin1 && xin1) ? v[3][c] : 0.f;
                        const float col = w00 * u0 + w01 * u1 + w10 * u2 + w11 * u3;
                        const int k = t * CIN + c;
                        const float hi = ptx::to_tf32(col);
                        const uint32_t o = arow + ((((k >> 2) ^ (rl & 7)) << 4) | ((k & 3) << 2));
                        ptx::sts_f32(o, hi);
                        ptx::sts_f32(o + S_TILE, col - hi);
                    }
                }
                }
                // contraction columns KC..S_KP-1 are zero
                if (g == 0)
                    for (int k = KC; k < S_KP; ++k) {
                        const uint32_t o = arow + ((((k >> 2) ^ (rl & 7)) << 4) | ((k & 3) << 2));
                        ptx::sts_f32(o, 0.f);
                        ptx::sts_f32(o + S_TILE, 0.f);
                    }
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                __syncthreads();
                if (*s_abort) break;  // read by all threads between the same two barriers: one decision
                if (tid == 0) {
                    ptx::tc_fence_after();
                    const uint32_t idesc = ptx::idesc_tf32_f32(S_BM, s.Cout);
                    const uint32_t b0 = ptx::smem_u32(sB);
                    const uint32_t a0 = abase + (uint32_t)tl * 2 * S_TILE;
                    const uint32_t d = tmem + (uint32_t)(tl * s.Cout);
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
                    ptx::mma_commit(ptx::smem_u32(&mma_bar[tl]));
                }
                ++mma_iss[tl];
            }
            if (tl == 0) continue;
            // epilogue of tile e: accumulator -> bias -> staging (tile e's A memory, free once its MMAs completed)
            const int e = tl - 1;
            const bool mok = __all_sync(0xffffffffu, ptx::mbar_wait(ptx::smem_u32(&mma_bar[e]), mma_wt[e] & 1, s_abort,
                                                                    a.status, WAIT_LIMIT));
            ++mma_wt[e];
            ptx::tc_fence_after();
            const uint32_t stg = abase + (uint32_t)e * 2 * S_TILE;
            if (mok && epi) {
                float v[16];
                tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(e * s.Cout + 16 * cq), v);
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] += __shfl_sync(0xffffffffu, bias_reg, i);
                const int row = 32 * q + lane;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    ptx::sts_v4(stg + (uint32_t)(cq >> 1) * S_TILE + sw_off(row, 4 * (cq & 1) + i),
                                make_uint4(__float_as_uint(v[4 * i]), __float_as_uint(v[4 * i + 1]),
                                           __float_as_uint(v[4 * i + 2]), __float_as_uint(v[4 * i + 3])));
            }
            ptx::tc_fence_before();
            ptx::fence_proxy_async_smem();
            __syncthreads();
            if (*s_abort) break;
            if (tid == 0) {
                // a whole tile in 128-row boxes; a shorter last tile in 8-row boxes
                const int p0 = r0 + e * S_BM, nrow = min(S_BM, nr - e * S_BM);
                for (int cb = 0; cb < ncb; ++cb) {
                    const uint32_t src = stg + (uint32_t)cb * S_TILE;
                    if (nrow == S_BM) {
                        ptx::tma_store_2d(&tmap_y, src, cb * 32, p0);
                    } else {
                        for (int r8 = 0; r8 < nrow; r8 += 8)
                            ptx::tma_store_2d(&tmap_y8, src + (uint32_t)r8 * 128, cb * 32, p0 + r8);
                    }
                }
                ptx::bulk_commit_group();
            }
        }
        if (*s_abort) break;
    }
    if (tid == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");  // stores complete

    // ------------------------------------------------------------ teardown --
    ptx::tc_fence_before();
    __syncthreads();
    if (*s_abort && tid == 0) {
        // MMAs may still be in flight: let them finish (bounded) before TMEM is released
        volatile int dummy = 0;
        for (int e = 0; e < B_TILES; ++e)
            if (mma_iss[e] > mma_wt[e])
                ptx::mbar_wait(ptx::smem_u32(&mma_bar[e]), (mma_iss[e] - 1) & 1, &dummy, nullptr, WAIT_LIMIT);
    }
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, (uint32_t)a.tmem_cols);
    }
}

struct BspPlan {
    uint32_t a_off, b_off, w_off, band_off, od_off, bar_off, smem_bytes;
    int tmem_cols;
};

BspPlan make_bsp_plan(const Shape& s) {
    BspPlan pl;
    pl.a_off = 0;                                              // B_TILES (hi, lo) A tiles; later the staging tiles
    pl.b_off = (uint32_t)B_TILES * 2 * S_TILE;                 // B hi, lo
    pl.w_off = pl.b_off + 2u * (uint32_t)s.Cout * 128;
    pl.band_off = pl.w_off + (((uint32_t)s.Cout * s.K2 * s.Cin * 4 + 15) & ~15u);
    pl.od_off = (pl.band_off + B_BAND_MAX + 1023) & ~1023u;
    pl.bar_off = pl.od_off + (uint32_t)B_MAX_CH * B_ROWS * 4;
    pl.smem_bytes = pl.bar_off + 64 + 1024;
    int cols = 32;
    while (cols < B_TILES * s.Cout) cols *= 2;
    pl.tmem_cols = cols;
    return pl;
}

template <int CIN>
cudaError_t launch_bsp(const Shape& s, const StemArgs& a0, const CUtensorMap& map, const CUtensorMap& map8,
                       cudaStream_t st) {
    const BspPlan pl = make_bsp_plan(s);
    const int plane = s.Ho * s.Wo;
    const bool od_ok = (reinterpret_cast<uintptr_t>(a0.off) & 15) == 0 &&
                       (!a0.mask || (reinterpret_cast<uintptr_t>(a0.mask) & 15) == 0) && plane % 4 == 0;
    // offsets [B * 2K^2 planes][Ho*Wo] and mask [B * K^2 planes][Ho*Wo] as 2-D float32 tensors,
    // boxes of 128 pixels x every plane of one image
    CUtensorMap map_off{}, map_mask{};
    if (od_ok) {
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
    cudaError_t e = max_dynamic_smem_once((const void*)stem_bsp_kernel<CIN>, 227 * 1024, attr);
    if (e != cudaSuccess) return e;
    BspArgs ba;
    ba.st = a0;
    ba.st.a_off = pl.a_off;
    ba.st.st_off = pl.a_off;
    ba.st.b_off = pl.b_off;
    ba.st.w_off = pl.w_off;
    ba.st.bias_off = pl.band_off;
    ba.st.bar_off = pl.bar_off;
    ba.st.tmem_cols = pl.tmem_cols;
    ba.band_off = pl.band_off;
    ba.od_off = pl.od_off;
    ba.od_ok = od_ok ? 1 : 0;
    ba.band_ok = ((reinterpret_cast<uintptr_t>(a0.x) & 15) == 0 && ((size_t)s.W * CIN * 4) % 16 == 0) ? 1 : 0;
    const int grid = (int)std::min<long long>(num_sms(), ((long long)s.P + 7) / 8);
    stem_bsp_kernel<CIN><<<grid, B_THREADS, pl.smem_bytes, st>>>(map, map8, map_off, map_mask, ba);
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
    if (s.Cout <= B_MAX_COUT && make_bsp_plan(s).smem_bytes <= 227 * 1024) return launch_bsp<CIN>(s, a, map, map8, st);
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
