// Device and host helpers shared by the bfloat16 gather-GEMM forward kernels
// (fwd_tc.cu: A operand in shared memory; fwd_tc_ts.cu: A operand in tensor
// memory): the stream-K split of (tile, chunk) units over persistent CTAs, the
// per-(row, tap) sampling records, the modulated bilinear blend, the partial
// tiles of shared output tiles and the epilogue that combines and stores them.
//
// The layer is the dense contraction Y[P x Cout] = Col[P x K*K*Cin] * W^T with
// P = B*Ho*Wo output pixels, where a row of Col holds the modulated bilinear
// samples m * x(p0 + p_k + dp_k) of one output pixel (the im2col view of the
// deformable convolution: the "Deformable ConvNets" notes, im2col appendix and
// the y(p0) equations). Included by one translation unit each; everything here
// has internal linkage.
#pragma once

#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <type_traits>

#include "kernels.h"
#include "tc_ptx.cuh"

namespace dcn {
namespace {

constexpr int BM = 128;                 // output pixels per tile (UMMA M); row index = e & 127 below
constexpr int BK = 64;                  // bf16 per K chunk (one 128-byte swizzle row)
constexpr long long WAIT_LIMIT = 2000000000LL;  // clock cycles (about a second)
constexpr int MAX_STAGES = 8;
constexpr int MAX_CTAS = 256;  // entries of the per-CTA start table in shared memory

struct FwdArgs {
    Shape s;
    const bf16* x;
    const bf16* off;
    const bf16* mask;
    const bf16* bias;
    bf16* y;
    float* partials;   // [ctas][2][BM][bn_total]
    int* counters;     // [tiles], zero on entry
    unsigned* status;
    int n_tiles, tiles, U, nq, ctas;
    int sw, nf, wl;    // pixel order: vertical strips of width sw (nf full strips, last one wl wide)
    long long total_units;
    int snap;          // a CTA never starts within the last snap-1 units of a tile (0: off)
    int bn_total;      // tile width in output channels (multiple of 16, <= 512)
    int nsub;          // accumulators per tile (1: N = bn_total; 2: 256 + rest)
    int box_rows;      // rows of one weight box
    int stages;
    int acc_cols;      // TMEM column stride between the two accumulator buffers (0: single buffer)
    int tmem_cols;
    uint32_t b_off, info_off, row_off, bar_off, b_stage_bytes;
};


// First unit of CTA c: an even split of the units, except that a start that
// would fall within the last snap-1 units of a tile moves to the next tile's
// first unit (the previous CTA takes those units), so that no CTA spends a
// segment, and its epilogue, on a sliver of a tile. Every CTA tabulates these
// starts once (starts[0..ctas], strictly increasing) and looks them up after.
__device__ __forceinline__ long long unit_begin(int c, const FwdArgs& a) {
    if (c >= a.ctas) return a.total_units;
    long long u = a.total_units * c / a.ctas;
    const long long k = u % a.U;
    if (k != 0 && k > a.U - a.snap) u += a.U - k;
    return u;
}
// The CTA whose range holds unit u: the last start at or before u.
__device__ __forceinline__ int cta_of_unit(long long u, const long long* starts, int ctas) {
    int lo = 0, hi = ctas - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (starts[mid] <= u) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// The tiles a CTA's unit range touches (its segments), in unit order.
struct SegList {
    long long ubeg, uend;
    int t0, ns, U;
};
struct Seg {
    int t, k0, k1;  // tile, and its units [k0, k1) that this CTA owns
};
__device__ __forceinline__ SegList seg_list(long long ubeg, long long uend, int U) {
    SegList L;
    L.ubeg = ubeg;
    L.uend = uend;
    L.U = U;
    if (uend <= ubeg) {
        L.t0 = 0;
        L.ns = 0;
        return L;
    }
    L.t0 = (int)(ubeg / U);
    L.ns = (int)((uend - 1) / U) - L.t0 + 1;
    return L;
}
__device__ __forceinline__ Seg seg_at(const SegList& L, int i) {
    Seg s;
    s.t = L.t0 + i;
    const long long tu = (long long)s.t * L.U;
    s.k0 = (i == 0) ? (int)(L.ubeg - tu) : 0;
    s.k1 = (i == L.ns - 1) ? (int)(L.uend - tu) : L.U;
    return s;
}

// Per-(row, tap) sampling record kept in shared memory for the current group:
// the four bilinear weights times the mask (zero for neighbours outside the
// map) as bf16 pairs, the pixel index of the top-left neighbour, and a mask of
// the neighbours to read (bit c for neighbour c = 2*dy + dx: inside the map
// and of nonzero weight). Neighbours not read take their values from a zero
// buffer instead.
struct __align__(16) TapRec {
    uint32_t w01_00;  // lo: w00, hi: w01
    uint32_t w11_10;  // lo: w10, hi: w11
    int base;         // (b*H + y0)*W + x0
    uint32_t vmask;
};

// 32 zero bytes: the source of every neighbour that is not read.
__device__ __align__(32) uint32_t g_zero_slice[8];

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&t);
}

// Modulated bilinear blend of one sample's four neighbour slices (16 channels
// each, as bf16 pairs) into 16 bf16 values: packed bf16x2 products and sums,
// each partial result rounded to bf16.
__device__ __forceinline__ void blend16(uint32_t (&r)[8], const uint32_t (&v)[4][8], uint32_t w01_00,
                                        uint32_t w11_10) {
    const uint32_t w00 = __byte_perm(w01_00, 0, 0x1010), w01 = __byte_perm(w01_00, 0, 0x3232);
    const uint32_t w10 = __byte_perm(w11_10, 0, 0x1010), w11 = __byte_perm(w11_10, 0, 0x3232);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        asm("{\n\t"
            "mul.rn.bf16x2 %0, %1, %5;\n\t"
            "fma.rn.bf16x2 %0, %2, %6, %0;\n\t"
            "fma.rn.bf16x2 %0, %3, %7, %0;\n\t"
            "fma.rn.bf16x2 %0, %4, %8, %0;\n\t}"
            : "=&r"(r[q])
            : "r"(v[0][q]), "r"(v[1][q]), "r"(v[2][q]), "r"(v[3][q]), "r"(w00), "r"(w01), "r"(w10), "r"(w11));
    }
}

// One neighbour's 16-channel slice. WIDE: a single 32-byte load from p;
// otherwise two 16-byte loads, the upper half from p_hi.
template <bool WIDE>
__device__ __forceinline__ void load_slice(uint32_t (&v)[8], const uint8_t* p, const uint8_t* p_hi) {
    if (WIDE) {
        ptx::ldg_v8(v, p);
    } else {
        const uint4 lo = ptx::ldg_v4(p), hi = ptx::ldg_v4(p_hi);
        v[0] = lo.x, v[1] = lo.y, v[2] = lo.z, v[3] = lo.w;
        v[4] = hi.x, v[5] = hi.y, v[6] = hi.z, v[7] = hi.w;
    }
}

// GEMM rows enumerate output pixels strip by strip: each image is cut into
// vertical strips sw pixels wide, rows of a strip are consecutive, so a tile of
// 128 rows covers a compact block of pixels whose bilinear neighbourhoods
// overlap in L1. Returns the raster index (b*Ho + ho)*Wo + wo, or -1 past the end.
__device__ __forceinline__ int strip_to_raster(int idx, const FwdArgs& a) {
    const Shape& s = a.s;
    if (idx >= s.P) return -1;
    const int plane = s.Ho * s.Wo;
    const int b = idx / plane;
    const int rem = idx - b * plane;
    const int full = a.nf * s.Ho * a.sw;
    int ho, wo;
    if (rem < full) {
        const int strip = rem / (s.Ho * a.sw);
        const int r2 = rem - strip * (s.Ho * a.sw);
        ho = r2 / a.sw;
        wo = strip * a.sw + (r2 - ho * a.sw);
    } else {
        const int r2 = rem - full;
        ho = r2 / a.wl;
        wo = a.nf * a.sw + (r2 - ho * a.wl);
    }
    return (b * s.Ho + ho) * s.Wo + wo;
}

// Partial tiles (float32) live in the workspace as [cta][slot][bn_total/32][8][BM][4]:
// slot 0 holds a CTA's first segment in unit order, slot 1 its last; within a tile, the four
// consecutive columns 4q..4q+3 of a 32-column block are stored for all 128
// rows side by side, so each warp-wide 16-byte access covers 512 contiguous bytes.
__device__ __forceinline__ const float* partial_base(const FwdArgs& a, const long long* starts, int c, long long tu0,
                                                    int row) {
    const int slot = (starts[c] >= tu0) ? 0 : 1;
    return a.partials + ((size_t)c * 2 + slot) * BM * a.bn_total + (size_t)row * 4;
}

// r[0..31] (float bits) += partial columns cc..cc+31 of this row (src from partial_base).
__device__ __forceinline__ void add_partial32(uint32_t (&r)[32], const float* src, int cc) {
    float4 f[8];
    const float* b = src + (size_t)(cc >> 5) * 8 * BM * 4;
#pragma unroll
    for (int q = 0; q < 8; ++q) f[q] = ptx::ldcg_f4(b + q * BM * 4);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        r[4 * q] = __float_as_uint(__uint_as_float(r[4 * q]) + f[q].x);
        r[4 * q + 1] = __float_as_uint(__uint_as_float(r[4 * q + 1]) + f[q].y);
        r[4 * q + 2] = __float_as_uint(__uint_as_float(r[4 * q + 2]) + f[q].z);
        r[4 * q + 3] = __float_as_uint(__uint_as_float(r[4 * q + 3]) + f[q].w);
    }
}

// As add_partial32, from a partial tile staged in shared memory.
__device__ __forceinline__ void add_partial32_smem(uint32_t (&r)[32], const float* src, int cc) {
    const float* b = src + (size_t)(cc >> 5) * 8 * BM * 4;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 f = *reinterpret_cast<const float4*>(b + q * BM * 4);
        r[4 * q] = __float_as_uint(__uint_as_float(r[4 * q]) + f.x);
        r[4 * q + 1] = __float_as_uint(__uint_as_float(r[4 * q + 1]) + f.y);
        r[4 * q + 2] = __float_as_uint(__uint_as_float(r[4 * q + 2]) + f.z);
        r[4 * q + 3] = __float_as_uint(__uint_as_float(r[4 * q + 3]) + f.w);
    }
}

// y[row, cc .. cc + 31] (columns < ncols of the tile) = r (float bits) + bias, as bf16;
// sb: the tile's bias in shared memory, or null. Overwrites r.
__device__ __forceinline__ void store_row32(bf16* yrow, int cc, int ncols, uint32_t (&r)[32], const float* sb) {
    if (sb) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 b = *reinterpret_cast<const float4*>(sb + cc + 4 * q);
            r[4 * q] = __float_as_uint(__uint_as_float(r[4 * q]) + b.x);
            r[4 * q + 1] = __float_as_uint(__uint_as_float(r[4 * q + 1]) + b.y);
            r[4 * q + 2] = __float_as_uint(__uint_as_float(r[4 * q + 2]) + b.z);
            r[4 * q + 3] = __float_as_uint(__uint_as_float(r[4 * q + 3]) + b.w);
        }
    }
    if (cc + 32 <= ncols) {
        uint4* dst = reinterpret_cast<uint4*>(yrow + cc);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t* w = r + 8 * q;
            dst[q] = make_uint4(pack_bf16(__uint_as_float(w[0]), __uint_as_float(w[1])),
                                pack_bf16(__uint_as_float(w[2]), __uint_as_float(w[3])),
                                pack_bf16(__uint_as_float(w[4]), __uint_as_float(w[5])),
                                pack_bf16(__uint_as_float(w[6]), __uint_as_float(w[7])));
        }
    } else {
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if (cc + e < ncols) yrow[cc + e] = __float2bfloat16_rn(__uint_as_float(r[e]));
    }
}

// As above for a float32 output row (no rounding): y[row, cc .. cc + 31] = r + bias.
__device__ __forceinline__ void store_row32(float* yrow, int cc, int ncols, uint32_t (&r)[32], const float* sb) {
    float v[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(r[e]) + (sb ? sb[cc + e] : 0.f);
    if (cc + 32 <= ncols) {
        float4* dst = reinterpret_cast<float4*>(yrow + cc);
#pragma unroll
        for (int q = 0; q < 8; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else {
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if (cc + e < ncols) yrow[cc + e] = v[e];
    }
}

// Walks this warp's 32 TMEM lanes over columns [0, ncols) in blocks of 32,
// calling f(r, cc) on each block; PIPE: while the next block's load is in
// flight (twice the registers). ncols is warp-uniform (the loads are
// warp-collective).
template <bool PIPE, typename F>
__device__ __forceinline__ void tmem_rows(uint32_t taddr, int ncols, F&& f) {
    if (!PIPE) {
        for (int cc = 0; cc < ncols; cc += 32) {
            uint32_t r[32];
            ptx::tmem_ld32_issue(taddr + cc, r);
            ptx::tmem_wait_ld(r);
            f(r, cc);
        }
        return;
    }
    uint32_t ra[32], rb[32];
    ptx::tmem_ld32_issue(taddr, ra);
    ptx::tmem_wait_ld(ra);
    for (int cc = 0; cc < ncols; cc += 64) {
        const bool has_b = cc + 32 < ncols;
        if (has_b) ptx::tmem_ld32_issue(taddr + cc + 32, rb);
        f(ra, cc);
        if (!has_b) break;
        ptx::tmem_wait_ld(rb);
        const bool has_a = cc + 64 < ncols;
        if (has_a) ptx::tmem_ld32_issue(taddr + cc + 64, ra);
        f(rb, cc + 32);
        if (has_a) ptx::tmem_wait_ld(ra);
    }
}

// y rows = bias + the tile's partial sums in contributor order c_lo..c_hi
// (columns [cc_begin, cc_end) of them),
// this CTA's own taken from its TMEM accumulator and every other one from
// `part(c)` (a row pointer in partial_base layout; in_smem: staged in shared
// memory). The fixed order makes the result independent of which CTA finishes
// the tile. Called by all 32 lanes of an epilogue warp (TMEM loads are
// warp-collective); lane l holds tile row warp*32 + l, whose output row is
// pr (-1: past the end). With a staging buffer (ybuf != 0: 32 rows x 128 B,
// 16-byte chunks swizzled by row) and a tile width that is a multiple of 64,
// every 64 columns of the warp's 32 rows go through it and leave as full
// 128-byte row segments, eight lanes per row; otherwise each lane stores its row.
// own_in_part: this CTA's own contribution is read back from part(cta) as
// well (its accumulator has already been released).
template <typename P, typename OutT>
__device__ __forceinline__ void combine_rows(uint32_t taddr, int ncols, int c_lo, int c_hi, int cta, bool in_smem,
                                             P&& part, const float* sb, uint32_t ybuf, OutT* ycol0, int pr,
                                             int ldy, int cc_begin = 0, int cc_end = 1 << 30,
                                             bool own_in_part = false) {
    const int lane = threadIdx.x & 31;
    // staged, coalesced stores for bf16 outputs (cc_begin must then be a multiple of 64)
    const bool coalesce = std::is_same<OutT, bf16>::value && ybuf != 0 && (ncols & 63) == 0;
    for (int cc = cc_begin; cc < min(ncols, cc_end); cc += 32) {
        uint32_t acc[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[e] = 0u;
        for (int c = c_lo; c < cta; ++c) {
            if (in_smem) add_partial32_smem(acc, part(c), cc);
            else add_partial32(acc, part(c), cc);
        }
        if (own_in_part) {
            add_partial32(acc, part(cta), cc);
        } else {
            uint32_t r[32];
            ptx::tmem_ld32_issue(taddr + cc, r);
            ptx::tmem_wait_ld(r);
#pragma unroll
            for (int e = 0; e < 32; ++e) acc[e] = __float_as_uint(__uint_as_float(acc[e]) + __uint_as_float(r[e]));
        }
        for (int c = cta + 1; c <= c_hi; ++c) {
            if (in_smem) add_partial32_smem(acc, part(c), cc);
            else add_partial32(acc, part(c), cc);
        }
        if (!coalesce) {
            if (pr >= 0) store_row32(ycol0 + (size_t)pr * ldy, cc, ncols, acc, sb);
            continue;
        }
        if constexpr (std::is_same<OutT, bf16>::value) {
            if (sb) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 b = *reinterpret_cast<const float4*>(sb + cc + 4 * q);
                    acc[4 * q] = __float_as_uint(__uint_as_float(acc[4 * q]) + b.x);
                    acc[4 * q + 1] = __float_as_uint(__uint_as_float(acc[4 * q + 1]) + b.y);
                    acc[4 * q + 2] = __float_as_uint(__uint_as_float(acc[4 * q + 2]) + b.z);
                    acc[4 * q + 3] = __float_as_uint(__uint_as_float(acc[4 * q + 3]) + b.w);
                }
            }
            const int h = (cc >> 5) & 1;  // which half of the 64-column group
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t* w = acc + 8 * j;
                ptx::sts_v4(ybuf + lane * 128 + (((4 * h + j) ^ (lane & 7)) << 4),
                            make_uint4(pack_bf16(__uint_as_float(w[0]), __uint_as_float(w[1])),
                                       pack_bf16(__uint_as_float(w[2]), __uint_as_float(w[3])),
                                       pack_bf16(__uint_as_float(w[4]), __uint_as_float(w[5])),
                                       pack_bf16(__uint_as_float(w[6]), __uint_as_float(w[7]))));
            }
            if (h == 1) {
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int rr = 4 * i + (lane >> 3), ch = lane & 7;
                    const uint4 v = ptx::lds_v4(ybuf + rr * 128 + ((ch ^ (rr & 7)) << 4));
                    const int prr = __shfl_sync(0xffffffffu, pr, rr);
                    if (prr >= 0) *reinterpret_cast<uint4*>(ycol0 + (size_t)prr * ldy + (cc - 32) + ch * 8) = v;
                }
                __syncwarp();
            }
        }
    }
}

// Barrier among the four epilogue warps (an mbarrier with a bounded wait).
__device__ __forceinline__ bool epi_sync(uint64_t* bar, uint32_t& ph, volatile int* abort, unsigned* status) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(ptx::smem_u32(bar));
    const bool ok = ptx::mbar_wait(ptx::smem_u32(bar), ph, abort, status, WAIT_LIMIT);
    ph ^= 1;
    return ok;
}

// Tile t -> (m tile, n tile); chunk u -> (group, channel chunk, tap).
struct Chunk {
    int g, q, tap;
};
__device__ __forceinline__ Chunk chunk_of(int u, const FwdArgs& a) {
    Chunk c;
    int per_g = a.nq * a.s.K2;
    c.g = u / per_g;
    int r = u - c.g * per_g;
    c.q = r / a.s.K2;
    c.tap = r - c.q * a.s.K2;
    return c;
}

// The sampling record of tile row `row`, tap `tp`, group g of m-tile mt (as
// build_records below computes it), for a pre-pass that writes all of them.
__device__ __forceinline__ TapRec record_at(const FwdArgs& a, int mt, int g, int row, int tp) {
    const Shape& s = a.s;
    const int plane = s.Ho * s.Wo;
    const int pr = strip_to_raster(mt * BM + row, a);
    TapRec rc;
    rc.w01_00 = rc.w11_10 = 0u;
    rc.base = 0;
    rc.vmask = 0u;
    if (pr < 0) return rc;
    const int bb = pr / plane, pix = pr - bb * plane;
    const int ho = pix / s.Wo, wo = pix - ho * s.Wo;
    const int i = tp / s.K, j = tp - i * s.K;
    const bf16* offp = a.off + ((size_t)bb * 2 * s.G * s.K2 + (size_t)g * 2 * s.K2 + 2 * tp) * plane + pix;
    const float dy = __bfloat162float(offp[0]), dx = __bfloat162float(offp[plane]);
    const float mk = a.mask ? __bfloat162float(a.mask[((size_t)bb * s.G * s.K2 + (size_t)g * s.K2 + tp) * plane + pix])
                            : 1.f;
    int y0, x0;
    float ly, lx;
    split_coord(ho * s.stride - s.pad + i * s.dil, dy, y0, ly);
    split_coord(wo * s.stride - s.pad + j * s.dil, dx, x0, lx);
    const bool v00 = inside(s, y0, x0), v01 = inside(s, y0, x0 + 1);
    const bool v10 = inside(s, y0 + 1, x0), v11 = inside(s, y0 + 1, x0 + 1);
    rc.w01_00 = pack_bf16(v00 ? (1.f - ly) * (1.f - lx) * mk : 0.f, v01 ? (1.f - ly) * lx * mk : 0.f);
    rc.w11_10 = pack_bf16(v10 ? ly * (1.f - lx) * mk : 0.f, v11 ? ly * lx * mk : 0.f);
    if (v00 | v01 | v10 | v11) rc.base = (bb * s.H + y0) * s.W + x0;
    rc.vmask = ((rc.w01_00 & 0x7FFFu) ? 1u : 0u) | ((rc.w01_00 & 0x7FFF0000u) ? 2u : 0u) |
               ((rc.w11_10 & 0x7FFFu) ? 4u : 0u) | ((rc.w11_10 & 0x7FFF0000u) ? 8u : 0u);
    return rc;
}

// Sampling records of tile row `row` for the taps of `part` (0..2: a third of
// the taps each; -1: all), for group g of m-tile mt:
// offsets and mask of the row's output pixel, split into integer corner and
// fractional weights (the bilinear kernel of the DCNv2 sampling equation, a
// neighbour outside the map contributing zero), written to recs[row*K2 + tap].
// The loads of up to REC_BATCH taps are in flight together.
constexpr int REC_BATCH = 9;
__device__ __forceinline__ void build_records(const FwdArgs& a, int mt, int g, int row, int part, TapRec* recs,
                                              const int2* s_tap) {
    const Shape& s = a.s;
    const int plane = s.Ho * s.Wo;
    const int pr = strip_to_raster(mt * BM + row, a);
    int pix = -1, bb = 0, oy = 0, ox = 0;
    if (pr >= 0) {
        bb = pr / plane;
        pix = pr - bb * plane;
        const int ho = pix / s.Wo, wo = pix - ho * s.Wo;
        oy = ho * s.stride - s.pad;
        ox = wo * s.stride - s.pad;
    }
    const bf16* offp = a.off + ((size_t)bb * 2 * s.G * s.K2 + (size_t)g * 2 * s.K2) * plane + (pix < 0 ? 0 : pix);
    const bf16* mp = a.mask ? a.mask + ((size_t)bb * s.G * s.K2 + (size_t)g * s.K2) * plane + (pix < 0 ? 0 : pix) : nullptr;
    const int tp_lo = part < 0 ? 0 : s.K2 * part / 3, tp_hi = part < 0 ? s.K2 : s.K2 * (part + 1) / 3;
    for (int tp0 = tp_lo; tp0 < tp_hi; tp0 += REC_BATCH) {
        float dy[REC_BATCH], dx[REC_BATCH], mk[REC_BATCH];
#pragma unroll
        for (int b = 0; b < REC_BATCH; ++b) {
            const int tp = tp0 + b;
            dy[b] = dx[b] = 0.f;
            mk[b] = 1.f;
            if (pix >= 0 && tp < tp_hi) {
                dy[b] = __bfloat162float(offp[(size_t)(2 * tp) * plane]);
                dx[b] = __bfloat162float(offp[(size_t)(2 * tp + 1) * plane]);
                if (mp) mk[b] = __bfloat162float(mp[(size_t)tp * plane]);
            }
        }
#pragma unroll
        for (int b = 0; b < REC_BATCH; ++b) {
            const int tp = tp0 + b;
            if (tp >= tp_hi) break;
            float w00 = 0.f, w01 = 0.f, w10 = 0.f, w11 = 0.f;
            int base = 0;
            if (pix >= 0) {
                const int2 to = s_tap[tp];
                int y0, x0;
                float ly, lx;
                split_coord(oy + to.x, dy[b], y0, ly);
                split_coord(ox + to.y, dx[b], x0, lx);
                const bool v00 = inside(s, y0, x0), v01 = inside(s, y0, x0 + 1);
                const bool v10 = inside(s, y0 + 1, x0), v11 = inside(s, y0 + 1, x0 + 1);
                w00 = v00 ? (1.f - ly) * (1.f - lx) * mk[b] : 0.f;
                w01 = v01 ? (1.f - ly) * lx * mk[b] : 0.f;
                w10 = v10 ? ly * (1.f - lx) * mk[b] : 0.f;
                w11 = v11 ? ly * lx * mk[b] : 0.f;
                if (v00 | v01 | v10 | v11) base = (bb * s.H + y0) * s.W + x0;
            }
            TapRec rc;
            rc.w01_00 = pack_bf16(w00, w01);
            rc.w11_10 = pack_bf16(w10, w11);
            rc.base = base;
            // read a neighbour only when it is inside the map and its bf16 weight is nonzero
            rc.vmask = ((rc.w01_00 & 0x7FFFu) ? 1u : 0u) | ((rc.w01_00 & 0x7FFF0000u) ? 2u : 0u) |
                       ((rc.w11_10 & 0x7FFFu) ? 4u : 0u) | ((rc.w11_10 & 0x7FFF0000u) ? 8u : 0u);
            recs[row * s.K2 + tp] = rc;
        }
    }
}

// ------------------------------------------------------------------- host --

// The stream-K split shared by the forward kernels: tiles of BM output pixels x
// bn_total output channels, units of one (group, 64-channel chunk, tap) each,
// divided over at most `sms` persistent CTAs, and the vertical-strip pixel order.
struct StreamK {
    int n_tiles, m_tiles, tiles, nq, U, ctas, sw, nf, wl, snap;
    long long total_units;
};

inline StreamK plan_stream_k(const Shape& s, int bn_total, int sms) {
    StreamK k{};
    k.n_tiles = (s.Cout + bn_total - 1) / bn_total;
    k.m_tiles = (s.P + BM - 1) / BM;
    k.tiles = k.m_tiles * k.n_tiles;
    k.nq = (s.Cg + BK - 1) / BK;
    // strip width: a divisor of Wo in [8, 16] if there is one, else 12 (or Wo when narrower)
    k.sw = std::min(s.Wo, 12);
    if (s.Wo > 16) {
        for (int c = 8; c <= 16; ++c)
            if (s.Wo % c == 0) k.sw = c;
    }
    k.nf = s.Wo / k.sw;
    k.wl = s.Wo - k.nf * k.sw;
    k.U = s.G * k.nq * s.K2;
    k.total_units = (long long)k.tiles * k.U;
    k.ctas = (int)std::min<long long>(std::min(sms, MAX_CTAS), k.total_units);
    // Snap starts away from a tile's last units when CTAs get at least 12 units
    // each. A share of n units, U <= n < 2U, spans three tiles when fewer than
    // n - U of them fall in its first tile, so snap at least that far; a CTA
    // whose successor was snapped ends on a tile boundary and spans two tiles.
    const long long per = (k.total_units + k.ctas - 1) / k.ctas;
    k.snap = 0;
    if (k.U >= 4 && k.total_units / k.ctas >= 12) {
        long long sn = 3;
        if (per >= k.U && per < 2 * k.U) sn = std::max<long long>(sn, per - k.U + 1);
        k.snap = (int)std::min<long long>(sn, k.U / 2);
    }
    return k;
}

inline PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

}  // namespace
}  // namespace dcn
