// Weight-side backward of DCNv2 on sm_100a tensor cores (bfloat16 in, float32
// out): grad_W[o, kc] = sum_p grad_y[p, o] * col[p, kc], with col[p, kc] the
// modulated bilinear sample m * x(p0 + p_k + dp_k) of the forward (the same
// im2col view of the layer; the column is regenerated, never stored in HBM).
//
// The contraction runs over output pixels, so both operands are MN-major:
//   A = grad_y^T [o x p]: TMA boxes of 64 o x 64 pixels from grad_y [P, Cout];
//   B = col^T [kc x p]: producer warps gather 64 pixels x 256 channels of one
//       (group, tap) per chunk into the UMMA 128-byte-swizzle MN-major layout.
// One CTA per SM walks a contiguous range of (N tile, 64-pixel chunk) units; an
// N tile is 256 channels of one (group, tap), two M=128 accumulators in TMEM
// cover up to 256 output channels. At the end of each range segment the
// epilogue adds its float32 partial into grad_W with vector atomics (grad_W is
// zeroed first). The sampling records of every (pixel, group, tap) come from a
// small pre-pass, stored tap-major so a chunk's 64 records are one 1 KB bulk
// copy staged by the TMA warp. All waits are bounded.
#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.h"
#include "tc_ptx.cuh"

namespace dcn {
namespace {

constexpr int BKP = 64;     // pixels per K chunk
constexpr int MH = 128;     // output channels per accumulator (UMMA M)
constexpr int NT = 256;     // input-channel columns per N tile (UMMA N)
constexpr int NUM_PROD_WARPS = 8;
constexpr int TMA_WARP = 4, MMA_WARP = 5, PROD_WARP0 = 6;  // warps 0-3: epilogue
constexpr int NUM_THREADS = (PROD_WARP0 + NUM_PROD_WARPS) * 32;
constexpr int GROUPS = 2;                                  // producer groups taking alternate chunks
constexpr int GROUP_WARPS = NUM_PROD_WARPS / GROUPS;
constexpr long long WAIT_LIMIT = 2000000000LL;
constexpr int MAX_STAGES = 4;
constexpr uint32_t MN_BLOCK = BKP * 128;                   // one 64-wide MN block of 64 K rows: 8 KB
constexpr uint32_t B_BYTES = (NT / 64) * MN_BLOCK;         // 32 KB
constexpr uint32_t R_BYTES = BKP * 16;                     // 64 sampling records

struct BwArgs {
    Shape s;
    const bf16* x;
    const uint4* rec;  // sampling records [G*K2][Ppad]: {w01_00, w11_10, base, 0}
    float* gw;
    unsigned* status;
    int nblk;          // 256-channel blocks per group
    int n_tiles, chunks, ppad, m_halves;
    long long total_units;
    int ctas, stages;
    uint32_t a_bytes, stage_bytes, bar_off;
};

__device__ __forceinline__ long long unit_begin(int c, const BwArgs& a) { return a.total_units * c / a.ctas; }

// Shared-memory descriptor of an MN-major operand in the 128-byte-swizzle
// canonical layout: rows of 128 B hold 64 consecutive MN elements of one K
// index, groups of 8 K rows are 1024 B apart (stride byte offset), and 64-wide
// MN blocks are `lbo` bytes apart (leading byte offset).
__device__ __forceinline__ uint64_t mn_sw128_desc(uint32_t saddr, uint32_t lbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// kind::f16 instruction descriptor, bf16 A and B both MN-major, f32 D.
__host__ __device__ constexpr uint32_t idesc_mn(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ uint4 blend_bf16x2(const uint4 (&v)[4], uint32_t w01_00, uint32_t w11_10) {
    const uint32_t w00 = __byte_perm(w01_00, 0, 0x1010), w01 = __byte_perm(w01_00, 0, 0x3232);
    const uint32_t w10 = __byte_perm(w11_10, 0, 0x1010), w11 = __byte_perm(w11_10, 0, 0x3232);
    const uint32_t* a0 = reinterpret_cast<const uint32_t*>(&v[0]);
    const uint32_t* a1 = reinterpret_cast<const uint32_t*>(&v[1]);
    const uint32_t* a2 = reinterpret_cast<const uint32_t*>(&v[2]);
    const uint32_t* a3 = reinterpret_cast<const uint32_t*>(&v[3]);
    uint32_t r[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        asm("{\n\t"
            "mul.rn.bf16x2 %0, %1, %5;\n\t"
            "fma.rn.bf16x2 %0, %2, %6, %0;\n\t"
            "fma.rn.bf16x2 %0, %3, %7, %0;\n\t"
            "fma.rn.bf16x2 %0, %4, %8, %0;\n\t}"
            : "=&r"(r[q])
            : "r"(a0[q]), "r"(a1[q]), "r"(a2[q]), "r"(a3[q]), "r"(w00), "r"(w01), "r"(w10), "r"(w11));
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    dcn_bwd_weight_tc_kernel(const __grid_constant__ CUtensorMap tmap_dy, const BwArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Shape& s = a.s;
    // stage layout: [A: m_halves*2 MN blocks][B: 4 MN blocks][R: 64 records]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.bar_off);
    uint64_t* full_t = bars;                   // TMA: A + records
    uint64_t* full_b = bars + MAX_STAGES;      // producers: B
    uint64_t* empty = bars + 2 * MAX_STAGES;   // MMA done with the stage
    uint64_t* acc_full = bars + 3 * MAX_STAGES;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* drain = acc_empty + 1;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.stages; ++i) {
            ptx::mbar_init(ptx::smem_u32(&full_t[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&full_b[i]), GROUP_WARPS);
            ptx::mbar_init(ptx::smem_u32(&empty[i]), 1);
        }
        ptx::mbar_init(ptx::smem_u32(acc_full), 1);
        ptx::mbar_init(ptx::smem_u32(acc_empty), 4);
        ptx::mbar_init(ptx::smem_u32(drain), 1);
        *s_abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == MMA_WARP) {
        ptx::tmem_alloc(ptx::smem_u32(s_tmem), 512);
        ptx::tmem_relinquish();
    }
    if (warp == TMA_WARP && lane == 0) ptx::prefetch_tmap(&tmap_dy);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const long long ubeg = unit_begin(blockIdx.x, a), uend = unit_begin(blockIdx.x + 1, a);
    // launched as a programmatic dependent of the records kernel (which the weight warp
    // waits for below); a bias-gradient kernel after this one may start alongside
    asm volatile("griddepcontrol.launch_dependents;");

    if (warp >= PROD_WARP0) {
        // ------------------------------------------------------ producers --
        // Each warp of a group gathers whole pixel rows: lane j takes channels
        // 8j..8j+7 of the 256-channel block (16 bytes of each neighbour).
        const int ptid = threadIdx.x - PROD_WARP0 * 32;
        const int grp = ptid / (GROUP_WARPS * 32);
        const int wg = (ptid / 32) % GROUP_WARPS;
        const int j = lane;
        int stage = 0;
        uint32_t phase = 0;
        int n = 0;
        bool ok = true;
        for (long long u = ubeg; u < uend && ok; ++u, ++n) {
            if ((n % GROUPS) == grp) {
                const int nt = (int)(u / a.chunks), pc = (int)(u - (long long)nt * a.chunks);
                const int gtap = nt / a.nblk, cb = nt - gtap * a.nblk;
                const int g = gtap / s.K2;
                const int cgrp = cb * NT + j * 8;  // channel within the group
                const bool cval = cgrp < s.Cg;
                const bf16* xc = a.x + g * s.Cg + cgrp;
                const long long rowpitch = (long long)s.W * s.Cin;
                if (!ptx::mbar_wait(ptx::smem_u32(&empty[stage]), phase ^ 1, s_abort, a.status, WAIT_LIMIT) ||
                    !ptx::mbar_wait(ptx::smem_u32(&full_t[stage]), phase, s_abort, a.status, WAIT_LIMIT)) {
                    ok = false;
                    break;
                }
                uint8_t* st = smem + stage * a.stage_bytes;
                const uint4* rec = reinterpret_cast<const uint4*>(st + a.a_bytes + B_BYTES);
                const uint32_t b0 = ptx::smem_u32(st + a.a_bytes);
                const uint32_t mb = (uint32_t)(j >> 3), ch16 = (uint32_t)(j & 7);
#pragma unroll 1
                for (int bt = 0; bt < BKP / GROUP_WARPS / 4; ++bt) {
                    uint4 v[4][4];
                    uint4 r[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int k = wg + GROUP_WARPS * (4 * bt + i);  // pixel within the chunk
                        r[i] = rec[k];
                        const bf16* pb = xc + (long long)(int)r[i].z * s.Cin;
                        uint32_t m = ((r[i].x & 0xFFFFu) ? 1u : 0u) | ((r[i].x >> 16) ? 2u : 0u) |
                                     ((r[i].y & 0xFFFFu) ? 4u : 0u) | ((r[i].y >> 16) ? 8u : 0u);
                        if (!cval) m = 0;
#ifdef DCN_CHECKED
                        {  // range-checked build: a neighbour load outside x is skipped (zeros) and recorded
                            const size_t xbytes = (size_t)s.B * s.H * s.W * s.Cin * sizeof(bf16);
                            const bf16* q[4] = {pb, pb + s.Cin, pb + rowpitch, pb + rowpitch + s.Cin};
                            for (int c = 0; c < 4; ++c)
                                if (((m >> c) & 1u) && !ptx::in_range(q[c], 16, a.x, xbytes, a.status)) m &= ~(1u << c);
                        }
#endif
                        ptx::ldg4_pred(v[i], pb, pb + s.Cin, pb + rowpitch, pb + rowpitch + s.Cin, m);
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int k = wg + GROUP_WARPS * (4 * bt + i);
                        const uint32_t addr = b0 + mb * MN_BLOCK + (uint32_t)(k >> 3) * 1024u +
                                              (uint32_t)(k & 7) * 128u + ((ch16 ^ (uint32_t)(k & 7)) << 4);
                        ptx::sts_v4(addr, blend_bf16x2(v[i], r[i].x, r[i].y));
                    }
                }
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&full_b[stage]));
            }
            if (++stage == a.stages) {
                stage = 0;
                phase ^= 1;
            }
        }
    } else if (warp == TMA_WARP) {
        // ------------------------------------------ grad_y tiles + records --
        asm volatile("griddepcontrol.wait;" ::: "memory");  // the records are written
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, issued = 0, issued_par = 0;
            const uint32_t bytes = a.a_bytes + R_BYTES;
            bool ok = true;
            for (long long u = ubeg; u < uend && ok; ++u) {
                const int nt = (int)(u / a.chunks), pc = (int)(u - (long long)nt * a.chunks);
                const int gtap = nt / a.nblk;
                if (!ptx::mbar_wait(ptx::smem_u32(&empty[stage]), phase ^ 1, s_abort, a.status, WAIT_LIMIT)) {
                    ok = false;
                    break;
                }
                uint8_t* st = smem + stage * a.stage_bytes;
                const uint32_t fb = ptx::smem_u32(&full_t[stage]);
                ptx::mbar_arrive_expect_tx(fb, bytes);
                for (int ob = 0; ob < 2 * a.m_halves; ++ob)
                    ptx::tma_load_2d(ptx::smem_u32(st + ob * MN_BLOCK), &tmap_dy, fb, ob * 64, pc * BKP);
                ptx::bulk_load(ptx::smem_u32(st + a.a_bytes + B_BYTES),
                               a.rec + (size_t)gtap * a.ppad + (size_t)pc * BKP, R_BYTES, fb);
                issued |= 1u << stage;
                issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                if (++stage == a.stages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            if (*s_abort) {
                volatile int dummy = 0;
                for (int i = 0; i < a.stages; ++i)
                    if ((issued >> i) & 1u)
                        ptx::mbar_wait(ptx::smem_u32(&full_t[i]), (issued_par >> i) & 1u, &dummy, nullptr,
                                       WAIT_LIMIT);
            }
        }
        __syncwarp();
    } else if (warp == MMA_WARP) {
        // ----------------------------------------------------------- MMA --
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, aphase = 0;
            const uint32_t idesc = idesc_mn(MH, NT);
            const uint32_t s0 = ptx::smem_u32(smem);
            bool ok = true;
            for (long long u = ubeg; u < uend && ok;) {
                const int nt = (int)(u / a.chunks);
                const long long seg_end = min(uend, (long long)(nt + 1) * a.chunks);
                if (!ptx::mbar_wait(ptx::smem_u32(acc_empty), aphase ^ 1, s_abort, a.status, WAIT_LIMIT)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                for (long long v = u; v < seg_end; ++v) {
                    if (!ptx::mbar_wait(ptx::smem_u32(&full_t[stage]), phase, s_abort, a.status, WAIT_LIMIT) ||
                        !ptx::mbar_wait(ptx::smem_u32(&full_b[stage]), phase, s_abort, a.status, WAIT_LIMIT)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t st = s0 + stage * a.stage_bytes;
#pragma unroll
                    for (int ks = 0; ks < BKP / 16; ++ks) {
                        const uint32_t acc = (v > u || ks > 0) ? 1u : 0u;
                        const uint64_t bdesc = mn_sw128_desc(st + a.a_bytes + ks * 2048u, MN_BLOCK);
                        for (int h = 0; h < a.m_halves; ++h)
                            ptx::mma_bf16(tmem_base + (uint32_t)(h * NT),
                                          mn_sw128_desc(st + h * 2 * MN_BLOCK + ks * 2048u, MN_BLOCK), bdesc, idesc,
                                          acc);
                    }
                    ptx::mma_commit(ptx::smem_u32(&empty[stage]));
                    if (++stage == a.stages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                ptx::mma_commit(ptx::smem_u32(acc_full));
                aphase ^= 1;
                u = seg_end;
            }
            ptx::mma_commit(ptx::smem_u32(drain));
            volatile int dummy = 0;
            ptx::mbar_wait(ptx::smem_u32(drain), 0, &dummy, a.status, WAIT_LIMIT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ epilogue --
        // Lane = output channel o within its accumulator; add the partial row of
        // this segment into grad_W[o, tap*Cin + g*Cg + cb*256 + c].
        const int quarter = warp & 3;
        uint32_t aphase = 0;
        bool ok = true;
        for (long long u = ubeg; u < uend && ok;) {
            const int nt = (int)(u / a.chunks);
            const long long seg_end = min(uend, (long long)(nt + 1) * a.chunks);
            if (!ptx::mbar_wait(ptx::smem_u32(acc_full), aphase, s_abort, a.status, WAIT_LIMIT)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const int gtap = nt / a.nblk, cb = nt - gtap * a.nblk;
            const int g = gtap / s.K2, tap = gtap - g * s.K2;
            const int c0 = cb * NT;
            const int ncols = min(NT, s.Cg - c0);
            for (int h = 0; h < a.m_halves; ++h) {
                const int o = h * MH + quarter * 32 + lane;
                float* dst = a.gw + (size_t)o * s.KC + (size_t)tap * s.Cin + g * s.Cg + c0;
                const uint32_t taddr = tmem_base + (uint32_t)(h * NT) + ((uint32_t)(quarter * 32) << 16);
                for (int cc = 0; cc < NT; cc += 32) {
                    float v[32];
                    ptx::tmem_ld32(taddr + cc, v);
                    if (o < s.Cout && cc < ncols) {
                        if (cc + 32 <= ncols) {
#pragma unroll
                            for (int q = 0; q < 8; ++q) ptx::red_add_v4(dst + cc + 4 * q, v[4 * q], v[4 * q + 1],
                                                                         v[4 * q + 2], v[4 * q + 3]);
                        } else {
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (cc + e < ncols) atomicAdd(dst + cc + e, v[e]);
                        }
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(acc_empty));
            aphase ^= 1;
            u = seg_end;
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, 512);
    }
}

// Sampling records [G*K2][Ppad]: for every (group, tap) and output pixel, the
// four bilinear weights times the mask as bf16 (zero for neighbours outside the
// map) and the pixel index of the top-left neighbour; zero past the last pixel.
__global__ void __launch_bounds__(256) dcn_records_kernel(Shape s, const bf16* __restrict__ off,
                                                          const bf16* __restrict__ mask, uint4* __restrict__ rec,
                                                          int ppad) {
    // the main kernel may start: it reads the records only after a griddepcontrol.wait
    asm volatile("griddepcontrol.launch_dependents;");
    const int p = blockIdx.x * blockDim.x + threadIdx.x;
    const int gt = blockIdx.y;
    if (p >= ppad) return;
    uint4 r = make_uint4(0, 0, 0, 0);
    if (p < s.P) {
        const int g = gt / s.K2, tap = gt - g * s.K2;
        TapSample t = tap_sample(s, off, mask, p, g, tap);
        const bool v00 = inside(s, t.y0, t.x0), v01 = inside(s, t.y0, t.x0 + 1);
        const bool v10 = inside(s, t.y0 + 1, t.x0), v11 = inside(s, t.y0 + 1, t.x0 + 1);
        const float w00 = v00 ? (1.f - t.ly) * (1.f - t.lx) * t.m : 0.f;
        const float w01 = v01 ? (1.f - t.ly) * t.lx * t.m : 0.f;
        const float w10 = v10 ? t.ly * (1.f - t.lx) * t.m : 0.f;
        const float w11 = v11 ? t.ly * t.lx * t.m : 0.f;
        __nv_bfloat162 a = __floats2bfloat162_rn(w00, w01), b = __floats2bfloat162_rn(w10, w11);
        r.x = *reinterpret_cast<uint32_t*>(&a);
        r.y = *reinterpret_cast<uint32_t*>(&b);
        r.z = (v00 | v01 | v10 | v11) ? (uint32_t)((t.b * s.H + t.y0) * s.W + t.x0) : 0u;
    }
    rec[(size_t)gt * ppad + p] = r;
}

struct BwPlan {
    bool ok;
    int nblk, n_tiles, chunks, ppad, m_halves, ctas, stages;
    long long total_units;
    uint32_t a_bytes, stage_bytes, bar_off, smem_bytes;
    size_t rec_bytes;
};

BwPlan make_bw_plan(const Shape& s, int sms) {
    BwPlan pl{};
    if (s.Cin % 8 || s.Cg % 8 || s.Cout % 8 || s.Cout > 2 * MH) return pl;
    pl.nblk = (s.Cg + NT - 1) / NT;
    pl.n_tiles = s.G * s.K2 * pl.nblk;
    pl.chunks = (s.P + BKP - 1) / BKP;
    pl.ppad = pl.chunks * BKP;
    pl.m_halves = (s.Cout + MH - 1) / MH;
    pl.total_units = (long long)pl.n_tiles * pl.chunks;
    pl.ctas = (int)std::min<long long>(sms, pl.total_units);
    pl.a_bytes = (uint32_t)(2 * pl.m_halves) * MN_BLOCK;
    pl.stage_bytes = (pl.a_bytes + B_BYTES + R_BYTES + 1023) & ~1023u;
    const uint32_t budget = 227 * 1024;
    int st = (int)((budget - 2048) / pl.stage_bytes);
    st = std::min(st, 3);
    if (st < 2) return pl;
    pl.stages = st;
    pl.bar_off = (uint32_t)st * pl.stage_bytes;
    pl.smem_bytes = pl.bar_off + (3 * MAX_STAGES + 3) * 8 + 16 + 1024;
    pl.rec_bytes = (size_t)s.G * s.K2 * pl.ppad * sizeof(uint4);
    if ((long long)s.B * s.H * s.W < (1LL << 31) && pl.smem_bytes <= budget) pl.ok = true;
    return pl;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

bool bwd_weight_tc_supported(const Shape& s) { return make_bw_plan(s, num_sms()).ok; }

size_t bwd_weight_tc_workspace(const Shape& s) {
    BwPlan pl = make_bw_plan(s, num_sms());
    return pl.ok ? pl.rec_bytes : 0;
}

cudaError_t bwd_weight_tc(const Shape& s, const void* x, const void* off, const void* mask, const void* gy,
                          float* gw, void* ws, size_t ws_bytes, unsigned* status, cudaStream_t st, int* launches) {
    BwPlan pl = make_bw_plan(s, num_sms());
    if (!pl.ok || !ws || ws_bytes < pl.rec_bytes) return cudaErrorInvalidValue;
    auto encode = encode_fn();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap map;
    cuuint64_t dims[2] = {(cuuint64_t)s.Cout, (cuuint64_t)s.P};
    cuuint64_t strides[1] = {(cuuint64_t)s.Cout * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)BKP};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(gy), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    static DeviceFlags attr_set;
    cudaError_t e = max_dynamic_smem_once((const void*)dcn_bwd_weight_tc_kernel, 227 * 1024, attr_set);
    if (e != cudaSuccess) return e;
    uint4* rec = reinterpret_cast<uint4*>(ws);
    e = cudaMemsetAsync(gw, 0, sizeof(float) * (size_t)s.Cout * s.KC, st);
    if (e != cudaSuccess) return e;
    dim3 rg((pl.ppad + 255) / 256, s.G * s.K2);
    dcn_records_kernel<<<rg, 256, 0, st>>>(s, (const bf16*)off, (const bf16*)mask, rec, pl.ppad);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    BwArgs a;
    a.s = s;
    a.x = (const bf16*)x;
    a.rec = rec;
    a.gw = gw;
    a.status = status;
    a.nblk = pl.nblk;
    a.n_tiles = pl.n_tiles;
    a.chunks = pl.chunks;
    a.ppad = pl.ppad;
    a.m_halves = pl.m_halves;
    a.total_units = pl.total_units;
    a.ctas = pl.ctas;
    a.stages = pl.stages;
    a.a_bytes = pl.a_bytes;
    a.stage_bytes = pl.stage_bytes;
    a.bar_off = pl.bar_off;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)pl.ctas);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = pl.smem_bytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, dcn_bwd_weight_tc_kernel, map, a);
    if (e != cudaSuccess) return e;
    if (launches) *launches += 3;
    return cudaGetLastError();
}

}  // namespace dcn
