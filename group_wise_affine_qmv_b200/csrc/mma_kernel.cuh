// mma_kernel.cuh -- tensor-core kernel for y = x . dequant(W)^T on sm_100a (tcgen05 / TMEM).
//
// Arithmetic (exact up to fp32 summation order).  With codes q, per-group scale s and bias b
// (w = s*q + b), each output is
//     y[n, t] = sum_g  s[n,g] * D_g[n, t]  +  b[n,g] * X_g[t],
//     D_g[n, t] = sum_{k in g} q[n, k] * x[t, k],    X_g[t] = sum_{k in g} x[t, k].
// The tensor core computes D_g with integer codes as its A operand, one fresh fp32
// accumulator per group; X_g is summed from x widened to fp32 before any addition ("mlx PR
// #4516", load_vector fix).  With bf16 activations and codes below 128 the A operand holds
// 128 + q (exact in bf16), which one OR per pair of codes produces, and the fold uses
// b - 128*s in place of b, since sum_k (128 + q) x = D + 128 * X; the extra fp32 accumulation
// error this brings is ~1e-5 of max|y|.  8-bit codes with bf16, and every width with f16
// (where the offset would be 1024), are converted to exact integers (OFF = 0).  The weights
// are never rounded: rounding s*q + b to bf16 would cost ~2e-3 of max|y| on its own.
//
// "Weights-stationary" tiles: 128 rows of W are the MMA's M side, 32 tokens its N side.  The
// pipeline advances one W stage at a time (128 rows x WSC codes, a 32..128-byte TMA row) and
// every hand-off between roles happens once per stage:
//   warp 0       W producer: TMA of each W stage onto wfull[s] (ring of up to 12).
//   warp 18      x producer: the CTA's token tile once (resident x), or per W stage its x
//                block (SUB boxes of [32 x 64], 128-byte swizzle, the UMMA B operand) onto a
//                ring of up to 4 x stages.
//   warp 1       MMA issuer: waits for the expanded codes of stage i (afull) and for its
//                accumulators to be free (dfree), issues SUB*4 tcgen05.mma kind::f16 with A
//                from tensor memory (one fresh accumulator per group, compile-time offsets and
//                accumulate flags), and one tcgen05.commit (sdone[i % 2]; a second commit frees
//                a streamed x stage).
//   warps 2..9   code expanders: thread <-> W row (TMEM lane), two warps per lane quarter
//                split each 64 codes.  Stage i goes into A block i % 2 once the MMAs of stage
//                i - 2 are complete; then wfree (shared-memory stage) and afull.
//   warps 10..17 folds: thread <-> W row, two warps per lane quarter take 16 tokens each.
//                Per stage, y += s*D' + (b - OFF*s)*X per group (tcgen05.ld of D), then dfree;
//                per tile, the store of y: with 16-byte aligned rows of y and N a multiple of
//                8 (ytma) the fold
//                threads write the tile into shared memory and one of them stores it with one
//                bulk tensor copy (element-wise 2-byte stores of scattered rows of y held the
//                folds ~1.3 us per tile and with them the next tile's MMAs), else element stores.
// Tensor memory: [A block 0 | A block 1 | D: 2 x GPS group accumulators of 32 columns].
//
// Rows of the last W tile that fall past N read TMA zero fill and the clamped last row's
// scale/bias and are simply not stored: no per-row check inside the K loop (the
// partial-rows idea of "mlx PR #4516").
//
// Every mbarrier wait is bounded (2 s); on expiry the CTA raises an abort flag, records an
// error word readable through aq_device_error(), drains its own outstanding copies and MMAs
// (bounded), frees its tensor memory and exits.
#pragma once

#include <mutex>
#include <type_traits>

#include "aq_internal.h"
#include "device_common.cuh"
#include "mma_common.cuh"
#include "sm100_ptx.cuh"

namespace aq {
namespace mma {

__device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

// Grouped mode: rows [*off, *off + *cnt) of x_sorted / y_sorted belong to expert e.  The device
// offsets are clamped into [0, M] and each end to at least its start, so no offsets array, however
// malformed, makes a CTA read or write a row outside the M rows of the call.
__device__ __forceinline__ void expert_rows(const Params& p, int e, int64_t* off, int64_t* cnt) {
    const int64_t lo = min64(max64(p.offsets[e], 0), p.M);
    const int64_t hi = min64(max64(p.offsets[e + 1], lo), p.M);
    *off = lo;
    *cnt = hi - lo;
}

struct TileInfo {
    int64_t wrow0;   // first W row of the tile in the W tensor (expert offset included)
    int64_t n0;      // first output column (row of W within the expert / matrix)
    int nvalid;      // valid W rows in this tile
    int64_t xrow0;   // first x row (token) of the tile within its batch / the sorted rows
    int tvalid;      // valid tokens in this tile
    int b0, b1;      // launch batch (non-grouped)
};

struct Smem {
    uint64_t* wfull;     // [MAX_STAGES] W stage landed (TMA)
    uint64_t* wfree;     // [MAX_STAGES] W stage read by the expander warps
    uint64_t* xfull;     // [MAX_XST] streamed x stage landed (TMA)
    uint64_t* xfree;     // [MAX_XST] streamed x stage read by its MMAs (commit)
    uint64_t* afull;     // [2] A block written (expander warps)
    uint64_t* sdone;     // [2] MMAs of a W stage complete (commit)
    uint64_t* dfree;     // [2] group accumulators of a W stage read (fold warps)
    uint64_t* sbar;      // [2] scale/bias chunk slots (fold threads)
    uint64_t* xbar;      // sum-of-x table (fold threads)
    uint64_t* xres_full; // resident x landed
    uint64_t* mdone;     // teardown: all MMAs retired
    uint64_t* red_full;  // split K: every rank's part of this CTA's rows has arrived (fold warps)
    uint64_t* ybar;      // ytma: the staged y tile is written (fold threads)
    uint32_t* tmem_base;
    int* abort;
    int* prefix;         // grouped: tile prefix sums [n_experts + 1]
    float* xtab;         // [groups of this CTA's K range][NT] sums of x per group and token
    float* red;          // split K: partial sums of this CTA's rows [ranks][128 / ranks][NT] from every rank
    uint16_t* ystg;      // ytma: [NT tokens][128 rows] of y, the source of the tile's TMA store
    uint8_t* xs;         // resident: [K/64][NT][128 B]; streamed: [xst][SUB][NT][128 B]
    uint8_t* ws;         // [stages][128 rows][ROWB]
    uint16_t* sb;        // [2 slots][2 arrays][128][SCP]
};

// ms: the most W stages of one CTA's K range
template <int SUB, int ROWB, int GPS>
__device__ __forceinline__ Smem carve(uint8_t* base, const Params& p, int ms) {
    Smem s;
    uint8_t* q = base;
    s.xs = q;
    const int64_t boxes = min64((int64_t)ms * SUB, p.K / KB);
    q += p.xres ? (size_t)boxes * NT * 128 : (size_t)p.xst * SUB * NT * 128;
    s.ws = q;
    q += (size_t)p.stages * 128 * ROWB;
    q += (1024u - (uint32_t)((q - base) & 1023)) & 1023u;   // base is 1024-byte aligned
    s.xtab = reinterpret_cast<float*>(q);
    q += (size_t)min(ms * GPS, p.kg) * NT * 4;
    s.red = reinterpret_cast<float*>(q);
    if (p.ksplit > 1) q += RED_BYTES;
    s.ystg = reinterpret_cast<uint16_t*>(q);
    if (p.ytma) q += YSTG_BYTES;
    s.sb = reinterpret_cast<uint16_t*>(q);
    q += 2 * 2 * 128 * SCP * 2;
    s.wfull = reinterpret_cast<uint64_t*>(q);
    s.wfree = s.wfull + MAX_STAGES;
    s.xfull = s.wfree + MAX_STAGES;
    s.xfree = s.xfull + MAX_XST;
    s.afull = s.xfree + MAX_XST;
    s.sdone = s.afull + 2;
    s.dfree = s.sdone + 2;
    s.sbar = s.dfree + 2;
    s.xbar = s.sbar + 2;
    s.xres_full = s.xbar + 1;
    s.mdone = s.xres_full + 1;
    s.red_full = s.mdone + 1;
    s.ybar = s.red_full + 1;
    s.tmem_base = reinterpret_cast<uint32_t*>(s.ybar + 1);
    s.abort = reinterpret_cast<int*>(s.tmem_base + 1);
    s.prefix = s.abort + 1;
    return s;
}

// a bounded wait of the CTA expired (or another role's did): abort the CTA; `at` names the role,
// recorded only by the first to give up
__device__ __forceinline__ void raise_abort(const Params& p, int* abort, int at) {
    atomicOr(p.err, ERR_TIMEOUT | (*(volatile int*)abort ? 0 : at));
    *(volatile int*)abort = 1;
}

__device__ __forceinline__ int total_tiles(const Params& p, const Smem& s) {
    if (p.offsets) return s.prefix[p.n_experts];
    return p.n_wtiles * p.n_ttiles * p.nbatch;
}

__device__ __forceinline__ TileInfo tile_info(const Params& p, const Smem& s, int t) {
    TileInfo ti;
    if (p.offsets) {
        int lo = 0, hi = p.n_experts;  // expert e with prefix[e] <= t < prefix[e+1]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (s.prefix[mid] <= t) lo = mid; else hi = mid;
        }
        const int e = lo;
        const int local = t - s.prefix[e];
        const int wt = local % p.n_wtiles, tt = local / p.n_wtiles;
        int64_t off, cnt;
        expert_rows(p, e, &off, &cnt);
        ti.n0 = (int64_t)wt * 128;
        ti.wrow0 = (int64_t)e * p.N + ti.n0;
        ti.nvalid = (int)min64(128, p.N - ti.n0);
        ti.xrow0 = off + (int64_t)tt * NT;
        ti.tvalid = (int)min64(NT, cnt - (int64_t)tt * NT);
        ti.b0 = ti.b1 = 0;
    } else {
        const int wt = t % p.n_wtiles;
        const int rest = t / p.n_wtiles;
        const int tt = rest % p.n_ttiles;
        const int b = rest / p.n_ttiles;
        ti.n0 = (int64_t)wt * 128;
        ti.wrow0 = ti.n0;
        ti.nvalid = (int)min64(128, p.N - ti.n0);
        ti.xrow0 = (int64_t)tt * NT;
        ti.tvalid = (int)min64(NT, p.M - ti.xrow0);
        ti.b1 = (int)(b % p.nb1);
        ti.b0 = (int)(b / p.nb1);
    }
    return ti;
}

// ---------------------------------------------------------------------------
// code expansion: one thread's 32 packed codes -> 16 pairs of OFF + q in the 16-bit MMA type
// (low half = even code)
// ---------------------------------------------------------------------------

// A stage written by TMA with a swizzle XORs byte-address bits [4..6] with bits [7..9] under
// SWZ (7: 128-byte, 3: 64-byte, 1: 32-byte, 0: none); the stage base is 1024-byte aligned, so
// stage-relative addresses swizzle the same way.
template <uint32_t SWZ>
__device__ __forceinline__ uint32_t swz_addr(uint32_t a) { return a ^ (((a >> 7) & SWZ) << 4); }

// this thread's 32 codes (sub-step j, half h) of W row `row`
template <int BITS, int ROWB>
__device__ __forceinline__ void load_w32(const uint8_t* stage, int row, int j, int h, uint32_t* w) {
    constexpr uint32_t SWZ = stage_swz(ROWB);
    const uint32_t a = (uint32_t)row * ROWB + (uint32_t)(j * KB + 32 * h) * BITS / 8;
    if constexpr (BITS == 4) {
        const uint4 v = *reinterpret_cast<const uint4*>(stage + swz_addr<SWZ>(a));
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (BITS == 8) {
        const uint4 v0 = *reinterpret_cast<const uint4*>(stage + swz_addr<SWZ>(a));
        const uint4 v1 = *reinterpret_cast<const uint4*>(stage + swz_addr<SWZ>(a + 16));
        w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
        w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
    } else if constexpr (BITS == 2) {
        const uint2 v = *reinterpret_cast<const uint2*>(stage + swz_addr<SWZ>(a));
        w[0] = v.x; w[1] = v.y;
    } else {
#pragma unroll
        for (int i = 0; i < BITS / 2; ++i) {
            const uint2 v = *reinterpret_cast<const uint2*>(stage + swz_addr<SWZ>(a + 8 * i));
            w[2 * i] = v.x; w[2 * i + 1] = v.y;
        }
    }
}

// the constant the A operand carries on top of each code
template <int BITS, typename XT>
__host__ __device__ constexpr float code_offset() {
    return std::is_same<XT, bf16_t>::value && BITS < 8 ? 128.0f : 0.0f;
}

// f16 pairs (1024 + q0, 1024 + q1) -> (q0, q1), exact
__device__ __forceinline__ uint32_t sub1024(uint32_t v) {
    const uint32_t off2 = 0x64006400u;
    const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&v), *reinterpret_cast<const __half2*>(&off2));
    return *reinterpret_cast<const uint32_t*>(&r);
}

template <int BITS, typename XT>
__device__ __forceinline__ void expand32(const uint32_t* w, uint32_t* out) {
    constexpr bool BF = std::is_same<XT, bf16_t>::value;
    // 0x4300 = 128.0 in bf16 (7 mantissa bits), 0x6400 = 1024.0 in f16 (10 mantissa bits):
    // OR-ing a code into the mantissa gives exactly 128 + q / 1024 + q; f16 then subtracts 1024.
    constexpr uint32_t MAGIC = BF ? 0x43004300u : 0x64006400u;
    auto fin = [](uint32_t v) { if constexpr (BF) return v; else return sub1024(v); };
    if constexpr (BITS == 4) {
        // byte j of a word holds codes (2j, 2j+1); the word shifted by 4 holds code 2j+1 in
        // the low nibble of byte j.  PRMT gathers both into the two halves.
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t word = w[i], shifted = w[i] >> 4;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t t = __byte_perm(word, shifted, j | (j << 4) | ((4 + j) << 8) | ((4 + j) << 12));
                out[4 * i + j] = fin((t & 0x000F000Fu) | MAGIC);
            }
        }
    } else if constexpr (BITS == 8 && !BF) {
        // bytes (q, 0x64) -> 1024 + q in each half
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 2; ++j)
                out[2 * i + j] = sub1024(__byte_perm(w[i], MAGIC, (2 * j) | (5 << 4) | ((2 * j + 1) << 8) | (7 << 12)));
    } else if constexpr (BITS == 8) {
        // bf16 cannot hold 128 + q for q >= 128: form q exactly in fp32 (2^23 + q minus 2^23),
        // then convert the pair (every q <= 255 is exact in bf16)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const float m0 = __uint_as_float(__byte_perm(w[i], 0x4B000000u, (2 * j) | (4 << 4) | (5 << 8) | (7 << 12)));
                const float m1 = __uint_as_float(__byte_perm(w[i], 0x4B000000u, (2 * j + 1) | (4 << 4) | (5 << 8) | (7 << 12)));
                const float2 qf = ptx::fadd2(make_float2(m0, m1), make_float2(-8388608.0f, -8388608.0f));
                const __nv_bfloat162 r = __floats2bfloat162_rn(qf.x, qf.y);
                out[2 * i + j] = *reinterpret_cast<const uint32_t*>(&r);
            }
        }
    } else {
        // 2 and 6 bits: funnel-shift extraction of both codes of a pair
        constexpr uint32_t MASK = (1u << BITS) - 1u;
        uint32_t ww[BITS + 1];
#pragma unroll
        for (int i = 0; i < BITS; ++i) ww[i] = w[i];
        ww[BITS] = 0;
#pragma unroll
        for (int pr = 0; pr < 16; ++pr) {
            const int p0 = (2 * pr) * BITS, p1 = p0 + BITS;
            const uint32_t q0 = __funnelshift_r(ww[p0 >> 5], ww[(p0 >> 5) + 1], p0 & 31) & MASK;
            const uint32_t q1 = __funnelshift_r(ww[p1 >> 5], ww[(p1 >> 5) + 1], p1 & 31) & MASK;
            out[pr] = fin(q0 | (q1 << 16) | MAGIC);
        }
    }
}

// ---------------------------------------------------------------------------
// scale/bias chunk loads: fold thread tid copies groups [g0, min(g0 + 32, g_end)) of row
// tid % 128, scales for tid < 128 and biases above, with 4-byte asynchronous copies
// ---------------------------------------------------------------------------
__device__ __forceinline__ void issue_sb_chunk(const Params& p, const TileInfo& ti, int g0, int g_end,
                                               uint16_t* slot, int tid) {
    const int pairs = min(SCW, g_end - g0) >> 1;  // g0 and g_end even
    const int r = tid & 127, arr = tid >> 7;
    const int64_t row = ti.wrow0 + min(r, ti.nvalid - 1);
    const uint16_t* src = (arr ? p.biases : p.scales) + row * p.kg + g0;
    uint16_t* dst = slot + arr * 128 * SCP + r * SCP;
    for (int pr = 0; pr < pairs; ++pr) ptx::cp_async_4(dst + 2 * pr, src + 2 * pr);
}

// sum over each group of x[t, k] (widened to fp32 first, added in k order) for the tile's
// tokens -> xtab[g][t], from global memory
template <typename XT, int G>
__device__ __forceinline__ void build_xtab(const Params& p, const TileInfo& ti, int g_lo, int g_hi, float* xtab,
                                           int tid) {
    const XT* xb = (const XT*)p.x + (p.offsets ? 0 : (int64_t)ti.b0 * p.xb[0] + (int64_t)ti.b1 * p.xb[1]);
    const int items = (g_hi - g_lo) * NT;
    constexpr int VPG = G / 8;  // 16-byte vectors of 8 elements per group
    for (int it = tid; it < items; it += FOLD_THREADS) {
        const int gr = it / NT, t = it - gr * NT, g = g_lo + gr;
        float acc = 0.0f;
        if (t < ti.tvalid) {
            const uint4* row = reinterpret_cast<const uint4*>(xb + (ti.xrow0 + t) * p.x_row + (int64_t)g * G);
#pragma unroll
            for (int v0 = 0; v0 < VPG; v0 += XV) {
                uint4 buf[XV];
#pragma unroll
                for (int v = 0; v < XV; ++v) buf[v] = __ldcg(row + v0 + v);   // x: L2, never a stale L1 line
#pragma unroll
                for (int v = 0; v < XV; ++v) {
                    float f[8];
                    unpack8(buf[v], f, XT{});
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc += f[e];
                }
            }
        }
        xtab[gr * NT + t] = acc;
    }
}

// the same sums from the resident x tile ([K/64][NT][128 B], 128-byte swizzle: 16-byte chunk
// c of token row t sits at chunk c ^ (t & 7)); rows past the valid tokens are zero fill
// (the resident buffer starts at group g_lo)
template <typename XT, int G>
__device__ __forceinline__ void build_xtab_smem(int ngroups, const uint8_t* xs, float* xtab, int tid) {
    const int items = ngroups * NT;
    constexpr int VPG = G / 8;
    for (int it = tid; it < items; it += FOLD_THREADS) {
        const int g = it / NT, t = it - g * NT;
        float acc = 0.0f;
#pragma unroll
        for (int v0 = 0; v0 < VPG; v0 += XV) {
            uint4 buf[XV];
#pragma unroll
            for (int v = 0; v < XV; ++v) {
                const int c = g * VPG + v0 + v;   // 16-byte chunk index along K
                buf[v] = *reinterpret_cast<const uint4*>(xs + (size_t)(c >> 3) * NT * 128 + t * 128 +
                                                         (((c & 7) ^ (t & 7)) << 4));
            }
#pragma unroll
            for (int v = 0; v < XV; ++v) {
                float f[8];
                unpack8(buf[v], f, XT{});
#pragma unroll
                for (int e = 0; e < 8; ++e) acc += f[e];
            }
        }
        xtab[g * NT + t] = acc;
    }
}

__device__ __forceinline__ void store_y(void* y, int64_t off, float v, int ydt, bf16_t) {
    if (ydt == (int)DT::F32) store_out((float*)y + off, v);
    else store_out((bf16_t*)y + off, v);
}
__device__ __forceinline__ void store_y(void* y, int64_t off, float v, int ydt, f16_t) {
    if (ydt == (int)DT::F32) store_out((float*)y + off, v);
    else store_out((f16_t*)y + off, v);
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
template <int BITS, typename XT, int G>
__global__ void __launch_bounds__(THREADS, 1) qmm_tc_kernel(const __grid_constant__ Params p) {
    constexpr int WSC = stage_codes(BITS, G);   // codes per W stage row
    constexpr int ROWB = stage_rowb(BITS, G);   // bytes per W stage row
    constexpr int SUB = WSC / KB;               // 64-code MMA sub-steps per stage
    constexpr int GPS = WSC / G;                // groups per stage
    constexpr int ACOLS = WSC / 2;              // tensor-memory columns of one A block
    constexpr int CS_W = SCW / GPS;             // W stages per scale/bias chunk
    constexpr int H = NT / 2;                   // tokens per fold thread
    constexpr float OFF = code_offset<BITS, XT>();
    static_assert(GPS >= 1 && GPS <= 4 && SUB >= 2 && SUB <= 4, "stage geometry");

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // aligned by an offset from the shared array itself, so that every pointer derived from it stays
    // in the shared address space (shared loads and stores, not generic ones)
    uint8_t* base = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    const int NWS = p.n_wstages;
    const int cs = p.ksplit;   // CTAs of a cluster splitting each tile's K (1: none)
    const Smem s = carve<SUB, ROWB, GPS>(base, p, cs > 1 ? split_max_stages(NWS, GPS, cs) : NWS);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.stages;
    const int KBLK = (int)(p.K / KB);
    const int NG = p.kg;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            ptx::mbar_init(&s.wfull[i], 1);
            ptx::mbar_init(&s.wfree[i], EXP_WARPS);
        }
        for (int i = 0; i < MAX_XST; ++i) {
            ptx::mbar_init(&s.xfull[i], 1);
            ptx::mbar_init(&s.xfree[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&s.afull[i], EXP_WARPS);
            ptx::mbar_init(&s.sdone[i], 1);
            ptx::mbar_init(&s.dfree[i], FOLD_WARPS);
            ptx::mbar_init(&s.sbar[i], FOLD_THREADS);
        }
        ptx::mbar_init(s.xbar, FOLD_THREADS);
        ptx::mbar_init(s.ybar, FOLD_THREADS);
        ptx::mbar_init(s.xres_full, 1);
        ptx::mbar_init(s.mdone, 1);
        if (cs > 1) {
            ptx::mbar_init(s.red_full, cs * FOLD_WARPS);
        }
        *s.abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&p.tx);
        ptx::prefetch_tmap(&p.tw);
    }
    if (warp == 1) {
        ptx::tmem_alloc(s.tmem_base, p.tmem_cols);
        ptx::tmem_relinquish();
    }
    // Programmatic dependent launch: the next kernel in the stream may start its own prologue
    // now.  x (and the grouped offsets) may be written by an earlier kernel and are read only
    // after the wait below, and no y is written before it; W, scales and biases are constant
    // operands of the call, so their staging may start before it.
    ptx::pdl_launch_dependents();
    if (!p.offsets && warp == 0) {
        // The scales and biases of the CTA's first two tiles go to L2 while the previous kernel in
        // the stream may still run (a prefetch changes no value that any load sees).  The W stages
        // themselves are copied only after the wait: with W stages (or TMA prefetches of them)
        // issued before it, a W copy sometimes never completed on some GPUs (the expanders' bounded
        // wait expired), at a few hundred to a few thousand decode steps apart.
        const int t0 = cs > 1 ? (int)(blockIdx.x / cs) : (int)blockIdx.x;
        const int nt_all = p.n_wtiles * p.n_ttiles * p.nbatch;
        for (int k = 0; k < (cs > 1 ? 1 : 2); ++k) {
            const int t = t0 + k * (int)gridDim.x;
            if (t >= nt_all) break;
            const int64_t n0 = (int64_t)(t % p.n_wtiles) * 128;
            const int64_t nr = min64(128, p.N - n0);
            ptx::prefetch_l2_range(p.scales + n0 * p.kg, (size_t)nr * p.kg * 2, lane, 32);
            ptx::prefetch_l2_range(p.biases + n0 * p.kg, (size_t)nr * p.kg * 2, lane, 32);
        }
    }
    ptx::pdl_wait();
    if (p.offsets && warp == 2) {
        // tiles per expert: ceil(count / NT) * n_wtiles, prefix-summed
        if (lane == 0) s.prefix[0] = 0;
        __syncwarp();
        int carry = 0;
        for (int e0 = 0; e0 < p.n_experts; e0 += 32) {
            const int e = e0 + lane;
            int v = 0;
            if (e < p.n_experts) {
                int64_t off, cnt;
                expert_rows(p, e, &off, &cnt);
                v = (int)((cnt + NT - 1) / NT) * p.n_wtiles;
            }
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
            }
            if (e < p.n_experts) s.prefix[e + 1] = carry + v;
            carry += __shfl_sync(0xffffffffu, v, 31);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (cs > 1) {
        // every CTA of the cluster has initialised its barriers before any remote arrival
        asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    }
    const uint32_t tbase = *s.tmem_base;
    const uint32_t d_tmem = tbase + (uint32_t)WSC;  // 2 x GPS group accumulators follow the two A blocks
    const int ntiles = total_tiles(p, s);
    // split K: cluster c takes tile c, its rank r the W stages [w0, w1); otherwise the CTA walks
    // tiles blockIdx.x, blockIdx.x + gridDim.x, ... over all stages
    const int rank = cs > 1 ? (int)(blockIdx.x % cs) : 0;
    const int tile0 = cs > 1 ? (int)(blockIdx.x / cs) : (int)blockIdx.x;
    const int tstep = cs > 1 ? ntiles : (int)gridDim.x;
    int w0 = 0, w1 = NWS;
    if (cs > 1) split_range(NWS, GPS, cs, rank, &w0, &w1);
    const int g_lo = w0 * GPS, g_hi = min(w1 * GPS, NG);
    const bool has_tiles = tile0 < ntiles;

    if (warp == 0) {
        // ======================= W producer =======================
        // Warp-wide loop (uniform coordinates and barrier phases); one lane issues the copies.
        const bool leader = lane == 0;
        uint32_t wg = 0;
        bool ok = true;
        for (int t = tile0; t < ntiles && ok; t += tstep) {
            const TileInfo ti = tile_info(p, s, t);
            for (int w = w0; w < w1; ++w) {
                const int st = wg % S;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.wfree[st], ((wg / S) & 1) ^ 1, s.abort, WAIT_ROLE_NS));
                if (!ok) break;
                if (leader) {
                    // columns past K (a partial last stage) read as zero fill
                    ptx::mbar_arrive_expect_tx(&s.wfull[st], 128u * ROWB);
                    ptx::tma_load_2d(s.ws + (size_t)st * 128 * ROWB, &p.tw, &s.wfull[st], w * (ROWB / 4),
                                     (int32_t)ti.wrow0);
                }
                ++wg;
            }
        }
        if (leader && !ok) {
            raise_abort(p, s.abort, DEVERR_AT_TC_WFREE);
            // drain: the copies of every issued stage must land before the CTA exits
            volatile int never = 0;
            for (uint32_t j = wg >= (uint32_t)S ? wg - S : 0; j < wg; ++j)
                ptx::mbar_wait(&s.wfull[j % S], (j / S) & 1, &never, 200000000ull);
        }
        __syncwarp();
    } else if (warp == XPROD_WARP) {
        // ======================= x producer =======================
        const bool leader = lane == 0;
        bool ok = true;
        uint32_t wg = 0;
        if (p.xres) {
            if (has_tiles && leader) {
                // the CTA's only token tile: its K range, once
                const TileInfo t0 = tile_info(p, s, tile0);
                const int kb0 = w0 * SUB, kb1 = min(w1 * SUB, KBLK);
                ptx::mbar_arrive_expect_tx(s.xres_full, (uint32_t)(kb1 - kb0) * NT * 128);
                for (int kb = kb0; kb < kb1; ++kb)
                    ptx::tma_load_4d(s.xs + (size_t)(kb - kb0) * NT * 128, &p.tx, s.xres_full, kb * KB,
                                     (int32_t)t0.xrow0, t0.b1, t0.b0);
                volatile int never = 0;
                ptx::mbar_wait(s.xres_full, 0, &never, 200000000ull);
            }
        } else {
            const int XS = p.xst;
            for (int t = tile0; t < ntiles && ok; t += tstep) {
                const TileInfo ti = tile_info(p, s, t);
                for (int w = w0; w < w1; ++w) {
                    const int xs = wg % XS;
                    ok = __all_sync(0xffffffffu,
                                    ptx::mbar_wait(&s.xfree[xs], ((wg / XS) & 1) ^ 1, s.abort, WAIT_NS));   // MMA commit
                    if (!ok) break;
                    if (leader) {
                        const int nsub = min(SUB, KBLK - w * SUB);
                        ptx::mbar_arrive_expect_tx(&s.xfull[xs], (uint32_t)nsub * NT * 128);
                        for (int j = 0; j < nsub; ++j)
                            ptx::tma_load_4d(s.xs + ((size_t)xs * SUB + j) * NT * 128, &p.tx, &s.xfull[xs],
                                             (w * SUB + j) * KB, (int32_t)ti.xrow0, ti.b1, ti.b0);
                    }
                    ++wg;
                }
            }
            if (leader && !ok) {
                raise_abort(p, s.abort, DEVERR_AT_TC_XFREE);
                volatile int never = 0;
                for (uint32_t j = wg >= (uint32_t)XS ? wg - XS : 0; j < wg; ++j)
                    ptx::mbar_wait(&s.xfull[j % XS], (j / XS) & 1, &never, 200000000ull);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ======================= MMA issuer =======================
        // Warp-wide loop so barrier phases stay warp-uniform; one lane issues the tcgen05
        // operations of a whole stage with compile-time operand offsets.
        const bool leader = lane == 0;
        uint32_t wg = 0;
        bool ok = true;
        int at = DEVERR_AT_TC_XFULL;   // which wait gave up
        if (p.xres && has_tiles) ok = __all_sync(0xffffffffu, ptx::mbar_wait(s.xres_full, 0, s.abort, WAIT_NS));
        for (int t = tile0; t < ntiles && ok; t += tstep) {
            for (int w = w0; w < w1; ++w, ++wg) {
                const int slot = wg & 1;
                const uint32_t ph = (wg >> 1) & 1;
                const int xs = p.xres ? 0 : (int)(wg % (uint32_t)p.xst);
                if (!p.xres) {
                    ok = __all_sync(0xffffffffu,
                                    ptx::mbar_wait(&s.xfull[xs], (wg / p.xst) & 1, s.abort, WAIT_NS));
                    if (!ok) break;
                }
                at = DEVERR_AT_TC_AFULL;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.afull[slot], ph, s.abort, WAIT_ROLE_NS));
                if (!ok) break;
                // the folds have read this slot's accumulators (stage wg - 2)
                at = DEVERR_AT_TC_DFREE;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.dfree[slot], ph ^ 1, s.abort, WAIT_ROLE_NS));
                if (!ok) break;
                at = DEVERR_AT_TC_XFULL;
                ptx::tc_fence_after();
                if (leader) {
                    const uint32_t a_blk = tbase + (uint32_t)(slot * ACOLS);
                    const uint32_t d_blk = d_tmem + (uint32_t)(slot * GPS * NT);
                    // B operand: the stage's first 64-code box; boxes are NT*128 bytes apart
                    const uint64_t bdesc = ptx::smem_desc_sw128(ptx::smem_u32(
                        p.xres ? s.xs + (size_t)(w - w0) * SUB * NT * 128 : s.xs + (size_t)xs * SUB * NT * 128));
                    const int nsub = min(SUB, KBLK - w * SUB);
#pragma unroll
                    for (int j = 0; j < SUB; ++j) {
                        if (j < nsub) {
#pragma unroll
                            for (int kk = 0; kk < KB / 16; ++kk) {
                                const int ks = j * KB + 16 * kk;   // code offset within the stage
                                const uint32_t d = d_blk + (uint32_t)((ks / G) * NT);
                                const uint32_t a = a_blk + (uint32_t)(j * 32 + kk * 8);
                                // descriptor start address: +NT*128 bytes per box, +32 bytes per K = 16 slice
                                const uint64_t b = bdesc + (uint64_t)(j * (NT * 128 / 16) + 2 * kk);
                                if (ks % G == 0) ptx::mma_ts_imm<0>(d, a, b, p.idesc);
                                else ptx::mma_ts_imm<1>(d, a, b, p.idesc);
                            }
                        }
                    }
                    ptx::mma_commit(&s.sdone[slot]);
                    if (!p.xres) ptx::mma_commit(&s.xfree[xs]);
                }
                __syncwarp();
            }
        }
        if (!ok && leader) raise_abort(p, s.abort, at);
        // every MMA this warp issued must retire before tensor memory is freed
        if (leader) {
            ptx::mma_commit(s.mdone);
            volatile int never = 0;
            ptx::mbar_wait(s.mdone, 0, &never, 200000000ull);
        }
        __syncwarp();
    } else if (warp < 2 + EXP_WARPS) {
        // ======================= code expanders =======================
        // Thread <-> W row (TMEM lane); warps q and q + 4 split each 64 codes.  Stage i is
        // written into A block i % 2 once the MMAs of stage i - 2 are complete.
        const int q = warp & 3;
        const int h = (warp - 2) >> 2;
        const int row = 32 * q + lane;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        uint32_t wg = 0;
        bool ok = true;
        int at = DEVERR_AT_TC_WFULL;   // which wait gave up
        for (int t = tile0; t < ntiles && ok; t += tstep) {
            for (int w = w0; w < w1; ++w, ++wg) {
                const int st = wg % S;
                at = DEVERR_AT_TC_WFULL;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.wfull[st], (wg / S) & 1, s.abort, WAIT_NS));
                if (!ok) break;
                // expand the whole stage into registers while the MMAs of stage wg - 2 may still
                // be reading A block wg % 2
                const uint8_t* wstage = s.ws + (size_t)st * 128 * ROWB;
                const int nsub = min(SUB, KBLK - w * SUB);
                uint32_t out[SUB][16];
#pragma unroll
                for (int j = 0; j < SUB; ++j) {
                    if (j < nsub) {
                        uint32_t wv[BITS];
                        load_w32<BITS, ROWB>(wstage, row, j, h, wv);
                        expand32<BITS, XT>(wv, out[j]);
                    }
                }
                if (wg >= 2) {
                    at = DEVERR_AT_TC_SDONE_E;
                    ok = __all_sync(0xffffffffu,
                                    ptx::mbar_wait(&s.sdone[wg & 1], ((wg >> 1) & 1) ^ 1, s.abort, WAIT_NS));
                    if (!ok) break;
                    ptx::tc_fence_after();
                }
                const uint32_t a_blk = tbase + lane_base + (uint32_t)((wg & 1) * ACOLS);
#pragma unroll
                for (int j = 0; j < SUB; ++j)
                    if (j < nsub) ptx::tmem_st16(a_blk + (uint32_t)(j * 32 + 16 * h), out[j]);
                ptx::tc_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    ptx::mbar_arrive(&s.wfree[st]);
                    ptx::mbar_arrive(&s.afull[wg & 1]);
                }
            }
        }
        if (!ok) raise_abort(p, s.abort, at);
    } else {
        // ======================= folds =======================
        // Thread <-> W row; warps q and q + 4 take 16 tokens each.  Per stage:
        // y += s*D'_g + (b - OFF*s)*X_g for each of its groups, then release the stage's
        // accumulators.  Per tile: store y (staged tile and one TMA store, or element stores).
        const int q = warp & 3;
        const int th = (warp - 2 - EXP_WARPS) >> 2;
        const int row = 32 * q + lane;
        const int tid = threadIdx.x - 32 * (2 + EXP_WARPS);   // 0..255
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        uint32_t wg = 0, xph = 0, ytile = 0;
        int unit = 0;
        bool ok = true;
        int at = DEVERR_AT_TC_FOLD;   // which wait gave up

        if (has_tiles) {
            const TileInfo t0 = tile_info(p, s, tile0);
            issue_sb_chunk(p, t0, g_lo, g_hi, s.sb, tid);
        }
        ptx::cp_async_commit();
        const uint16_t* sbslot = s.sb;
        int g_chunk0 = 0;
        int64_t cur_x0 = -1;
        int cur_b0 = -1, cur_b1 = -1, cur_tv = -1;

        for (int t = tile0; t < ntiles && ok; t += tstep) {
            const TileInfo ti = tile_info(p, s, t);
            if (ti.xrow0 != cur_x0 || ti.b0 != cur_b0 || ti.b1 != cur_b1 || ti.tvalid != cur_tv) {
                // sums of x for this token tile
                ptx::mbar_arrive(s.xbar);  // everyone is done reading the previous table
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(s.xbar, xph & 1, s.abort, WAIT_ROLE_NS));
                ++xph;
                if (!ok) break;
                if (p.xres) {
                    ok = __all_sync(0xffffffffu, ptx::mbar_wait(s.xres_full, 0, s.abort, WAIT_NS));
                    if (!ok) break;
                    build_xtab_smem<XT, G>(g_hi - g_lo, s.xs, s.xtab, tid);
                } else {
                    build_xtab<XT, G>(p, ti, g_lo, g_hi, s.xtab, tid);
                }
                ptx::mbar_arrive(s.xbar);
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(s.xbar, xph & 1, s.abort, WAIT_ROLE_NS));
                ++xph;
                if (!ok) break;
                cur_x0 = ti.xrow0;
                cur_b0 = ti.b0;
                cur_b1 = ti.b1;
                cur_tv = ti.tvalid;
            }
            float2 acc[H / 2];
#pragma unroll
            for (int i = 0; i < H / 2; ++i) acc[i] = make_float2(0.0f, 0.0f);
            for (int w = w0; w < w1; ++w, ++wg) {
                if ((w - w0) % CS_W == 0) {
                    // this stage opens a scale/bias chunk: its copies were issued a chunk earlier.
                    // (ytma: every tile opens with a chunk, and the store of the previous tile's y has
                    // read the staging tile before any fold thread passes this barrier)
                    ptx::cp_async_wait_all();
                    if (p.ytma && tid == 0) ptx::bulk_wait_read_all();
                    ptx::mbar_arrive(&s.sbar[unit & 1]);
                    ok = __all_sync(0xffffffffu,
                                    ptx::mbar_wait(&s.sbar[unit & 1], (unit >> 1) & 1, s.abort, WAIT_ROLE_NS));
                    if (!ok) break;
                    sbslot = s.sb + (unit & 1) * 2 * 128 * SCP;
                    g_chunk0 = g_lo + ((w - w0) / CS_W) * SCW;
                    uint16_t* nslot = s.sb + ((unit + 1) & 1) * 2 * 128 * SCP;
                    if (g_chunk0 + SCW < g_hi) {
                        issue_sb_chunk(p, ti, g_chunk0 + SCW, g_hi, nslot, tid);
                    } else if (t + tstep < ntiles) {
                        const TileInfo tn = tile_info(p, s, t + tstep);
                        issue_sb_chunk(p, tn, g_lo, g_hi, nslot, tid);
                    }
                    ptx::cp_async_commit();
                    ++unit;
                }
                const int slot = wg & 1;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.sdone[slot], (wg >> 1) & 1, s.abort, WAIT_NS));
                if (!ok) {
                    at = DEVERR_AT_TC_SDONE_F;
                    break;
                }
                ptx::tc_fence_after();
#pragma unroll
                for (int lg = 0; lg < GPS; ++lg) {
                    const int g = w * GPS + lg;
                    if (g < NG) {
                        const int gl = g - g_chunk0;
                        uint32_t v[H];
                        ptx::tmem_ld16(d_tmem + (uint32_t)((slot * GPS + lg) * NT + th * H) + lane_base, v);
                        const float sv = half_bits_to_float(sbslot[row * SCP + gl], XT{});
                        const float bv = half_bits_to_float(sbslot[128 * SCP + row * SCP + gl], XT{});
                        const float bo = OFF == 0.0f ? bv : fmaf(-OFF, sv, bv);   // b - OFF*s
                        const float2 s2 = make_float2(sv, sv), b2 = make_float2(bo, bo);
                        const float* xg = s.xtab + (g - g_lo) * NT + th * H;
                        ptx::tc_wait_ld();
#pragma unroll
                        for (int c = 0; c < H; c += 4) {
                            const float4 xv = *reinterpret_cast<const float4*>(xg + c);
                            float2& a0 = acc[c / 2];
                            float2& a1 = acc[c / 2 + 1];
                            a0 = ptx::ffma2(b2, make_float2(xv.x, xv.y), a0);
                            a1 = ptx::ffma2(b2, make_float2(xv.z, xv.w), a1);
                            a0 = ptx::ffma2(s2, make_float2(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), a0);
                            a1 = ptx::ffma2(s2, make_float2(__uint_as_float(v[c + 2]), __uint_as_float(v[c + 3])), a1);
                        }
                    }
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&s.dfree[slot]);
            }
            if (!ok) break;
            if (cs > 1) {
                // ---- split K: rank r owns rows [r*RPR, (r+1)*RPR) of the tile.  Every rank pushes
                //      its partial sums of each row into the owner's buffer (distributed shared
                //      memory stores), then the owner adds the ranks' parts in rank order
                //      (deterministic) and stores its rows.  One remote arrival per warp and owner:
                //      the warp barrier orders every lane's stores before lane 0's release. ----
                const int rpr = 128 / cs;
                const int owner = row / rpr;
                const uint32_t dst = ptx::mapa(
                    ptx::smem_u32(s.red + ((size_t)rank * rpr + (row - owner * rpr)) * NT + th * H), (uint32_t)owner);
#pragma unroll
                for (int i = 0; i < H / 4; ++i)
                    ptx::st_cluster_f4(dst + 16 * i, make_float4(acc[2 * i].x, acc[2 * i].y, acc[2 * i + 1].x,
                                                                 acc[2 * i + 1].y));
                __syncwarp();
                if (lane == 0)
                    for (int r = 0; r < cs; ++r) ptx::mbar_arrive_cluster(ptx::mapa(ptx::smem_u32(s.red_full), (uint32_t)r));
                ok = __all_sync(0xffffffffu, ptx::mbar_wait_cluster(s.red_full, 0, s.abort, WAIT_ROLE_NS));
                if (!ok) break;
                // this thread: elements [tid*F, tid*F + F) of the owned [rpr][NT] block
                const int F = (128 * NT) / (cs * FOLD_THREADS);
                for (int f = 0; f < F; ++f) {
                    const int e = tid * F + f;
                    float v = 0.0f;
                    for (int r = 0; r < cs; ++r) v += s.red[(size_t)r * rpr * NT + e];
                    const int rloc = rank * rpr + e / NT, tok = e % NT;
                    if (rloc < ti.nvalid && tok < ti.tvalid) {
                        int64_t off = (ti.xrow0 + tok) * p.y_row + ti.n0 + rloc;
                        if (!p.offsets) off += (int64_t)ti.b0 * p.yb[0] + (int64_t)ti.b1 * p.yb[1];
                        store_y(p.y, off, v, p.ydt, XT{});
                    }
                }
                break;   // one tile per cluster
            }
            if (p.ytma) {
                // ---- the tile's y: every fold thread writes its row of its half of the tokens into
                //      the staging tile, then one thread stores the tile with TMA (rows past N and
                //      tokens past M fall outside the tensor map and are not written; N is a multiple
                //      of 8, so a row's end is a 16-byte boundary of the store) ----
                uint16_t* stg = s.ystg + row;
#pragma unroll
                for (int i = 0; i < H / 2; ++i) {
                    const int tok = th * H + 2 * i;
                    stg[tok * 128] = float_to_half_bits(acc[i].x, XT{});
                    stg[(tok + 1) * 128] = float_to_half_bits(acc[i].y, XT{});
                }
                ptx::fence_proxy_async();
                ptx::mbar_arrive(s.ybar);
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(s.ybar, ytile & 1, s.abort, WAIT_ROLE_NS));
                ++ytile;
                if (!ok) break;
                if (tid == 0) {
                    ptx::tma_store_4d(&p.ty, s.ystg, (int32_t)ti.n0, (int32_t)ti.xrow0, ti.b1, ti.b0);
                    ptx::bulk_commit_group();
                }
                continue;
            }
            // ---- this thread's row of y for its half of the tokens ----
            if (row < ti.nvalid) {
                const int64_t n = ti.n0 + row;
                int64_t off = ti.xrow0 * p.y_row + n;
                if (!p.offsets) off += (int64_t)ti.b0 * p.yb[0] + (int64_t)ti.b1 * p.yb[1];
#pragma unroll
                for (int i = 0; i < H / 2; ++i) {
                    const int tok = th * H + 2 * i;
                    if (tok < ti.tvalid) store_y(p.y, off + (int64_t)tok * p.y_row, acc[i].x, p.ydt, XT{});
                    if (tok + 1 < ti.tvalid) store_y(p.y, off + (int64_t)(tok + 1) * p.y_row, acc[i].y, p.ydt, XT{});
                }
            }
        }
        ptx::cp_async_wait_all();
        if (p.ytma && tid == 0) ptx::bulk_wait_all();   // every tile's store is complete before the CTA exits
        if (!ok) raise_abort(p, s.abort, at);
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tbase, p.tmem_cols);
    }
}

// ---------------------------------------------------------------------------
// launch (per device: raise the dynamic shared memory limit once)
// ---------------------------------------------------------------------------
constexpr size_t SMEM_LIMIT = 227 * 1024;

template <int BITS, typename XT, int G>
cudaError_t launch_t(const Params& prm, int grid, size_t smem, cudaStream_t s) {
    static std::mutex mu;
    static bool done[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!done[dev]) {
            e = cudaFuncSetAttribute(qmm_tc_kernel<BITS, XT, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)SMEM_LIMIT);
            if (e != cudaSuccess) return e;
            done[dev] = true;
        }
    }
    // launched as a programmatic dependent of the previous kernel in the stream (see the kernel's
    // prologue for what it does before the previous grid completes)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)prm.ksplit;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, qmm_tc_kernel<BITS, XT, G>, prm);
}

template <int BITS, typename XT>
cudaError_t launch_g(int group, const Params& prm, int grid, size_t smem, cudaStream_t s) {
    switch (group) {
        case 32: return launch_t<BITS, XT, 32>(prm, grid, smem, s);
        case 64: return launch_t<BITS, XT, 64>(prm, grid, smem, s);
        case 128: return launch_t<BITS, XT, 128>(prm, grid, smem, s);
    }
    return cudaErrorInvalidValue;
}

template <int BITS>
cudaError_t launch(bool bf16, int group, const Params& prm, int grid, size_t smem, cudaStream_t stream) {
    return bf16 ? launch_g<BITS, bf16_t>(group, prm, grid, smem, stream)
                : launch_g<BITS, f16_t>(group, prm, grid, smem, stream);
}

}  // namespace mma
}  // namespace aq
