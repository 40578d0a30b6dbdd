// kernels_mma.cu -- tensor-core kernel for y = x . dequant(W)^T on sm_100a (tcgen05 / TMEM).
//
// Arithmetic (exact up to fp32 summation order).  With codes q, per-group
// scale s and bias b (w = s*q + b), each output is
//     y[n, t] = sum_g  s[n,g] * D_g[n, t]  +  b[n,g] * X_g[t],
//     D_g[n, t] = sum_{k in g} q[n, k] * x[t, k],    X_g[t] = sum_{k in g} x[t, k].
// The tensor core computes D_g with the INTEGER codes as its A operand (exact
// in bf16/f16) and x as B, one fresh fp32 accumulator per group; the epilogue
// warps fold s and b in with fp32 FMAs.  X_g is summed from x widened to fp32
// before any addition ("mlx PR #4516", load_vector fix).  Rounding w to bf16
// before the MMA would cost ~2e-3 of max|y| on its own, while the output
// rounding to bf16 already spends 2^-8 of the 4e-3 error budget, so the
// weights are never rounded here.
//
// "Weights-stationary" tiles: 128 rows of W are the MMA's M side, up to 32
// tokens its N side.  The pipeline advances one W stage at a time (128 rows x
// WSC codes, WSC = 128 or 256 so that a stage row is a 64..128-byte TMA line)
// and every hand-off between roles happens once per stage:
//   warp 0      W producer: TMA of each W stage onto wfull[s] (ring of up to 12).
//   warp 10     x producer: the CTA's token tile once (resident x), or per W
//               stage its x block (SUB boxes of [NT x 64], 128-byte swizzle, the
//               UMMA B operand) onto a ring of up to 4 x stages.
//   warp 1      MMA issuer (warp-wide loop, one lane issues): waits for the
//               expanded codes of the stage (afull) and for its accumulators to
//               be free (dfree), then issues SUB*4 tcgen05.mma kind::f16 with A
//               from tensor memory, one fresh accumulator per group, and one
//               tcgen05.commit (sdone[w % 2]; a second one frees a streamed x stage).
//   warps 2..9  code expanders + epilogue: thread <-> W row (TMEM lane), two
//               warps per lane quarter split each 64 codes.  Per stage they
//               expand the packed codes into bf16/f16 integers (tcgen05.st into
//               A block w % 2), release the shared-memory stage (wfree), then
//               fold the previous stage's groups into fp32 registers
//               (tcgen05.ld of D, + s*D + b*X) and release its accumulators.
// Tensor memory: [A block 0 | A block 1 | D: 2 x GPS group accumulators of NT
// columns]; with GPS = WSC / group <= 4 this fits 512 columns.
//
// Rows of the last W tile that fall past N read TMA zero fill and the clamped
// last row's scale/bias and are simply not stored: no per-row check inside the
// K loop (the partial-rows idea of "mlx PR #4516").
//
// Every mbarrier wait is bounded (2 s); on expiry the CTA raises an abort flag,
// records an error word readable through aq_device_error(), drains its own
// outstanding copies and MMAs (bounded), frees its tensor memory and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>
#include <type_traits>

#include "aq_internal.h"
#include "device_common.cuh"
#include "sm100_ptx.cuh"

namespace aq {

__device__ int g_device_error = 0;

namespace {

constexpr int MMA_THREADS = 352;          // 11 warps
constexpr int DQ_THREADS = 256;           // warps 2..9
constexpr int KB = 64;                    // codes per MMA sub-step (4 tcgen05.mma of K = 16)
constexpr int SCW = 32;                   // groups per scale/bias chunk
constexpr int SCP = SCW + 2;              // padded row pitch (halves) of a chunk in shared memory
constexpr int MAX_STAGES = 12;
constexpr int MAX_XST = 4;                // streamed x stages
constexpr int MAX_EXPERTS = 1024;
constexpr int XTAB_MAX_BYTES = 32 * 1024; // sum-of-x table per token tile
constexpr int NT_MAX = 32;                // tokens per tile
constexpr uint64_t WAIT_NS = 2000000000ull;  // 2 s per wait
constexpr int ERR_TIMEOUT = 1;

struct MmaParams {
    CUtensorMap tx;  // x: 4D {K, rows, nb1, nb0} u16, box {64, NT, 1, 1}, 128B swizzle
    CUtensorMap tw;  // W: 2D {K*bits/32, rows} u32, box {rowb/4, 128}
    const void* x;
    void* y;
    const uint16_t* scales;
    const uint16_t* biases;
    int64_t M, N, K;
    int64_t x_row, y_row;
    int64_t xb[2], yb[2];
    int64_t nb1;
    int n_wtiles, n_ttiles, nbatch;
    int group, log2g;
    int kg;              // groups per row = K / group
    int ydt;             // DT of y
    int wsc;             // codes per W stage (128 or 256)
    int rowb;            // bytes per W row per stage
    int sub;             // 64-code MMA sub-steps per stage
    int gps;             // groups per stage
    uint32_t swz;        // swizzle mask of the W stage (see swz_addr)
    int n_wstages;       // W stages per tile
    int stages;          // W ring depth
    int cs_w;            // W stages per scale/bias chunk
    int xres;            // 1: the CTA's single x tile stays resident in shared memory
    int xst;             // streamed x ring depth (x stages of SUB boxes) when not resident
    uint32_t tmem_cols;
    uint32_t idesc;
    const int64_t* offsets;  // grouped mode when non-null
    int n_experts;
};

__device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

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
    uint64_t* wfree;     // [MAX_STAGES] W stage read by the 8 expander warps
    uint64_t* xfull;     // [MAX_XST] streamed x stage landed (TMA)
    uint64_t* xfree;     // [MAX_XST] streamed x stage read by its MMAs (commit)
    uint64_t* afull;     // [2] A block written (8 expander warps)
    uint64_t* sdone;     // [2] MMAs of a W stage complete (commit)
    uint64_t* dfree;     // [2] group accumulators of a W stage read (8 epilogue warps)
    uint64_t* sbar;      // [2] scale/bias chunk slots: 256 arrivals
    uint64_t* xbar;      // sum-of-x table: 256 arrivals
    uint64_t* xres_full; // resident x landed
    uint64_t* mdone;     // teardown: all MMAs retired
    uint32_t* tmem_base;
    int* abort;
    int* prefix;         // grouped: tile prefix sums [n_experts + 1]
    float* xtab;         // [kg][NT] sums of x per group and token
    uint8_t* xs;         // resident: [K/64][NT][128 B]; streamed: [xst][SUB][NT][128 B]
    uint8_t* ws;         // [stages][128 rows][rowb]
    uint16_t* sb;        // [2 slots][2 arrays][128][SCP]
};

template <int NT>
__device__ __forceinline__ Smem carve(uint8_t* base, const MmaParams& p) {
    Smem s;
    uint8_t* q = base;
    s.xs = q;
    q += p.xres ? (size_t)(p.K / KB) * NT * 128 : (size_t)p.xst * p.sub * NT * 128;
    s.ws = q;
    q += (size_t)p.stages * 128 * p.rowb;
    q = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(q) + 1023) & ~uintptr_t(1023));
    s.xtab = reinterpret_cast<float*>(q);
    q += (size_t)p.kg * NT * 4;
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
    s.tmem_base = reinterpret_cast<uint32_t*>(s.mdone + 1);
    s.abort = reinterpret_cast<int*>(s.tmem_base + 1);
    s.prefix = s.abort + 1;
    return s;
}

__host__ __device__ constexpr size_t smem_fixed_bytes() {
    return 2 * 2 * 128 * SCP * 2 + (2 * MAX_STAGES + 2 * MAX_XST + 2 * 4 + 3) * 8 + 8 + (MAX_EXPERTS + 1) * 4 + 2 * 1024 /*align*/;
}

__device__ __forceinline__ void raise_abort(int* abort) {
    *(volatile int*)abort = 1;
    atomicExch(&g_device_error, ERR_TIMEOUT);
}

__device__ __forceinline__ int total_tiles(const MmaParams& p, const Smem& s) {
    if (p.offsets) return s.prefix[p.n_experts];
    return p.n_wtiles * p.n_ttiles * p.nbatch;
}

template <int NT>
__device__ __forceinline__ TileInfo tile_info(const MmaParams& p, const Smem& s, int t) {
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
        const int64_t off = p.offsets[e], cnt = p.offsets[e + 1] - off;
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
// code expansion: one thread's 32 packed codes -> 16 pairs of exact integers
// in the 16-bit MMA type (low half = even code)
// ---------------------------------------------------------------------------

// This thread's 32 codes (sub-step j, half h) of W row `row` in a stage whose rows are
// `rowb` bytes apart.  TMA wrote the stage with a swizzle that XORs byte-address bits
// [4..6] with bits [7..9] under `swz` (7: 128-byte, 3: 64-byte, 1: 32-byte, 0: none);
// the stage base is 1024-byte aligned, so stage-relative addresses swizzle the same way.
__device__ __forceinline__ uint32_t swz_addr(uint32_t a, uint32_t swz) { return a ^ (((a >> 7) & swz) << 4); }

template <int BITS>
__device__ __forceinline__ void load_w32(const uint8_t* stage, int rowb, uint32_t swz, int row, int j, int h,
                                         uint32_t* w) {
    const uint32_t a = (uint32_t)row * rowb + (uint32_t)(j * KB + 32 * h) * BITS / 8;
    if constexpr (BITS == 4) {
        const uint4 v = *reinterpret_cast<const uint4*>(stage + swz_addr(a, swz));
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (BITS == 8) {
        const uint4 v0 = *reinterpret_cast<const uint4*>(stage + swz_addr(a, swz));
        const uint4 v1 = *reinterpret_cast<const uint4*>(stage + swz_addr(a + 16, swz));
        w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
        w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
    } else if constexpr (BITS == 2) {
        const uint2 v = *reinterpret_cast<const uint2*>(stage + swz_addr(a, swz));
        w[0] = v.x; w[1] = v.y;
    } else {
#pragma unroll
        for (int i = 0; i < BITS / 2; ++i) {
            const uint2 v = *reinterpret_cast<const uint2*>(stage + swz_addr(a + 8 * i, swz));
            w[2 * i] = v.x; w[2 * i + 1] = v.y;
        }
    }
}

// (OFF + q0, OFF + q1) in both halves -> (q0, q1), exact
__device__ __forceinline__ uint32_t sub_off(uint32_t v, uint32_t off2, bf16_t) {
    const __nv_bfloat162 r = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&v),
                                     *reinterpret_cast<const __nv_bfloat162*>(&off2));
    return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t sub_off(uint32_t v, uint32_t off2, f16_t) {
    const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&v), *reinterpret_cast<const __half2*>(&off2));
    return *reinterpret_cast<const uint32_t*>(&r);
}

template <int BITS, typename XT>
__device__ __forceinline__ void expand32(const uint32_t* w, uint32_t* out) {
    constexpr bool BF = std::is_same<XT, bf16_t>::value;
    // 0x4300 = 128.0 in bf16 (7 mantissa bits), 0x6400 = 1024.0 in f16 (10 mantissa bits):
    // OR-ing a code into the mantissa gives exactly OFF + q.
    constexpr uint32_t MAGIC = BF ? 0x43004300u : 0x64006400u;
    if constexpr (BITS == 4) {
        // byte j of a word holds codes (2j, 2j+1); the word shifted by 4 holds code 2j+1 in
        // the low nibble of byte j.  PRMT gathers both into the two halves.
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t word = w[i], shifted = w[i] >> 4;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t t = __byte_perm(word, shifted, j | (j << 4) | ((4 + j) << 8) | ((4 + j) << 12));
                out[4 * i + j] = sub_off((t & 0x000F000Fu) | MAGIC, MAGIC, XT{});
            }
        }
    } else if constexpr (BITS == 8 && !BF) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 2; ++j)
                out[2 * i + j] = sub_off(
                    __byte_perm(w[i], MAGIC, (2 * j) | (5 << 4) | ((2 * j + 1) << 8) | (7 << 12)), MAGIC, XT{});
    } else if constexpr (BITS == 8) {
        // bf16 cannot hold 128 + q for q >= 128: form q exactly in fp32 (2^23 + q minus 2^23), then
        // convert the pair (every q <= 255 is exact in bf16)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const float q0 = __uint_as_float(__byte_perm(w[i], 0x4B000000u, (2 * j) | (4 << 4) | (5 << 8) | (7 << 12))) - 8388608.0f;
                const float q1 = __uint_as_float(__byte_perm(w[i], 0x4B000000u, (2 * j + 1) | (4 << 4) | (5 << 8) | (7 << 12))) - 8388608.0f;
                const __nv_bfloat162 r = __floats2bfloat162_rn(q0, q1);
                out[2 * i + j] = *reinterpret_cast<const uint32_t*>(&r);
            }
        }
    } else {
        // generic widths (2, 6): funnel-shift extraction of both codes of a pair
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
            out[pr] = sub_off(q0 | (q1 << 16) | MAGIC, MAGIC, XT{});
        }
    }
}

// ---------------------------------------------------------------------------
// scale/bias chunk loads (asynchronous 4-byte copies by the 256 expander threads)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void issue_sb_chunk(const MmaParams& p, const TileInfo& ti, int chunk, uint16_t* slot,
                                               int tid) {
    const int g0 = chunk * SCW;
    const int ng = min(SCW, p.kg - g0);          // even (kg even, SCW even)
    const int pairs = ng >> 1;
    const int items = 128 * pairs * 2;
    for (int it = tid; it < items; it += DQ_THREADS) {
        const int arr = it / (128 * pairs);
        const int rem = it - arr * 128 * pairs;
        const int r = rem / pairs, pr = rem - r * pairs;
        const int64_t row = ti.wrow0 + min(r, ti.nvalid - 1);
        const uint16_t* src = (arr == 0 ? p.scales : p.biases) + row * p.kg + g0 + 2 * pr;
        uint16_t* dst = slot + arr * 128 * SCP + r * SCP + 2 * pr;
        ptx::cp_async_4(dst, src);
    }
}

// sum over each group of x[t, k] (widened to fp32 first) for the tile's tokens -> xtab[g][t]
template <typename XT, int NT>
__device__ __forceinline__ void build_xtab(const MmaParams& p, const TileInfo& ti, float* xtab, int tid) {
    const XT* xb = (const XT*)p.x + (p.offsets ? 0 : (int64_t)ti.b0 * p.xb[0] + (int64_t)ti.b1 * p.xb[1]);
    const int items = p.kg * NT;
    const int vec_per_group = p.group >> 3;  // 16-byte vectors of 8 elements
    for (int it = tid; it < items; it += DQ_THREADS) {
        const int g = it / NT, t = it - g * NT;
        float acc = 0.0f;
        if (t < ti.tvalid) {
            const XT* row = xb + (ti.xrow0 + t) * p.x_row + (int64_t)g * p.group;
            for (int v = 0; v < vec_per_group; ++v) {
                float f[8];
                unpack8(__ldg(reinterpret_cast<const uint4*>(row) + v), f, XT{});
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
template <int BITS, typename XT, int NT>
__global__ void __launch_bounds__(MMA_THREADS, 1) qmm_tc_kernel(const __grid_constant__ MmaParams p) {
    constexpr int H = NT / 2;            // tokens per epilogue thread
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const Smem s = carve<NT>(base, p);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.stages;
    const int KBLK = (int)(p.K / KB);
    const int G = p.group;
    const int NG = p.kg;
    const int NWS = p.n_wstages;
    const int SUB = p.sub;
    const int GPS = p.gps;
    const int ACOLS = p.wsc / 2;            // tensor-memory columns of one A block
    const int NCH = (NG + SCW - 1) / SCW;   // scale/bias chunks per tile

#ifdef AQ_TRACE
    if (threadIdx.x < 64) ::aq_trace_smem[threadIdx.x] = 0;
#endif
    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            ptx::mbar_init(&s.wfull[i], 1);
            ptx::mbar_init(&s.wfree[i], 8);
        }
        for (int i = 0; i < MAX_XST; ++i) {
            ptx::mbar_init(&s.xfull[i], 1);
            ptx::mbar_init(&s.xfree[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&s.afull[i], 8);
            ptx::mbar_init(&s.sdone[i], 1);
            ptx::mbar_init(&s.dfree[i], 8);
            ptx::mbar_init(&s.sbar[i], DQ_THREADS);
        }
        ptx::mbar_init(s.xbar, DQ_THREADS);
        ptx::mbar_init(s.xres_full, 1);
        ptx::mbar_init(s.mdone, 1);
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
    if (p.offsets && warp == 2) {
        // tiles per expert: ceil(count / NT) * n_wtiles, prefix-summed
        if (lane == 0) s.prefix[0] = 0;
        __syncwarp();
        int carry = 0;
        for (int e0 = 0; e0 < p.n_experts; e0 += 32) {
            const int e = e0 + lane;
            int v = 0;
            if (e < p.n_experts) {
                const int64_t cnt = p.offsets[e + 1] - p.offsets[e];
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
    const uint32_t tbase = *s.tmem_base;
    const uint32_t d_tmem = tbase + (uint32_t)p.wsc;  // 2 x GPS group accumulators follow the two A blocks
    const int ntiles = total_tiles(p, s);
    const bool has_tiles = (int)blockIdx.x < ntiles;

    if (warp == 0) {
        // ======================= W producer =======================
        // Warp-wide loop (uniform coordinates and barrier phases); one lane issues the copies.
        const bool leader = lane == 0;
        const uint32_t wbytes = 128u * (uint32_t)p.rowb;
        uint32_t wg = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const TileInfo ti = tile_info<NT>(p, s, t);
            for (int w = 0; w < NWS; ++w) {
                const int st = wg % S;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.wfree[st], ((wg / S) & 1) ^ 1, s.abort, WAIT_NS, 0));
                if (!ok) break;
                if (leader) {
                    // columns past K (a partial last stage) read as zero fill
                    ptx::mbar_arrive_expect_tx(&s.wfull[st], wbytes);
                    ptx::tma_load_2d(s.ws + (size_t)st * 128 * p.rowb, &p.tw, &s.wfull[st], w * (p.rowb / 4),
                                     (int32_t)ti.wrow0);
                }
                ++wg;
            }
        }
        if (leader && !ok) {
            raise_abort(s.abort);
            // drain: the copies of every issued stage must land before the CTA exits
            volatile int never = 0;
            for (uint32_t j = wg >= (uint32_t)S ? wg - S : 0; j < wg; ++j)
                ptx::mbar_wait(&s.wfull[j % S], (j / S) & 1, &never, 200000000ull);
        }
        __syncwarp();
    } else if (warp == 10) {
        // ======================= x producer =======================
        const bool leader = lane == 0;
        bool ok = true;
        uint32_t wg = 0;
        if (p.xres) {
            if (has_tiles && leader) {
                // the CTA's only token tile: all of K, once
                const TileInfo t0 = tile_info<NT>(p, s, blockIdx.x);
                ptx::mbar_arrive_expect_tx(s.xres_full, (uint32_t)KBLK * NT * 128);
                for (int kb = 0; kb < KBLK; ++kb)
                    ptx::tma_load_4d(s.xs + (size_t)kb * NT * 128, &p.tx, s.xres_full, kb * KB, (int32_t)t0.xrow0,
                                     t0.b1, t0.b0);
                volatile int never = 0;
                ptx::mbar_wait(s.xres_full, 0, &never, 200000000ull);
            }
        } else {
            const int XS = p.xst;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                const TileInfo ti = tile_info<NT>(p, s, t);
                for (int w = 0; w < NWS; ++w) {
                    const int xs = wg % XS;
                    ok = __all_sync(0xffffffffu,
                                    ptx::mbar_wait(&s.xfree[xs], ((wg / XS) & 1) ^ 1, s.abort, WAIT_NS, 9));
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
                raise_abort(s.abort);
                volatile int never = 0;
                for (uint32_t j = wg >= (uint32_t)XS ? wg - XS : 0; j < wg; ++j)
                    ptx::mbar_wait(&s.xfull[j % XS], (j / XS) & 1, &never, 200000000ull);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ======================= MMA issuer =======================
        // Warp-wide loop so barrier phases, tensor-memory addresses and descriptors stay
        // warp-uniform; one lane issues the tcgen05 operations.
        const bool leader = lane == 0;
        uint32_t wg = 0;
        bool ok = true;
        if (p.xres && has_tiles) ok = __all_sync(0xffffffffu, ptx::mbar_wait(s.xres_full, 0, s.abort, WAIT_NS, 1));
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            for (int w = 0; w < NWS; ++w, ++wg) {
                const int slot = wg & 1;
                const uint32_t ph = (wg >> 1) & 1;
                const int xs = p.xres ? 0 : (int)(wg % (uint32_t)p.xst);
                if (!p.xres) {
                    ok = __all_sync(0xffffffffu,
                                    ptx::mbar_wait(&s.xfull[xs], (wg / p.xst) & 1, s.abort, WAIT_NS, 1));
                    if (!ok) break;
                }
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.afull[slot], ph, s.abort, WAIT_NS, 2));
                if (!ok) break;
                // the epilogue has read this slot's accumulators (stage wg - 2)
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.dfree[slot], ph ^ 1, s.abort, WAIT_NS, 3));
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t a_blk = tbase + (uint32_t)(slot * ACOLS);
                const uint32_t d_blk = d_tmem + (uint32_t)(slot * GPS * NT);
                for (int j = 0; j < SUB; ++j) {
                    const int kb = w * SUB + j;
                    if (kb >= KBLK) break;
                    const uint64_t bdesc = ptx::smem_desc_sw128(ptx::smem_u32(
                        p.xres ? s.xs + (size_t)kb * NT * 128 : s.xs + ((size_t)xs * SUB + j) * NT * 128));
#pragma unroll
                    for (int kk = 0; kk < KB / 16; ++kk) {
                        const int ks = j * KB + 16 * kk;            // code offset within the stage
                        const uint32_t lg = (uint32_t)(ks >> p.log2g);  // group within the stage
                        const bool gstart = (ks & (G - 1)) == 0;
                        // descriptor start address advances 32 bytes (2 units of 16 B) per K = 16 step
                        if (leader)
                            ptx::mma_ts(d_blk + lg * NT, a_blk + (uint32_t)(j * 32 + kk * 8), bdesc + (uint64_t)(2 * kk),
                                        p.idesc, gstart ? 0u : 1u);
                    }
                }
                if (leader) {
                    ptx::mma_commit(&s.sdone[slot]);
                    if (!p.xres) ptx::mma_commit(&s.xfree[xs]);
                }
            }
        }
        if (!ok && leader) raise_abort(s.abort);
        // every MMA this warp issued must retire before tensor memory is freed
        if (leader) {
            ptx::mma_commit(s.mdone);
            volatile int never = 0;
            ptx::mbar_wait(s.mdone, 0, &never, 200000000ull);
        }
        __syncwarp();
    } else {
        // ======================= code expanders + epilogue =======================
        const int q = warp & 3;                 // TMEM lane quarter
        const int h = (warp - 2) >> 2;          // which 32 codes of each 64 / which half of the tokens
        const int row = 32 * q + lane;          // W row within the tile == TMEM lane
        const int tid = threadIdx.x - 64;       // 0..255
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        uint32_t wg = 0, xph = 0;
        int unit = 0;
        bool ok = true;
        int64_t cur_x0 = -1;
        int cur_b = -1, cur_tv = -1;
        float2 acc[H / 2];

        if (has_tiles) {
            const TileInfo t0 = tile_info<NT>(p, s, blockIdx.x);
            issue_sb_chunk(p, t0, 0, s.sb, tid);
        }
        ptx::cp_async_commit();
        const uint16_t* sbslot = s.sb;
        int g_chunk0 = 0;

        // fold the groups of W stage `wl` (global stage counter wgE) of tile `ti` into acc
        auto epilogue_stage = [&](uint32_t wgE, int wl, const TileInfo& ti, int t) -> bool {
            if (wl % p.cs_w == 0) {
                // this stage opens a scale/bias chunk: its copies were issued a chunk earlier
                ptx::cp_async_wait_all();
                ptx::mbar_arrive(&s.sbar[unit & 1]);
                if (!__all_sync(0xffffffffu,
                                ptx::mbar_wait(&s.sbar[unit & 1], (unit >> 1) & 1, s.abort, WAIT_NS, 7)))
                    return false;
                sbslot = s.sb + (unit & 1) * 2 * 128 * SCP;
                const int c = wl / p.cs_w;
                g_chunk0 = c * SCW;
                uint16_t* nslot = s.sb + ((unit + 1) & 1) * 2 * 128 * SCP;
                if (c + 1 < NCH) {
                    issue_sb_chunk(p, ti, c + 1, nslot, tid);
                } else if (t + (int)gridDim.x < ntiles) {
                    const TileInfo tn = tile_info<NT>(p, s, t + gridDim.x);
                    issue_sb_chunk(p, tn, 0, nslot, tid);
                }
                ptx::cp_async_commit();
                ++unit;
            }
            const int slot = wgE & 1;
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(&s.sdone[slot], (wgE >> 1) & 1, s.abort, WAIT_NS, 6)))
                return false;
            ptx::tc_fence_after();
            for (int lg = 0; lg < GPS; ++lg) {
                const int g = wl * GPS + lg;
                if (g >= NG) break;
                const int gl = g - g_chunk0;
                const float sv = half_bits_to_float(sbslot[row * SCP + gl], XT{});
                const float bv = half_bits_to_float(sbslot[128 * SCP + row * SCP + gl], XT{});
                const float2 s2 = make_float2(sv, sv), b2 = make_float2(bv, bv);
                const float* xg = s.xtab + g * NT + h * H;
                const uint32_t dcol = d_tmem + (uint32_t)((slot * GPS + lg) * NT + h * H);
                uint32_t v[16];
                if constexpr (H >= 16) ptx::tmem_ld16(dcol + lane_base, v);
                else ptx::tmem_ld8(dcol + lane_base, v);
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
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&s.dfree[slot]);
            return true;
        };

        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const TileInfo ti = tile_info<NT>(p, s, t);
            // ---- sums of x for this token tile (rebuilt only when the tokens change) ----
            const int bkey = ti.b0 * 65536 + ti.b1;
            if (ti.xrow0 != cur_x0 || bkey != cur_b || ti.tvalid != cur_tv) {
                ptx::mbar_arrive(s.xbar);  // everyone is done reading the previous table
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(s.xbar, xph & 1, s.abort, WAIT_NS, 8));
                ++xph;
                if (!ok) break;
                build_xtab<XT, NT>(p, ti, s.xtab, tid);
                ptx::mbar_arrive(s.xbar);
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(s.xbar, xph & 1, s.abort, WAIT_NS, 8));
                ++xph;
                if (!ok) break;
                cur_x0 = ti.xrow0;
                cur_b = bkey;
                cur_tv = ti.tvalid;
            }
#pragma unroll
            for (int i = 0; i < H / 2; ++i) acc[i] = make_float2(0.0f, 0.0f);
            for (int w = 0; w < NWS && ok; ++w, ++wg) {
                const int st = wg % S;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.wfull[st], (wg / S) & 1, s.abort, WAIT_NS, 4));
                if (!ok) break;
                // A block wg & 1 was last read by the MMAs of stage wg - 2, whose completion the
                // epilogue of that stage has already waited for (it ran before this expansion)
                const uint8_t* wstage = s.ws + (size_t)st * 128 * p.rowb;
                const uint32_t a_blk = tbase + lane_base + (uint32_t)((wg & 1) * ACOLS);
                for (int j = 0; j < SUB; ++j) {
                    if (w * SUB + j >= KBLK) break;
                    uint32_t wv[BITS];
                    load_w32<BITS>(wstage, p.rowb, p.swz, row, j, h, wv);
                    uint32_t out[16];
                    expand32<BITS, XT>(wv, out);
                    ptx::tmem_st16(a_blk + (uint32_t)(j * 32 + 16 * h), out);
                }
                ptx::tc_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    ptx::mbar_arrive(&s.wfree[st]);
                    ptx::mbar_arrive(&s.afull[wg & 1]);
                }
                // fold the previous stage while this one is being multiplied
                if (w > 0) {
                    ok = epilogue_stage(wg - 1, w - 1, ti, t);
                    if (!ok) break;
                }
            }
            if (!ok) break;
            ok = epilogue_stage(wg - 1, NWS - 1, ti, t);
            if (!ok) break;
            // ---- store this thread's row of y for its half of the tokens ----
            if (row < ti.nvalid) {
                const int64_t n = ti.n0 + row;
                int64_t off = ti.xrow0 * p.y_row + n;
                if (!p.offsets) off += (int64_t)ti.b0 * p.yb[0] + (int64_t)ti.b1 * p.yb[1];
#pragma unroll
                for (int i = 0; i < H / 2; ++i) {
                    const int tok = h * H + 2 * i;
                    if (tok < ti.tvalid) store_y(p.y, off + (int64_t)tok * p.y_row, acc[i].x, p.ydt, XT{});
                    if (tok + 1 < ti.tvalid) store_y(p.y, off + (int64_t)(tok + 1) * p.y_row, acc[i].y, p.ydt, XT{});
                }
            }
        }
        ptx::cp_async_wait_all();
        if (!ok) raise_abort(s.abort);
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tbase, p.tmem_cols);
    }
#ifdef AQ_TRACE
    if (threadIdx.x < 64) atomicAdd(&::aq_trace_ns[threadIdx.x], ::aq_trace_smem[threadIdx.x]);
#endif
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

int num_sms() {
    static int n[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    if (n[dev] == 0) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        n[dev] = v > 0 ? v : 148;
    }
    return n[dev];
}

// tokens per tile: 16 or 32 (more tokens take more token tiles)
int pick_nt(const MmaProblem& p) {
    int64_t m = p.M;
    if (p.offsets) m = 2 * ((p.M + p.n_experts - 1) / p.n_experts);
    return m <= 16 ? 16 : 32;
}

#ifdef AQ_TRACE
constexpr size_t SMEM_LIMIT = 226 * 1024;  // the trace counters take static shared memory
#else
constexpr size_t SMEM_LIMIT = 227 * 1024;
#endif
constexpr int MIN_STAGES = 3;

// W stage geometry: WSC codes per row per stage, at most 4 groups per stage and a row of at most
// one 128-byte swizzle atom (two A blocks plus 2 x 4 accumulators of 32 columns fill 512 columns).
struct Geom {
    int wsc, rowb, sub, gps;
    uint32_t swz;
    CUtensorMapSwizzle tma_swz;
};
Geom geometry(int bits, int group) {
    Geom g;
    int wsc = bits == 6 ? 128 : 1024 / bits;
    if (wsc > 256) wsc = 256;
    if (wsc > 4 * group) wsc = 4 * group;
    g.wsc = wsc;
    g.rowb = wsc * bits / 8;
    g.sub = wsc / KB;
    g.gps = wsc / group;
    switch (g.rowb) {
        case 128: g.swz = 7; g.tma_swz = CU_TENSOR_MAP_SWIZZLE_128B; break;
        case 64: g.swz = 3; g.tma_swz = CU_TENSOR_MAP_SWIZZLE_64B; break;
        case 32: g.swz = 1; g.tma_swz = CU_TENSOR_MAP_SWIZZLE_32B; break;
        default: g.swz = 0; g.tma_swz = CU_TENSOR_MAP_SWIZZLE_NONE; break;
    }
    return g;
}

// x in shared memory: all of K when resident, else `xst` x stages of SUB boxes
size_t fixed_bytes(int nt, int64_t K, int64_t kg, int xres, int xst, const Geom& g) {
    return (xres ? (size_t)(K / KB) * nt * 128 : (size_t)xst * g.sub * nt * 128) + (size_t)kg * nt * 4 +
           smem_fixed_bytes();
}
size_t smem_for(int nt, int stages, int64_t K, int64_t kg, int xres, int xst, const Geom& g) {
    return (size_t)stages * 128 * g.rowb + fixed_bytes(nt, K, kg, xres, xst, g);
}
int pick_stages(int nt, int64_t K, int64_t kg, int xres, int xst, const Geom& g) {
    const size_t fixed = fixed_bytes(nt, K, kg, xres, xst, g);
    if (fixed >= SMEM_LIMIT) return 0;
    int st = (int)((SMEM_LIMIT - fixed) / ((size_t)128 * g.rowb));
    if (st > MAX_STAGES) st = MAX_STAGES;
    return st;
}
// x stays resident when a CTA sees one token tile and that leaves a deep enough W pipeline;
// otherwise the deepest x ring (<= 4) that keeps at least 4 W stages
struct XPlan {
    int xres, xst, stages;
};
XPlan pick_x(const MmaProblem& p, int nt, int64_t kg, const Geom& g) {
    XPlan r{0, 2, 0};
    if (!p.offsets && p.M <= nt && p.nb[0] * p.nb[1] == 1 && pick_stages(nt, p.K, kg, 1, 0, g) >= 6) {
        r.xres = 1;
        r.xst = 0;
    } else {
        for (int xst = MAX_XST; xst > 2; --xst)
            if (pick_stages(nt, p.K, kg, 0, xst, g) >= 4) {
                r.xst = xst;
                break;
            }
    }
    r.stages = pick_stages(nt, p.K, kg, r.xres, r.xst, g);
    return r;
}

template <int BITS, typename XT, int NT>
cudaError_t launch_t(const MmaParams& prm, int grid, size_t smem, cudaStream_t s) {
    static std::mutex mu;
    static bool done[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!done[dev]) {
            e = cudaFuncSetAttribute(qmm_tc_kernel<BITS, XT, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)SMEM_LIMIT);
            if (e != cudaSuccess) return e;
            done[dev] = true;
        }
    }
    qmm_tc_kernel<BITS, XT, NT><<<grid, MMA_THREADS, smem, s>>>(prm);
    return cudaGetLastError();
}

template <int BITS, typename XT>
cudaError_t launch_nt(int nt, const MmaParams& prm, int grid, size_t smem, cudaStream_t s) {
    return nt == 16 ? launch_t<BITS, XT, 16>(prm, grid, smem, s) : launch_t<BITS, XT, 32>(prm, grid, smem, s);
}

template <typename XT>
cudaError_t launch_bits(int bits, int nt, const MmaParams& prm, int grid, size_t smem, cudaStream_t s) {
    switch (bits) {
        case 2: return launch_nt<2, XT>(nt, prm, grid, smem, s);
        case 4: return launch_nt<4, XT>(nt, prm, grid, smem, s);
        case 6: return launch_nt<6, XT>(nt, prm, grid, smem, s);
        case 8: return launch_nt<8, XT>(nt, prm, grid, smem, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

bool mma_supported(const MmaProblem& p, const char** why) {
    auto no = [&](const char* r) { if (why) *why = r; return false; };
    if (!(p.bits == 2 || p.bits == 4 || p.bits == 6 || p.bits == 8)) return no("tensor-core kernel takes bits 2/4/6/8");
    if (p.K < KB || p.K % KB != 0) return no("K must be a multiple of 64 for the tensor-core kernel");
    if (((uintptr_t)p.x & 15) || (p.M > 1 && p.x_row % 8 != 0)) return no("x rows not 16-byte aligned");
    for (int i = 0; i < 2; ++i)
        if (p.nb[i] > 1 && p.xb[i] % 8 != 0) return no("x batch strides not 16-byte aligned");
    if (((uintptr_t)p.wq & 15) || (p.w_row * 4) % 16 != 0) return no("W rows not 16-byte aligned");
    const int64_t kg = p.K / p.group;
    if (kg % 2 != 0) return no("K/group must be even for the tensor-core kernel");
    if (((uintptr_t)p.scales & 3) || ((uintptr_t)p.biases & 3)) return no("scales/biases not 4-byte aligned");
    if (p.offsets) {
        if (p.n_experts > MAX_EXPERTS) return no("too many experts");
        if (p.w_expert != p.N * p.w_row) return no("expert bank rows must be contiguous");
        if (p.s_expert != p.N * kg || p.b_expert != p.N * kg) return no("scale/bias bank rows must be contiguous");
    }
    if (p.M > INT32_MAX / 2 || p.N * (p.offsets ? p.n_experts : 1) > INT32_MAX / 2)
        return no("problem too large for 32-bit tile coordinates");
    const int nt = pick_nt(p);
    const Geom g = geometry(p.bits, p.group);
    if ((size_t)kg * nt * 4 > XTAB_MAX_BYTES || pick_stages(nt, p.K, kg, 0, 2, g) < MIN_STAGES)
        return no("K/group too large for the sum-of-x table of the tensor-core kernel");
    if (!get_encode()) return no("driver entry point cuTensorMapEncodeTiled unavailable");
    return true;
}

cudaError_t launch_mma(const MmaProblem& pb, cudaStream_t stream) {
    auto encode = get_encode();
    if (!encode) return cudaErrorNotSupported;
    MmaParams prm;
    memset(&prm, 0, sizeof prm);
    const int nt = pick_nt(pb);
    const int bits = pb.bits;
    const int64_t kg = pb.K / pb.group;
    const Geom geo = geometry(bits, pb.group);
    const XPlan xp = pick_x(pb, nt, kg, geo);
    const int stages = xp.stages;
    if (stages < MIN_STAGES) return cudaErrorInvalidValue;
    const int64_t rows_total = pb.M;
    // ---- x tensor map: {K, rows, nb1, nb0}
    {
        cuuint64_t dims[4] = {(cuuint64_t)pb.K, (cuuint64_t)rows_total, (cuuint64_t)pb.nb[1], (cuuint64_t)pb.nb[0]};
        const int64_t rowb = rows_total > 1 ? pb.x_row * 2 : (pb.K * 2 + 15) / 16 * 16;
        const int64_t s1 = pb.nb[1] > 1 ? pb.xb[1] * 2 : rowb * rows_total;
        const int64_t s2 = pb.nb[0] > 1 ? pb.xb[0] * 2 : s1 * (int64_t)pb.nb[1];
        cuuint64_t strides[3] = {(cuuint64_t)rowb, (cuuint64_t)((s1 + 15) / 16 * 16), (cuuint64_t)((s2 + 15) / 16 * 16)};
        cuuint32_t box[4] = {64, (cuuint32_t)nt, 1, 1};
        cuuint32_t estr[4] = {1, 1, 1, 1};
        CUresult r = encode(&prm.tx, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, const_cast<void*>(pb.x), dims, strides, box,
                            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    // ---- W tensor map: {K*bits/32 words, rows}, box {rowb/4 words, 128 rows}
    {
        const int64_t wrows = pb.offsets ? pb.N * pb.n_experts : pb.N;
        cuuint64_t dims[2] = {(cuuint64_t)(pb.K * bits / 32), (cuuint64_t)wrows};
        cuuint64_t strides[1] = {(cuuint64_t)(pb.w_row * 4)};
        cuuint32_t box[2] = {(cuuint32_t)(geo.rowb / 4), 128};
        cuuint32_t estr[2] = {1, 1};
        CUresult r = encode(&prm.tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(pb.wq), dims, strides,
                            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, geo.tma_swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    prm.x = pb.x;
    prm.y = pb.y;
    prm.scales = (const uint16_t*)pb.scales;
    prm.biases = (const uint16_t*)pb.biases;
    prm.M = pb.M;
    prm.N = pb.N;
    prm.K = pb.K;
    prm.x_row = pb.x_row;
    prm.y_row = pb.y_row;
    prm.xb[0] = pb.xb[0];
    prm.xb[1] = pb.xb[1];
    prm.yb[0] = pb.yb[0];
    prm.yb[1] = pb.yb[1];
    prm.nb1 = pb.nb[1];
    prm.n_wtiles = (int)((pb.N + 127) / 128);
    prm.n_ttiles = (int)((pb.M + nt - 1) / nt);
    prm.nbatch = (int)(pb.nb[0] * pb.nb[1]);
    prm.group = pb.group;
    int lg = 0;
    while ((1 << lg) < pb.group) ++lg;
    prm.log2g = lg;
    prm.kg = (int)kg;
    prm.ydt = (int)pb.ydt;
    prm.wsc = geo.wsc;
    prm.rowb = geo.rowb;
    prm.sub = geo.sub;
    prm.gps = geo.gps;
    prm.swz = geo.swz;
    prm.n_wstages = (int)((pb.K + geo.wsc - 1) / geo.wsc);
    prm.stages = stages;
    prm.cs_w = SCW / geo.gps;
    prm.xres = xp.xres;
    prm.xst = xp.xst;
    uint32_t cols = (uint32_t)(geo.wsc + 2 * geo.gps * nt), pw = 32;
    while (pw < cols) pw <<= 1;
    prm.tmem_cols = pw;
    prm.idesc = ptx::idesc_f16(nt, pb.xdt == DT::BF16 ? 1 : 0);
    prm.offsets = pb.offsets;
    prm.n_experts = pb.n_experts;

    const int sms = num_sms();
    int grid;
    if (pb.offsets) {
        grid = sms;
    } else {
        const int64_t tiles = (int64_t)prm.n_wtiles * prm.n_ttiles * prm.nbatch;
        grid = (int)(tiles < sms ? tiles : sms);
    }
    const size_t smem = smem_for(nt, stages, pb.K, kg, xp.xres, xp.xst, geo);
    if (pb.xdt == DT::BF16) return launch_bits<bf16_t>(bits, nt, prm, grid, smem, stream);
    return launch_bits<f16_t>(bits, nt, prm, grid, smem, stream);
}

#ifdef AQ_TRACE
extern "C" __attribute__((visibility("default"))) int aq_trace_read(unsigned long long* out, int reset) {
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    if (cudaMemcpyFromSymbol(out, ::aq_trace_ns, sizeof(unsigned long long) * 64) != cudaSuccess) return -1;
    if (reset) {
        unsigned long long z[64] = {0};
        if (cudaMemcpyToSymbol(::aq_trace_ns, z, sizeof z) != cudaSuccess) return -1;
    }
    return 0;
}
#endif

cudaError_t read_and_clear_device_error(int* value, cudaStream_t s) {
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
}

}  // namespace aq
