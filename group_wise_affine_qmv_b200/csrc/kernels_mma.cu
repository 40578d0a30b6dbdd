// kernels_mma.cu -- tensor-core kernel for y = x . dequant(W)^T on sm_100a (tcgen05 / TMEM).
//
// The contraction is done "weights-stationary": a tile of 128 rows of W is
// the MMA's M side, the tokens of x (16..256 per tile) are its N side, so the
// same kernel serves decode batches (tens of tokens) and prefill (hundreds).
//
//   warp 0      TMA producer: per 64-code stage, the x tile [NT tokens x 64]
//               (128-byte swizzled, K-major: the UMMA B operand) and the packed
//               W tile [128 rows x 64 codes], onto one mbarrier.
//   warp 1      MMA issuer: tcgen05.mma kind::f16, A from tensor memory
//               (dequantized W), B from shared memory (x), fp32 accumulator
//               D [128 x NT] in tensor memory; tcgen05.commit releases stages.
//   warps 2..9  dequantizers: thread <-> W row (TMEM lane), two warps per lane
//               quarter split each stage's 64 codes; w' = s*q + b rounded once
//               to bf16/f16 is written with tcgen05.st into an A slot.  The
//               same warps run the epilogue (tcgen05.ld of D, convert, store y).
//
// Dequantizing into tensor memory instead of shared memory keeps the
// shared-memory traffic at the packed weights plus the x tile; the per-group
// scales/biases of a tile are brought in with asynchronous 4-byte copies.
//
// Rows of the last W tile that fall past N are read as TMA zero fill (or as
// the clamped last row's scale/bias) and simply not stored: no per-row check
// inside the K loop (the partial-rows idea of "mlx PR #4516").
//
// Every mbarrier wait is bounded (2 s); on expiry the CTA raises an abort
// flag, records an error word readable through aq_device_error(), drains its
// own outstanding copies (bounded), frees its tensor memory and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "aq_internal.h"
#include "device_common.cuh"
#include "sm100_ptx.cuh"

namespace aq {

__device__ int g_device_error = 0;

namespace {

constexpr int MMA_THREADS = 320;          // 10 warps
constexpr int DQ_THREADS = 256;           // warps 2..9
constexpr int KB = 64;                    // codes per pipeline stage
constexpr int SA = 4;                     // A slots in tensor memory, 32 columns each
constexpr int SCW = 32;                   // groups per scale/bias chunk
constexpr int SCP = SCW + 2;              // padded row pitch (halves) of a chunk in shared memory
constexpr int MAX_STAGES = 16;
constexpr int MAX_EXPERTS = 1024;
constexpr uint64_t WAIT_NS = 2000000000ull;  // 2 s per wait
constexpr int ERR_TIMEOUT = 1;

struct MmaParams {
    CUtensorMap tx;  // x: 4D {K, rows, nb1, nb0} u16, box {64, nt, 1, 1}, 128B swizzle
    CUtensorMap tw;  // W: 2D {K*bits/32, rows} u32, box {2*bits, 128}
    void* y;
    const uint16_t* scales;
    const uint16_t* biases;
    int64_t M, N, K;
    int64_t y_row;
    int64_t yb[2];
    int64_t nb1;
    int nt;
    int n_wtiles, n_ttiles, nbatch;
    int log2g;
    int stages;
    int kg;              // groups per row = K / group
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
    int64_t xrow0;   // first x row (token) coordinate
    int tvalid;      // valid tokens in this tile
    int b0, b1;      // launch batch (non-grouped)
};

struct Smem {
    uint64_t* full;
    uint64_t* empty;
    uint64_t* afull;
    uint64_t* aempty;
    uint64_t* dfull;
    uint64_t* sbar;      // [2] scale/bias chunk slots: 256 dequant-thread arrivals
    uint64_t* mdone;     // all MMAs of this CTA retired (teardown)
    uint32_t* tmem_base;
    int* abort;
    int* prefix;     // grouped: tile prefix sums [n_experts + 1]
    uint8_t* xs;     // stages * nt * 128
    uint8_t* ws;     // stages * 1024 * bits
    uint16_t* sb;    // [2 slots][2 arrays][128][SCP]
};

template <int BITS>
__device__ __forceinline__ Smem carve(uint8_t* base, const MmaParams& p) {
    Smem s;
    uint8_t* q = base;
    s.xs = q;
    q += (size_t)p.stages * p.nt * 128;
    s.ws = q;
    q += (size_t)p.stages * 1024 * BITS;
    s.sb = reinterpret_cast<uint16_t*>(q);
    q += 2 * 2 * 128 * SCP * 2;
    s.full = reinterpret_cast<uint64_t*>(q);
    s.empty = s.full + MAX_STAGES;
    s.afull = s.empty + MAX_STAGES;
    s.aempty = s.afull + SA;
    s.dfull = s.aempty + SA;
    s.sbar = s.dfull + 1;
    s.mdone = s.sbar + 2;
    s.tmem_base = reinterpret_cast<uint32_t*>(s.mdone + 1);
    s.abort = reinterpret_cast<int*>(s.tmem_base + 1);
    s.prefix = s.abort + 1;
    return s;
}

__host__ __device__ constexpr size_t smem_fixed_bytes() {
    return 2 * 2 * 128 * SCP * 2 + (2 * MAX_STAGES + 2 * SA + 4) * 8 + 8 + (MAX_EXPERTS + 1) * 4 + 1024 /*align*/;
}

__device__ __forceinline__ void raise_abort(int* abort) {
    *(volatile int*)abort = 1;
    atomicExch(&g_device_error, ERR_TIMEOUT);
}

// total number of tiles (grouped mode reads the prefix sums in shared memory)
__device__ __forceinline__ int total_tiles(const MmaParams& p, const Smem& s) {
    if (p.offsets) return s.prefix[p.n_experts];
    return p.n_wtiles * p.n_ttiles * p.nbatch;
}

__device__ __forceinline__ TileInfo tile_info(const MmaParams& p, const Smem& s, int t) {
    TileInfo ti;
    if (p.offsets) {
        // expert e with prefix[e] <= t < prefix[e+1]
        int lo = 0, hi = p.n_experts;
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
        ti.xrow0 = off + (int64_t)tt * p.nt;
        ti.tvalid = (int)min64(p.nt, cnt - (int64_t)tt * p.nt);
        ti.b0 = ti.b1 = 0;
    } else {
        const int wt = t % p.n_wtiles;
        const int rest = t / p.n_wtiles;
        const int tt = rest % p.n_ttiles;
        const int b = rest / p.n_ttiles;
        ti.n0 = (int64_t)wt * 128;
        ti.wrow0 = ti.n0;
        ti.nvalid = (int)min64(128, p.N - ti.n0);
        ti.xrow0 = (int64_t)tt * p.nt;
        ti.tvalid = (int)min64(p.nt, p.M - ti.xrow0);
        ti.b1 = (int)(b % p.nb1);
        ti.b0 = (int)(b / p.nb1);
    }
    return ti;
}

// ---------------------------------------------------------------------------
// dequantization of one thread's 32 codes into 16 packed A-operand pairs
// ---------------------------------------------------------------------------

// swizzled byte offset of a 16-byte chunk written by TMA (bits 4.. XOR bits 7..)
template <int BITS>
__device__ __forceinline__ uint32_t wswz(uint32_t off) {
    if constexpr (BITS == 4) return off ^ (((off >> 7) & 1u) << 4);   // 32-byte swizzle
    else if constexpr (BITS == 8) return off ^ (((off >> 7) & 3u) << 4);  // 64-byte swizzle
    else return off;
}

template <int BITS>
__device__ __forceinline__ void load_w32(const uint8_t* stage, int row, int h, uint32_t* w) {
    constexpr uint32_t RB = 8 * BITS;  // bytes per row per stage (64 codes)
    const uint32_t base = (uint32_t)row * RB + (uint32_t)h * (RB / 2);
    if constexpr (BITS == 4) {
        const uint4 v = *reinterpret_cast<const uint4*>(stage + wswz<4>(base));
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (BITS == 8) {
        const uint4 v0 = *reinterpret_cast<const uint4*>(stage + wswz<8>(base));
        const uint4 v1 = *reinterpret_cast<const uint4*>(stage + wswz<8>(base + 16));
        w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
        w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
    } else {
#pragma unroll
        for (int i = 0; i < BITS / 2; ++i) {
            const uint2 v = *reinterpret_cast<const uint2*>(stage + base + 8 * i);
            w[2 * i] = v.x; w[2 * i + 1] = v.y;
        }
    }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi, bf16_t) {
    const __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi, f16_t) {
    const __half2 r = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&r);
}

// (offset + q) pairs to s*q + b, rounded once, in the 16-bit type
__device__ __forceinline__ uint32_t affine2(uint32_t qo, uint32_t s2, uint32_t b2, uint32_t off2, bf16_t) {
    const __nv_bfloat162 q = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&qo),
                                     *reinterpret_cast<const __nv_bfloat162*>(&off2));
    const __nv_bfloat162 r = __hfma2(*reinterpret_cast<const __nv_bfloat162*>(&s2), q,
                                     *reinterpret_cast<const __nv_bfloat162*>(&b2));
    return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t affine2(uint32_t qo, uint32_t s2, uint32_t b2, uint32_t off2, f16_t) {
    const __half2 q = __hsub2(*reinterpret_cast<const __half2*>(&qo), *reinterpret_cast<const __half2*>(&off2));
    const __half2 r = __hfma2(*reinterpret_cast<const __half2*>(&s2), q, *reinterpret_cast<const __half2*>(&b2));
    return *reinterpret_cast<const uint32_t*>(&r);
}

template <int BITS, typename XT>
__device__ __forceinline__ void dequant32(const uint32_t* w, uint16_t sbits, uint16_t bbits, uint32_t* out) {
    const uint32_t s2 = (uint32_t)sbits | ((uint32_t)sbits << 16);
    const uint32_t b2 = (uint32_t)bbits | ((uint32_t)bbits << 16);
    constexpr bool BF = std::is_same<XT, bf16_t>::value;
    if constexpr (BITS == 4) {
        // byte j of a word holds codes (2j, 2j+1); the word shifted by 4 holds code 2j+1 in
        // the low nibble of byte j.  PRMT gathers both into the two halves, LOP3 makes
        // (offset + q) in each half: 128 + q in bf16 (0x4300 | q), 1024 + q in f16 (0x6400 | q).
        constexpr uint32_t MAGIC = BF ? 0x43004300u : 0x64006400u;
        constexpr uint32_t OFF2 = MAGIC;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t word = w[i], shifted = w[i] >> 4;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t t = __byte_perm(word, shifted, j | (j << 4) | ((4 + j) << 8) | ((4 + j) << 12));
                const uint32_t qo = (t & 0x000F000Fu) | MAGIC;
                out[4 * i + j] = affine2(qo, s2, b2, OFF2, XT{});
            }
        }
    } else if constexpr (BITS == 8 && !BF) {
        // f16: 1024 + q is exact for every 8-bit code
#pragma unroll
        for (int i = 0; i < 8; ++i) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const uint32_t qo = __byte_perm(w[i], 0x64006400u, (2 * j) | (5 << 4) | ((2 * j + 1) << 8) | (7 << 12));
                out[2 * i + j] = affine2(qo, s2, b2, 0x64006400u, XT{});
            }
        }
    } else if constexpr (BITS == 8) {
        // bf16 cannot hold 128 + q for q >= 128: go through fp32 (2^23 + q is exact there)
        const float s = __uint_as_float((uint32_t)sbits << 16), b = __uint_as_float((uint32_t)bbits << 16);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const float q0 = __uint_as_float(__byte_perm(w[i], 0x4B000000u, (2 * j) | (4 << 4) | (5 << 8) | (7 << 12))) - 8388608.0f;
                const float q1 = __uint_as_float(__byte_perm(w[i], 0x4B000000u, (2 * j + 1) | (4 << 4) | (5 << 8) | (7 << 12))) - 8388608.0f;
                out[2 * i + j] = pack2(fmaf(s, q0, b), fmaf(s, q1, b), XT{});
            }
        }
    } else {
        // generic width (2, 6): funnel-shift extraction, fp32 affine, one rounding
        const float s = half_bits_to_float(sbits, XT{}), b = half_bits_to_float(bbits, XT{});
        constexpr uint32_t MASK = (1u << BITS) - 1u;
        uint32_t ww[BITS + 1];
#pragma unroll
        for (int i = 0; i < BITS; ++i) ww[i] = w[i];
        ww[BITS] = 0;
#pragma unroll
        for (int pr = 0; pr < 16; ++pr) {
            float v[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int pos = (2 * pr + e) * BITS;
                const int wi = pos >> 5, sh = pos & 31;
                const uint32_t q = __funnelshift_r(ww[wi], ww[wi + 1], sh) & MASK;
                v[e] = fmaf(s, (float)q, b);
            }
            out[pr] = pack2(v[0], v[1], XT{});
        }
    }
}

// ---------------------------------------------------------------------------
// scale/bias chunk loads (dequant warps, asynchronous 4-byte copies)
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

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
template <int BITS, typename XT, typename YT>
__global__ void __launch_bounds__(MMA_THREADS, 1) qmm_tc_kernel(const __grid_constant__ MmaParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const Smem s = carve<BITS>(base, p);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.stages;
    const int KBLK = (int)(p.K / KB);
    const int CS = (SCW << p.log2g) / KB;   // stages per scale/bias chunk
    const int NCH = (p.kg + SCW - 1) / SCW; // chunks per tile

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            ptx::mbar_init(&s.full[i], 1);
            ptx::mbar_init(&s.empty[i], 1);
        }
        for (int i = 0; i < SA; ++i) {
            ptx::mbar_init(&s.afull[i], 8);
            ptx::mbar_init(&s.aempty[i], 1);
        }
        ptx::mbar_init(s.dfull, 1);
        ptx::mbar_init(&s.sbar[0], DQ_THREADS);
        ptx::mbar_init(&s.sbar[1], DQ_THREADS);
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
        // tiles per expert: ceil(count / nt) * n_wtiles, prefix-summed
        if (lane == 0) s.prefix[0] = 0;
        __syncwarp();
        int carry = 0;
        for (int e0 = 0; e0 < p.n_experts; e0 += 32) {
            const int e = e0 + lane;
            int v = 0;
            if (e < p.n_experts) {
                const int64_t cnt = p.offsets[e + 1] - p.offsets[e];
                v = (int)((cnt + p.nt - 1) / p.nt) * p.n_wtiles;
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
    const uint32_t d_tmem = tbase + SA * 32;  // accumulator columns follow the A slots
    const int ntiles = total_tiles(p, s);

    if (warp == 0) {
        // ======================= TMA producer =======================
        if (lane == 0) {
            const uint32_t xbytes = (uint32_t)p.nt * 128;
            const uint32_t wbytes = 1024u * BITS;
            uint32_t it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                const TileInfo ti = tile_info(p, s, t);
                for (int kb = 0; kb < KBLK; ++kb, ++it) {
                    const int st = it % S;
                    const uint32_t ph = (it / S) & 1;
                    if (!ptx::mbar_wait(&s.empty[st], ph ^ 1, s.abort, WAIT_NS)) { ok = false; break; }
                    ptx::mbar_arrive_expect_tx(&s.full[st], xbytes + wbytes);
                    ptx::tma_load_4d(s.xs + (size_t)st * p.nt * 128, &p.tx, &s.full[st], kb * KB, (int32_t)ti.xrow0,
                                     ti.b1, ti.b0);
                    ptx::tma_load_2d(s.ws + (size_t)st * 1024 * BITS, &p.tw, &s.full[st], kb * 2 * BITS,
                                     (int32_t)ti.wrow0);
                }
            }
            if (!ok) {
                raise_abort(s.abort);
                // drain: the copies of every issued stage must land before the CTA exits
                volatile int never = 0;
                const uint32_t first = it >= (uint32_t)S ? it - S : 0;
                for (uint32_t j = first; j < it; ++j)
                    ptx::mbar_wait(&s.full[j % S], (j / S) & 1, &never, 200000000ull);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ======================= MMA issuer =======================
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                for (int kb = 0; kb < KBLK; ++kb, ++it) {
                    const int st = it % S;
                    const uint32_t ph = (it / S) & 1;
                    const int a = it % SA;
                    const uint32_t aph = (it / SA) & 1;
                    if (!ptx::mbar_wait(&s.full[st], ph, s.abort, WAIT_NS) ||
                        !ptx::mbar_wait(&s.afull[a], aph, s.abort, WAIT_NS)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t xaddr = ptx::smem_u32(s.xs + (size_t)st * p.nt * 128);
#pragma unroll
                    for (int j = 0; j < KB / 16; ++j) {
                        const uint64_t bdesc = ptx::smem_desc_sw128(xaddr + 32 * j);
                        ptx::mma_ts(d_tmem, tbase + a * 32 + j * 8, bdesc, p.idesc, (kb | j) != 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(&s.empty[st]);
                    ptx::mma_commit(&s.aempty[a]);
                }
                if (ok) ptx::mma_commit(s.dfull);
            }
            if (!ok) raise_abort(s.abort);
            // every MMA this thread issued must retire before tensor memory is freed
            ptx::mma_commit(s.mdone);
            volatile int never = 0;
            ptx::mbar_wait(s.mdone, 0, &never, 200000000ull);
        }
        __syncwarp();
    } else {
        // ======================= dequantizers + epilogue =======================
        const int q = warp & 3;                 // TMEM lane quarter
        const int h = (warp - 2) >> 2;          // which 32 codes of each stage
        const int row = 32 * q + lane;          // W row within the tile == TMEM lane
        const int tid = threadIdx.x - 64;       // 0..255
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        uint32_t it = 0;
        int unit = 0;
        bool ok = true;
        // first scale/bias chunk of the first tile
        if (blockIdx.x < ntiles) {
            const TileInfo t0 = tile_info(p, s, blockIdx.x);
            issue_sb_chunk(p, t0, 0, s.sb, tid);
        }
        ptx::cp_async_commit();
        int tile_iter = 0;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++tile_iter) {
            const TileInfo ti = tile_info(p, s, t);
            const uint16_t* slot = s.sb;
            int g_chunk0 = 0;
            for (int kb = 0; kb < KBLK; ++kb, ++it) {
                if (kb % CS == 0) {
                    // this chunk's copies were issued one chunk earlier: each thread waits for its
                    // own, then the 256 dequant threads meet on the slot's mbarrier (release/acquire)
                    ptx::cp_async_wait_all();
                    ptx::mbar_arrive(&s.sbar[unit & 1]);
                    ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.sbar[unit & 1], (unit >> 1) & 1, s.abort, WAIT_NS));
                    if (!ok) break;
                    slot = s.sb + (unit & 1) * 2 * 128 * SCP;
                    g_chunk0 = (kb / CS) * SCW;
                    // prefetch the next chunk (this tile's next, or the next tile's first)
                    const int c = kb / CS;
                    uint16_t* nslot = s.sb + ((unit + 1) & 1) * 2 * 128 * SCP;
                    if (c + 1 < NCH) {
                        issue_sb_chunk(p, ti, c + 1, nslot, tid);
                    } else if (t + (int)gridDim.x < ntiles) {
                        const TileInfo tn = tile_info(p, s, t + gridDim.x);
                        issue_sb_chunk(p, tn, 0, nslot, tid);
                    }
                    ptx::cp_async_commit();
                    ++unit;
                }
                const int st = it % S;
                const uint32_t ph = (it / S) & 1;
                const int a = it % SA;
                const uint32_t aph = (it / SA) & 1;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.full[st], ph, s.abort, WAIT_NS));
                if (!ok) break;
                uint32_t wv[BITS];
                load_w32<BITS>(s.ws + (size_t)st * 1024 * BITS, row, h, wv);
                const int g = ((kb * KB + 32 * h) >> p.log2g) - g_chunk0;
                const uint16_t sbits = slot[row * SCP + g];
                const uint16_t bbits = slot[128 * SCP + row * SCP + g];
                uint32_t out[16];
                dequant32<BITS, XT>(wv, sbits, bbits, out);
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.aempty[a], aph ^ 1, s.abort, WAIT_NS));
                if (!ok) break;
                ptx::tmem_st16(tbase + lane_base + a * 32 + 16 * h, out);
                ptx::tc_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&s.afull[a]);
            }
            if (!ok) break;
            // ---- epilogue: D[128 x nt] -> y ----
            ok = __all_sync(0xffffffffu, ptx::mbar_wait(s.dfull, tile_iter & 1, s.abort, WAIT_NS));
            if (!ok) break;
            ptx::tc_fence_after();
            const int half = p.nt >> 1;
            const int c0 = h * half;
            const int64_t n = ti.n0 + row;
            const bool row_ok = row < ti.nvalid;
            YT* ybase;
            if (p.offsets) ybase = (YT*)p.y + ti.xrow0 * p.y_row + n;
            else ybase = (YT*)p.y + ti.b0 * p.yb[0] + ti.b1 * p.yb[1] + ti.xrow0 * p.y_row + n;
            for (int cc = 0; cc < half; cc += 8) {
                uint32_t v[8];
                ptx::tmem_ld8(d_tmem + lane_base + c0 + cc, v);
                ptx::tc_wait_ld();
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int tok = c0 + cc + e;
                    if (row_ok && tok < ti.tvalid) store_out(ybase + (int64_t)tok * p.y_row, __uint_as_float(v[e]));
                }
            }
            ptx::tc_fence_before();
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

int pick_nt(const MmaProblem& p) {
    int64_t m;
    if (p.offsets) {
        const int64_t avg = (p.M + p.n_experts - 1) / p.n_experts;
        m = 2 * avg;
        if (m > 128) m = 128;
    } else {
        m = p.M;
    }
    int64_t nt = (m + 15) / 16 * 16;
    if (nt < 16) nt = 16;
    if (nt > 256) nt = 256;
    return (int)nt;
}

size_t smem_for(int nt, int bits, int stages) {
    return (size_t)stages * ((size_t)nt * 128 + 1024 * (size_t)bits) + smem_fixed_bytes();
}

constexpr size_t SMEM_LIMIT = 227 * 1024;

int pick_stages(int nt, int bits) {
    const size_t per = (size_t)nt * 128 + 1024 * (size_t)bits;
    int st = (int)((SMEM_LIMIT - smem_fixed_bytes()) / per);
    if (st > MAX_STAGES) st = MAX_STAGES;
    return st;
}

template <int BITS, typename XT, typename YT>
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
            e = cudaFuncSetAttribute(qmm_tc_kernel<BITS, XT, YT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)SMEM_LIMIT);
            if (e != cudaSuccess) return e;
            done[dev] = true;
        }
    }
    qmm_tc_kernel<BITS, XT, YT><<<grid, MMA_THREADS, smem, s>>>(prm);
    return cudaGetLastError();
}

template <typename XT, typename YT>
cudaError_t launch_bits(int bits, const MmaParams& prm, int grid, size_t smem, cudaStream_t s) {
    switch (bits) {
        case 2: return launch_t<2, XT, YT>(prm, grid, smem, s);
        case 4: return launch_t<4, XT, YT>(prm, grid, smem, s);
        case 6: return launch_t<6, XT, YT>(prm, grid, smem, s);
        case 8: return launch_t<8, XT, YT>(prm, grid, smem, s);
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
    const int stages = pick_stages(nt, bits);
    const int64_t rows_total = pb.offsets ? pb.M : pb.M;
    // ---- x tensor map: {K, rows, nb1, nb0}
    {
        cuuint64_t dims[4] = {(cuuint64_t)pb.K, (cuuint64_t)rows_total, (cuuint64_t)pb.nb[1], (cuuint64_t)pb.nb[0]};
        const int64_t rowb = pb.x_row * 2;
        int64_t s1 = pb.nb[1] > 1 ? pb.xb[1] * 2 : rowb * (rows_total > 0 ? rows_total : 1);
        int64_t s2 = pb.nb[0] > 1 ? pb.xb[0] * 2 : s1 * (int64_t)pb.nb[1];
        if (rows_total <= 1) { /* a single row: any 16-byte multiple works as its stride */ }
        cuuint64_t strides[3] = {(cuuint64_t)(rows_total > 1 ? rowb : ((pb.K * 2 + 15) / 16 * 16)),
                                 (cuuint64_t)((s1 + 15) / 16 * 16), (cuuint64_t)((s2 + 15) / 16 * 16)};
        cuuint32_t box[4] = {64, (cuuint32_t)nt, 1, 1};
        cuuint32_t estr[4] = {1, 1, 1, 1};
        CUresult r = encode(&prm.tx, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, const_cast<void*>(pb.x), dims, strides, box,
                            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    // ---- W tensor map: {K*bits/32 words, rows}
    {
        const int64_t wrows = pb.offsets ? pb.N * pb.n_experts : pb.N;
        cuuint64_t dims[2] = {(cuuint64_t)(pb.K * bits / 32), (cuuint64_t)wrows};
        cuuint64_t strides[1] = {(cuuint64_t)(pb.w_row * 4)};
        cuuint32_t box[2] = {(cuuint32_t)(2 * bits), 128};
        cuuint32_t estr[2] = {1, 1};
        CUtensorMapSwizzle sw = bits == 4 ? CU_TENSOR_MAP_SWIZZLE_32B
                                : bits == 8 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE;
        CUresult r = encode(&prm.tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(pb.wq), dims, strides,
                            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    prm.y = pb.y;
    prm.scales = (const uint16_t*)pb.scales;
    prm.biases = (const uint16_t*)pb.biases;
    prm.M = pb.M;
    prm.N = pb.N;
    prm.K = pb.K;
    prm.y_row = pb.y_row;
    prm.yb[0] = pb.yb[0];
    prm.yb[1] = pb.yb[1];
    prm.nb1 = pb.nb[1];
    prm.nt = nt;
    prm.n_wtiles = (int)((pb.N + 127) / 128);
    prm.n_ttiles = (int)((pb.M + nt - 1) / nt);
    prm.nbatch = (int)(pb.nb[0] * pb.nb[1]);
    int lg = 0;
    while ((1 << lg) < pb.group) ++lg;
    prm.log2g = lg;
    prm.stages = stages;
    prm.kg = (int)(pb.K / pb.group);
    uint32_t cols = SA * 32 + nt, pw = 32;
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
    const size_t smem = smem_for(nt, bits, stages);
    if (pb.xdt == DT::BF16) {
        return pb.ydt == DT::F32 ? launch_bits<bf16_t, float>(bits, prm, grid, smem, stream)
                                 : launch_bits<bf16_t, bf16_t>(bits, prm, grid, smem, stream);
    }
    return pb.ydt == DT::F32 ? launch_bits<f16_t, float>(bits, prm, grid, smem, stream)
                             : launch_bits<f16_t, f16_t>(bits, prm, grid, smem, stream);
}

cudaError_t read_and_clear_device_error(int* value, cudaStream_t s) {
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
}

}  // namespace aq
