// warp_mma_kernel.cuh -- warp-level tensor-core kernel for decode batches (up to 32 rows of x
// per launch batch).
//
// What it computes, like the other kernels of the library (the factored form of
// x . (s*q + b)^T, "mlx PR #4516", load_vector fix):
//     y[t, n] = sum_g  s[n,g] * D[n,g,t]  +  b[n,g] * X[g,t]
//     D[n,g,t] = sum_{k in g} q[n,k] * x[t,k]   (tensor cores, exact integer codes, fp32 sums)
//     X[g,t]   = sum_{k in g} x[t,k]            (tensor cores against an all-ones tile: the
//                                                products are exact, the sums fp32)
//
// Why a warp-level MMA here.  At a few dozen tokens the contraction has too few columns to keep
// a tcgen05 tile busy: a tcgen05.mma of 32 columns costs as much time as one of 64, the
// tensor-memory kernel's time goes into moving expanded codes into tensor memory and each
// group's accumulator out of it, and its set-up (TMEM allocation, barrier rings, a pipeline of
// specialised warps) dominates the small projections of a decode step.  Here every step stays
// in the registers of one warp: the packed codes come from shared memory, are expanded in place
// into mma.sync A fragments, and each group's accumulator is folded into the running output with
// two FMAs per element.
//
// Layout of the work.  A warp owns 32 W rows (two m16 tiles) x NT = 8*NTL tokens (NTL n8 tiles)
// and a contiguous range of groups; a CTA holds wr x wk warps, wr blocks of rows times wk slices
// of K, whose partial tiles are summed in shared memory in slice order at the end.  When one row
// block per CTA would still leave most SMs idle, a thread-block cluster of cs CTAs splits the K
// of each row block; after a cluster barrier every CTA adds the CTAs' partial tiles, in rank
// order, for its share of the outputs over distributed shared memory.  No sum depends on timing.
// Within a sub-block of KS = min(G, 64) codes, lane (r = lane/4, c = lane%4) owns codes
// c*KS/4 .. c*KS/4 + KS/4 - 1 of W rows r and r+8 of each m tile, and of x row r of each n tile;
// k step s of the MMA takes codes 4s .. 4s+3 of every lane's span.  The order of k inside an MMA
// is thus a permutation of the group's codes, the same for A (codes) and B (x), which leaves
// every group sum unchanged and lets a lane load its x as plain 16-byte vectors and its codes as
// one 4-, 8- or 16-byte word run.  Each n tile's x fragments also feed one more MMA per k step
// with an all-ones A tile, whose every row is then X of the tile's tokens 2c and 2c + 1.
//
// Memory.  W streams through a per-warp ring of RD sub-blocks in shared memory, each slot filled
// by one TMA box (32 rows of one sub-block; gate/up: 16 rows of each matrix) completing on the
// slot's mbarrier; a lane reads its fragment words back after the slot's wait and the warp's
// synchronisation, and one lane refills the slot.  The scales and biases of the CTA's rows are
// staged by bulk copies.  Both those copies and the first RD boxes of every ring are issued before
// the wait on the previous kernel in the stream (weights are constant operands of the call); the
// x tile (when it fits in shared memory), one bulk copy per token row, follows the wait.  An x
// tile too large to stage is read through L2.
//
// Partial rows and tokens: loads of rows past N and of tokens past M are clamped to the last
// valid one; only the final stores check bounds, so the inner loop carries no bounds test.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>
#include <type_traits>

#include "aq_internal.h"
#include "device_common.cuh"
#include "sm100_ptx.cuh"
#include "warp_mma.cuh"

namespace aq {
namespace wm {

template <int BITS, int G>
struct Geo {
    static constexpr int KS = G < 64 ? G : 64;         // codes per sub-block
    static constexpr int SPG = G / KS;                 // sub-blocks per group
    static constexpr int STEPS = KS / 16;              // MMA k steps per sub-block
    static constexpr int KSB = KS * BITS / 8;          // bytes of one W row per sub-block
    static constexpr int LB = KSB / 4;                 // bytes of one W row per lane
    static constexpr int WS = LB / 4;                  // words of one W row per lane
    static constexpr int XV = KS / 32;                 // 16-byte x vectors per lane per n tile
    static_assert(WS >= 1 && KSB % 16 == 0 && 2 * ROWS * KSB <= RING_BYTES, "sub-block geometry");
};

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// d += A (16 x 16, row) . B (16 x 8, col), fp32 accumulation
template <bool BF>
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    if constexpr (BF)
        asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    else
        asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// f16 pairs (1024 + q0, 1024 + q1) -> (q0, q1), exact
__device__ __forceinline__ uint32_t f16_minus_1024(uint32_t v) {
    const uint32_t off = 0x64006400u;
    const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&v), *reinterpret_cast<const __half2*>(&off));
    return *reinterpret_cast<const uint32_t*>(&r);
}

// The codes 4s .. 4s+3 of one W row of a lane's span, for every k step s, as two 16-bit pairs:
// a[s][0] = (code 4s, code 4s+1), a[s][1] = (code 4s+2, code 4s+3).
//   bf16, 2/4 bits: 128 + q (a code OR-ed into the mantissa of 128.0; the fold removes the 128)
//   bf16, 8 bits:   q, formed exactly in fp32 (2^23 + q minus 2^23) and converted (q <= 255)
//   f16, any:       q, from 1024 + q (OR-ed into the mantissa of 1024.0) minus 1024
template <int BITS, bool BF, int STEPS>
__device__ __forceinline__ void expand_row(const uint32_t* wv, uint32_t (*a)[2]) {
    constexpr uint32_t MAGIC = BF ? 0x43004300u : 0x64006400u;
    auto fin = [](uint32_t v) -> uint32_t {
        if constexpr (BF) return v;
        else return f16_minus_1024(v);
    };
    if constexpr (BITS == 4) {
        // byte b of a word holds codes (2b, 2b+1); the word shifted right by 4 holds code 2b+1 in
        // the low nibble of byte b.  PRMT puts byte b of each into the low byte of a half.
#pragma unroll
        for (int s = 0; s < STEPS; ++s) {
            const uint32_t w = wv[s >> 1], sh = w >> 4;
            const int b = 2 * (s & 1);
            a[s][0] = fin((__byte_perm(w, sh, b | ((4 + b) << 8)) & 0x000F000Fu) | MAGIC);
            a[s][1] = fin((__byte_perm(w, sh, (b + 1) | ((5 + b) << 8)) & 0x000F000Fu) | MAGIC);
        }
    } else if constexpr (BITS == 2) {
        // byte b holds codes 4b .. 4b+3 in bit pairs 0-1, 2-3, 4-5, 6-7
#pragma unroll
        for (int s = 0; s < STEPS; ++s) {
            const uint32_t w = wv[s >> 2];
            const int b = s & 3;
            a[s][0] = fin((__byte_perm(w, w >> 2, b | ((4 + b) << 8)) & 0x00030003u) | MAGIC);
            a[s][1] = fin((__byte_perm(w >> 4, w >> 6, b | ((4 + b) << 8)) & 0x00030003u) | MAGIC);
        }
    } else {
        static_assert(BITS == 8, "bits");
#pragma unroll
        for (int s = 0; s < STEPS; ++s) {
            const uint32_t w = wv[s];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                if constexpr (BF) {
                    const float m0 = __uint_as_float(__byte_perm(w, 0x4B000000u, (2 * j) | (4 << 4) | (5 << 8) | (7 << 12)));
                    const float m1 = __uint_as_float(__byte_perm(w, 0x4B000000u, (2 * j + 1) | (4 << 4) | (5 << 8) | (7 << 12)));
                    const float2 qf = ptx::fadd2(make_float2(m0, m1), make_float2(-8388608.0f, -8388608.0f));
                    const __nv_bfloat162 q = __floats2bfloat162_rn(qf.x, qf.y);
                    a[s][j] = *reinterpret_cast<const uint32_t*>(&q);
                } else {
                    a[s][j] = f16_minus_1024(__byte_perm(w, MAGIC, (2 * j) | (5 << 4) | ((2 * j + 1) << 8) | (7 << 12)));
                }
            }
        }
    }
}

template <int LB>
__device__ __forceinline__ void load_lane_words(const uint8_t* p, uint32_t* w) {
    if constexpr (LB == 16) {
        const uint4 v = *reinterpret_cast<const uint4*>(p);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (LB == 8) {
        const uint2 v = *reinterpret_cast<const uint2*>(p);
        w[0] = v.x; w[1] = v.y;
    } else {
        w[0] = *reinterpret_cast<const uint32_t*>(p);
    }
}

// Activations (x, a residual) may have been written by the previous kernel in the stream, which
// a programmatic dependent starts next to: an L1 line of such a buffer, cached on this SM by an
// earlier kernel, could still hold the old values.  Every global read of them goes to L2 (.cg),
// which is coherent; only weights are read through L1.
// element `off` of a tensor of y's dtype (fp32, or the activation dtype XT), as fp32
template <typename XT>
__device__ __forceinline__ float load_out(const void* r, int64_t off, int ydt) {
    if (ydt == (int)DT::F32) return __ldcg(reinterpret_cast<const float*>(r) + off);
    return half_bits_to_float(__ldcg(reinterpret_cast<const unsigned short*>(r) + off), XT{});
}

template <typename XT>
__device__ __forceinline__ void store_pair(void* y, int64_t off, float v0, float v1, bool both, bool vec, int ydt) {
    if (ydt == (int)DT::F32) {
        float* p = reinterpret_cast<float*>(y) + off;
        if (both && vec) *reinterpret_cast<float2*>(p) = make_float2(v0, v1);
        else { p[0] = v0; if (both) p[1] = v1; }
    } else if constexpr (std::is_same<XT, bf16_t>::value) {
        __nv_bfloat16* p = reinterpret_cast<__nv_bfloat16*>(y) + off;
        if (both && vec) *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v0, v1);
        else { p[0] = __float2bfloat16_rn(v0); if (both) p[1] = __float2bfloat16_rn(v1); }
    } else {
        __half* p = reinterpret_cast<__half*>(y) + off;
        if (both && vec) *reinterpret_cast<__half2*>(p) = __floats2half2_rn(v0, v1);
        else { p[0] = __float2half_rn(v0); if (both) p[1] = __float2half_rn(v1); }
    }
}

// Where logical row r of a launch lives: segment, row of that segment's W (clamped to its last
// row for loads) and whether it exists.  Plain and fused-projection layouts: row block r / ROWS
// belongs to the segment whose blocks contain it.  Gate/up layout: block b holds rows
// 16 b .. 16 b + 15 of the gate matrix (logical rows 0..15 of the block) and the same rows of the
// up matrix (logical rows 16..31), so both halves of every output sit in one warp's m tiles.
struct RowRef {
    int seg;
    int64_t n;
    bool valid;
};
__device__ __forceinline__ RowRef row_ref(const WParams& p, int64_t r) {
    RowRef o;
    const int64_t blk = r / ROWS;
    const int j = (int)(r - blk * ROWS);
    if (p.glu) {
        o.seg = j >= ROWS / 2 ? 1 : 0;
        o.n = blk * (ROWS / 2) + (j & (ROWS / 2 - 1));
    } else {
        int s = 0;
        while (s + 1 < p.nseg && blk >= p.seg[s + 1].rb0) ++s;
        o.seg = s;
        o.n = (blk - p.seg[s].rb0) * ROWS + j;
    }
    const int64_t N = p.seg[o.seg].N;
    o.valid = o.n < N;
    if (!o.valid) o.n = N - 1;
    return o;
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + __expf(-g)); }

template <int BITS, typename XT, int G, int NTL>
__global__ void __launch_bounds__(MAX_WARPS * 32, 2) qmm_warp_kernel(const __grid_constant__ WParams p) {
    using Gm = Geo<BITS, G>;
    constexpr bool BF = std::is_same<XT, bf16_t>::value;
    constexpr int NT = 8 * NTL;
    constexpr int KS = Gm::KS, SPG = Gm::SPG, STEPS = Gm::STEPS, KSB = Gm::KSB, LB = Gm::LB, WS = Gm::WS;
    constexpr int XV = Gm::XV;
    const int RD = p.rd;   // ring slots of this warp
    constexpr float OFF = (BF && BITS < 8) ? 128.0f : 0.0f;   // code offset of the expanded A values

    extern __shared__ __align__(128) uint8_t smem_raw[];
    // TMA writes the ring slots: 128-byte aligned (every slot and half slot is a multiple of 128 bytes)
    // aligned by an offset from the shared array itself, so that every pointer derived from it stays
    // in the shared address space (shared loads and stores, not generic ones)
    uint8_t* smem = smem_raw + ((128u - (ptx::smem_u32(smem_raw) & 127u)) & 127u);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const int rw = warp % p.wr, kw = warp / p.wr;
    const int r = lane >> 2, c = lane & 3;
    const int kg = p.kg;
    const int rows_cta = p.wr * ROWS;
    const int cs = p.cs;
    const int rank = cs > 1 ? (int)ptx::cluster_ctarank() : 0;   // K slice of this CTA in its cluster
    // [rings][scales, biases: rows_cta x kg each][partial tile: NT x rows_cta fp32, clusters only]
    // [sums of squares of x, RMS-normalised inputs only: MAX_WARPS + 1 rows of NT fp32, one per
    // K-slice warp, then the CTA's total][x tile: NT x x_pitch][mbarriers: staging, rings][abort flag]
    uint8_t* ring = smem + (size_t)warp * p.ring_bytes;
    uint16_t* s_s = reinterpret_cast<uint16_t*>(smem + (size_t)nwarps * p.ring_bytes);
    uint16_t* s_b = s_s + rows_cta * kg;
    float* cpart = reinterpret_cast<float*>(s_b + rows_cta * kg);
    float* xsq = cpart + (cs > 1 ? NT * rows_cta : 0);
    uint8_t* xt = reinterpret_cast<uint8_t*>(xsq + (p.rms ? (MAX_WARPS + 1) * NT : 0));
    uint64_t* sbar = reinterpret_cast<uint64_t*>(xt + (p.xsm ? NT * p.x_pitch : 0));
    uint64_t* wfull = sbar + 2 + warp * MAX_RD;   // this warp's ring slots
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sbar + 2 + MAX_WARPS * MAX_RD);
    const int xp = p.x_pitch;

    const int64_t bz = blockIdx.z;
    const int64_t bo = bz / p.nb1, bi = bz - bo * p.nb1;
    const uint16_t* x = p.x + bo * p.xb[0] + bi * p.xb[1];
    const int64_t tok0 = (int64_t)blockIdx.y * NT;
    const int64_t rowc = (int64_t)(blockIdx.x / cs) * rows_cta; // first logical row of the CTA
    const int64_t roww = rowc + rw * ROWS;                       // first logical row of this warp
    const int cg0 = rank * p.kgc, cg1 = min(cg0 + p.kgc, kg);   // groups of this CTA
    const int ckg = cg1 > cg0 ? cg1 - cg0 : 0;
    const int g0 = cg0 + kw * p.gpw;                             // groups of this warp
    const int g1 = min(g0 + p.gpw, cg1);
    const bool warp_rows = roww / ROWS < p.nrb;
    const int nsub = (warp_rows && g1 > g0) ? (g1 - g0) * SPG : 0;

    const int sb_parts = p.glu ? 2 : 1;   // scale/bias copies per row block: one per matrix part
    if (threadIdx.x == 0) {
        ptx::mbar_init(&sbar[0], 1);
        ptx::mbar_init(&sbar[1], p.wr * sb_parts);
        *abort_flag = 0;
        // the x tile's barrier is armed with its bytes here, before the block-wide barrier below, so
        // that every x copy (issued by several warps after the dependent-launch wait) completes on a
        // barrier that already expects it
        if (p.xsm) ptx::mbar_arrive_expect_tx(&sbar[0], (uint32_t)(NT * ckg * G * 2));
    }
    if (lane == 0)
        for (int s = 0; s < RD; ++s) ptx::mbar_init(&wfull[s], 1);
    ptx::fence_mbar_init();

    // The W box of this warp's rows for ring step j: one box of 32 rows, or (gate/up) two of 16 rows,
    // one from each matrix.  TMA reads rows past a matrix's end as zeros.
    const RowRef wr0 = row_ref(p, min(roww, p.nrb * ROWS - 1));
    const RowRef wr1 = row_ref(p, min(roww + ROWS / 2, p.nrb * ROWS - 1));
    auto load_w = [&](int j, int slot) {
        uint8_t* dst = ring + slot * ROWS * KSB;
        const int32_t wc = (g0 * SPG + j) * (KSB / 4);   // word coordinate: a multiple of 16 bytes
        ptx::mbar_arrive_expect_tx(&wfull[slot], (uint32_t)(ROWS * KSB));
        if (p.glu) {
            ptx::tma_load_2d(dst, &p.tw[0], &wfull[slot], wc, (int32_t)wr0.n);
            ptx::tma_load_2d(dst + (ROWS / 2) * KSB, &p.tw[1], &wfull[slot], wc, (int32_t)wr1.n);
        } else {
            ptx::tma_load_2d(dst, &p.tw[wr0.seg], &wfull[slot], wc, (int32_t)wr0.n);
        }
    };

    ptx::pdl_launch_dependents();
    __syncthreads();   // barrier initialisation visible to every thread and to the copy engine

    // ---- weights first.  W, its scales and its biases are constant operands of the call (the
    // kernel before this one in the stream does not write them), so they are staged before the wait
    // for that kernel and their copies overlap its tail: the scale/bias blocks of the CTA's rows
    // (one bulk copy each per block and matrix part) on sbar[1], where every copying thread arrives
    // with its own bytes, and the first RD W boxes of every warp on its ring.  Bulk copies are issued
    // one at a time within a warp, so they are spread over the warps. ----
    if (p.sb16) {
        const int q = warp + nwarps * lane;   // part q: block q / parts, half q % parts
        if (q < p.wr * sb_parts) {
            const int b = q / sb_parts, hp = q - b * sb_parts;
            const int64_t r0 = rowc + b * ROWS;
            int64_t nrow = 0, n0 = 0;
            int sgi = 0;
            if (r0 / ROWS < p.nrb) {
                const RowRef rr = row_ref(p, r0 + hp * (ROWS / 2));
                sgi = rr.seg;
                n0 = rr.n;
                nrow = min((int64_t)(p.glu ? ROWS / 2 : ROWS), p.seg[sgi].N - n0);
                if (nrow < 0) nrow = 0;
            }
            ptx::mbar_arrive_expect_tx(&sbar[1], 2u * (uint32_t)(nrow * kg * 2));
            if (nrow > 0) {
                const WSeg& sg = p.seg[sgi];
                const int so = (b * ROWS + hp * (ROWS / 2)) * kg;
                ptx::bulk_load(s_s + so, sg.scales + n0 * kg, (uint32_t)(nrow * kg * 2), &sbar[1]);
                ptx::bulk_load(s_b + so, sg.biases + n0 * kg, (uint32_t)(nrow * kg * 2), &sbar[1]);
            }
        }
    }
    if (!p.sb16) {   // 4-byte copies, rows past a matrix's end clamped to its last row
        const uint32_t ss = ptx::smem_u32(s_s), sb = ptx::smem_u32(s_b);
        const int cpr = kg / 2;
        const int total = rows_cta * cpr;
        for (int i = threadIdx.x; i < total; i += blockDim.x) {
            const int rl = i / cpr, col = i - rl * cpr;
            const RowRef rr = row_ref(p, min(rowc + rl, p.nrb * ROWS - 1));
            const WSeg& sg = p.seg[rr.seg];
            const int64_t go = rr.n * kg + col * 2;
            const uint32_t so = (uint32_t)((rl * kg + col * 2) * 2);
            cp_async4(ss + so, sg.scales + go);
            cp_async4(sb + so, sg.biases + go);
        }
        cp_async_commit();
    }
    if (lane == 0)
        for (int j = 0; j < RD && j < nsub; ++j) load_w(j, j);

    // x may be the output of the previous kernel in the stream: read nothing before it completed
    ptx::pdl_wait();

    // ---- the CTA's x tile, one bulk copy per token row (spread over the warps) on sbar[0], armed
    // with the tile's bytes in the prologue ----
    if (p.xsm) {
        const int tr = warp + nwarps * lane;   // codes [cg0 G, cg1 G) of token row tr
        if (tr < NT) {
            const int64_t tok = min(tok0 + tr, p.M - 1);
            ptx::bulk_load(xt + tr * xp, x + tok * p.x_row + (int64_t)cg0 * G, (uint32_t)(ckg * G * 2), &sbar[0]);
        }
    }
    int issued = min(RD, nsub);   // W boxes issued on this warp's ring (warp-uniform count)
    int waited = 0;               // ... and waited for

    {
        int at = 0;
        if (p.xsm && !ptx::mbar_wait(&sbar[0], 0, abort_flag, WAIT_NS)) at = DEVERR_AT_WARP_X;
        else if (p.sb16 && !ptx::mbar_wait(&sbar[1], 0, abort_flag, WAIT_NS)) at = DEVERR_AT_WARP_SB;
        if (at) {
            atomicOr(p.err, DEVERR_TIMEOUT | (*abort_flag ? 0 : at));
            *abort_flag = 1;
        }
    }
    if (!p.sb16) cp_async_wait<0>();
    __syncthreads();
    bool ok = *abort_flag == 0;   // CTA-uniform after the barrier
    if (!ok && threadIdx.x == 0) {
        // a staging copy may still be in flight: let it land before its buffers are reused
        volatile int never = 0;
        if (p.xsm) ptx::mbar_wait(&sbar[0], 0, &never, 200000000ull);
        if (p.sb16) ptx::mbar_wait(&sbar[1], 0, &never, 200000000ull);
    }

    // ---- this lane's rows of the scale/bias tiles and x rows ----
    int sb_row[4];   // (row - rowc) * kg for rows roww + 16 m + 8 h + r, index 2 m + h
#pragma unroll
    for (int mh = 0; mh < 4; ++mh) sb_row[mh] = (rw * ROWS + 16 * (mh >> 1) + 8 * (mh & 1) + r) * kg;
    const uint8_t* xrow[NTL];   // this lane's span of x row 8 t + r (shared memory or global)
#pragma unroll
    for (int t = 0; t < NTL; ++t) {
        if (p.xsm) {
            xrow[t] = xt + (8 * t + r) * xp + c * (KS / 2);
        } else {
            const int64_t tok = min(tok0 + 8 * t + r, p.M - 1);
            xrow[t] = reinterpret_cast<const uint8_t*>(x + tok * p.x_row + c * (KS / 4));
        }
    }
    const uint8_t* rd_lane = ring + r * KSB + c * LB;

    float acc[2][NTL][4];
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int t = 0; t < NTL; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[m][t][e] = 0.0f;
    float d[2][NTL][4];
    // X of the group for this lane's tokens, from an all-ones A tile on the tensor cores: every
    // row of the product holds the column sums of the x tile, so a lane's accumulator elements
    // 0 and 1 are X for tokens 2c and 2c + 1 of n tile t (the products are exact, the sums fp32)
    float xsum[NTL][4];
    const uint32_t ONES = BF ? 0x3F803F80u : 0x3C003C00u;   // (1, 1) in the activation dtype
    // RMS-normalised inputs: the Gram matrix of the n tile's x rows on the tensor cores, A being the
    // same x fragments as B (rows 8..15 of A repeat rows 0..7), so that its diagonal element
    // (token 8 t + n, n) holds the sum of squares of token 8 t + n over the warp's K slice: lane
    // (r = n, c = n / 2), element n % 2 (the products are exact, the sums fp32)
    float sq[NTL][4];
#pragma unroll
    for (int t = 0; t < NTL; ++t) sq[t][0] = sq[t][1] = sq[t][2] = sq[t][3] = 0.0f;
    int slot = 0;          // ring slot of sub-block j, and the parity of its fill
    uint32_t par = 0;

#pragma unroll 1
    for (int j = 0; j < nsub; ++j) {
        const int g = g0 + j / SPG, sub = j % SPG;
        if (sub == 0) {
#pragma unroll
            for (int t = 0; t < NTL; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    d[0][t][e] = d[1][t][e] = 0.0f;
                    xsum[t][e] = 0.0f;
                }
        }
        // codes of this sub-block from the ring (a bounded wait; after an expiry the warp computes
        // on whatever the slot holds and the error word says the results are void)
        if (ok) {
            ok = __all_sync(0xffffffffu, ptx::mbar_wait(&wfull[slot], par, abort_flag, WAIT_NS));
            if (ok) {
                waited = j + 1;
            } else if (lane == 0) {
                atomicOr(p.err, DEVERR_TIMEOUT | (*abort_flag ? 0 : DEVERR_AT_WARP_W));
                *abort_flag = 1;
            }
        }
        uint32_t wv[4][WS];
        {
            const uint8_t* sp = rd_lane + slot * ROWS * KSB;
#pragma unroll
            for (int mh = 0; mh < 4; ++mh) load_lane_words<LB>(sp + (16 * (mh >> 1) + 8 * (mh & 1)) * KSB, wv[mh]);
        }
        __syncwarp();   // every lane has read the slot before it is refilled
        if (ok && j + RD < nsub) {
            if (lane == 0) load_w(j + RD, slot);
            issued = j + RD + 1;
        }
        if (++slot == RD) {
            slot = 0;
            par ^= 1u;
        }

        uint32_t a[4][STEPS][2];
#pragma unroll
        for (int mh = 0; mh < 4; ++mh) expand_row<BITS, BF, STEPS>(wv[mh], a[mh]);

        const int kx2 = ((g - (p.xsm ? cg0 : 0)) * G + sub * KS) * 2;   // sub-block's byte offset in an x row
#pragma unroll
        for (int t = 0; t < NTL; ++t) {
            uint4 xv[XV];
#pragma unroll
            for (int v = 0; v < XV; ++v) {
                const uint4* xp4 = reinterpret_cast<const uint4*>(xrow[t] + kx2) + v;
                xv[v] = p.xsm ? *xp4 : __ldcg(xp4);
            }
            const uint32_t* xw = reinterpret_cast<const uint32_t*>(xv);
#pragma unroll
            for (int s = 0; s < STEPS; ++s) {
#pragma unroll
                for (int m = 0; m < 2; ++m)
                    mma16816<BF>(d[m][t], a[2 * m][s][0], a[2 * m + 1][s][0], a[2 * m][s][1], a[2 * m + 1][s][1],
                                 xw[2 * s], xw[2 * s + 1]);
                mma16816<BF>(xsum[t], ONES, ONES, ONES, ONES, xw[2 * s], xw[2 * s + 1]);
                if (p.rms) mma16816<BF>(sq[t], xw[2 * s], xw[2 * s], xw[2 * s + 1], xw[2 * s + 1], xw[2 * s], xw[2 * s + 1]);
            }
        }

        if (sub == SPG - 1) {   // fold the group: acc += s * D + (b - OFF * s) * X
            float sv[4], bv[4];
#pragma unroll
            for (int mh = 0; mh < 4; ++mh) {
                sv[mh] = half_bits_to_float(s_s[sb_row[mh] + g], XT{});
                bv[mh] = half_bits_to_float(s_b[sb_row[mh] + g], XT{});
                if (OFF != 0.0f) bv[mh] = fmaf(-OFF, sv[mh], bv[mh]);
            }
            // on fp32 pairs (the two tokens of a lane's accumulator row): the same two roundings per
            // element as one fmaf for b X and one for s D
#pragma unroll
            for (int t = 0; t < NTL; ++t) {
                const float2 X = make_float2(xsum[t][0], xsum[t][1]);
#pragma unroll
                for (int m = 0; m < 2; ++m)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float s = sv[2 * m + h], b = bv[2 * m + h];
                        float2 v = make_float2(acc[m][t][2 * h], acc[m][t][2 * h + 1]);
                        v = ptx::ffma2(make_float2(b, b), X, v);
                        v = ptx::ffma2(make_float2(s, s), make_float2(d[m][t][2 * h], d[m][t][2 * h + 1]), v);
                        acc[m][t][2 * h] = v.x;
                        acc[m][t][2 * h + 1] = v.y;
                    }
            }
        }
    }

    // ---- outputs: sum the warps' K slices in slice order; without a cluster, store; with one,
    // keep the CTA's partial tile for the cluster-wide sum.  An output item is a pair of adjacent
    // rows of one segment's y, or (gate/up layout) a pair of adjacent silu(gate) * up values, whose
    // gate and up sums sit 16 logical rows apart in the same row block. ----
    const int lipb = p.glu ? 3 : 4;                // log2 of the items per row block (8 or 16)
    const int lipt = lipb + (31 - __clz(p.wr));    // log2 of the items per token (wr: a power of two)
    const int ipb = 1 << lipb, ipt = 1 << lipt;
    const int total = NT * ipt;
    const int64_t ybase = bo * p.yb[0] + bi * p.yb[1];
    // local logical row of item element e (0, 1) and half (0: the value, or gate; 1: up)
    auto lrow = [&](int wrr, int it, int e, int half) {
        return wrr * ROWS + (p.glu ? 2 * it + e + half * (ROWS / 2) : 2 * it + e);
    };
    // the items this CTA emits: all of them, or with a cluster its rank's share
    const int per = cs > 1 ? (total + cs - 1) / cs : total;
    const int i_lo = cs > 1 ? rank * per : 0, i_hi = min(i_lo + per, total);
    // residual (plain calls only) of this thread's first item, read now: its L2 latency overlaps
    // the partial-tile barrier and sums (and with a cluster, the cluster barrier)
    float r_first[2] = {0.0f, 0.0f};
    if (p.seg[0].r != nullptr && i_lo + (int)threadIdx.x < i_hi) {
        const int i = i_lo + threadIdx.x;
        const int tt = i >> lipt, rp = i & (ipt - 1);
        const RowRef rr = row_ref(p, rowc + lrow(rp >> lipb, rp & (ipb - 1), 0, 0));
        const int64_t tok = tok0 + tt;
        if (tok < p.M && rr.valid) {
            const int64_t ro = ybase + tok * p.seg[0].r_row + rr.n;
            r_first[0] = load_out<XT>(p.seg[0].r, ro, p.ydt);
            if (rr.n + 1 < p.seg[0].N) r_first[1] = load_out<XT>(p.seg[0].r, ro + 1, p.ydt);
        }
    }

    // ---- partial tile of this warp into its own ring.  Every W box issued has been waited for,
    // unless a wait expired: then the warp first waits (bounded, ignoring the abort flag) for the
    // boxes still in flight, so that no copy lands in the ring after it is reused or freed ----
    if (waited < issued && lane == 0) {
        volatile int never = 0;
        for (int j = waited; j < issued; ++j) ptx::mbar_wait(&wfull[j % RD], (uint32_t)((j / RD) & 1), &never, 200000000ull);
    }
    __syncwarp();
    if (p.rms && rw == 0 && c == (r >> 1)) {   // the warp's sum of squares per token (its K slice)
#pragma unroll
        for (int t = 0; t < NTL; ++t) xsq[kw * NT + 8 * t + r] = (r & 1) ? sq[t][1] : sq[t][0];
    }
    {
        float* red = reinterpret_cast<float*>(ring);
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int t = 0; t < NTL; ++t)
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int e = 0; e < 2; ++e)
                        red[(8 * t + 2 * c + e) * RED_PITCH + 16 * m + 8 * h + r] = acc[m][t][2 * h + e];
    }
    __syncthreads();

    // RMS-normalised inputs: 1 / sqrt(mean_k x[t,k]^2 + eps) for token tt: the K-slice warps' sums
    // of squares added in slice order, then (clusters) the CTAs' totals in rank order (every CTA's
    // total is written before the first cluster barrier, which precedes every call with cs > 1)
    auto rms_scale = [&](int tt) -> float {
        float s2 = 0.0f;
        if (cs == 1) {
            for (int k = 0; k < p.wk; ++k) s2 += xsq[k * NT + tt];
        } else {
            const uint32_t a = ptx::smem_u32(xsq + MAX_WARPS * NT + tt);
            for (int q = 0; q < cs; ++q) s2 += ptx::ld_cluster_f32(ptx::mapa(a, (uint32_t)q));
        }
        return rsqrtf(s2 / (float)p.K + p.rms_eps);
    };
    auto emit = [&](int i, int tt, int wrr, int it, const float (&v)[2][2]) {
        const int64_t tok = tok0 + tt;
        const RowRef rr = row_ref(p, rowc + lrow(wrr, it, 0, 0));
        if (tok >= p.M || !rr.valid) return;
        const WSeg& sg = p.seg[p.glu ? 0 : rr.seg];
        const bool both = rr.n + 1 < sg.N;
        const float sc = p.rms ? rms_scale(tt) : 1.0f;
        float o0 = v[0][0] * sc, o1 = v[1][0] * sc;
        if (p.glu) {
            o0 = silu(o0) * (v[0][1] * sc);
            o1 = silu(o1) * (v[1][1] * sc);
        }
        if (sg.r) {   // residual: added in fp32 before the one rounding to y's dtype
            if (i == i_lo + (int)threadIdx.x) {
                o0 += r_first[0];
                o1 += r_first[1];
            } else {
                const int64_t ro = ybase + tok * sg.r_row + rr.n;
                o0 += load_out<XT>(sg.r, ro, p.ydt);
                if (both) o1 += load_out<XT>(sg.r, ro + 1, p.ydt);
            }
        }
        store_pair<XT>(sg.y, ybase + tok * sg.y_row + rr.n, o0, o1, both, p.yvec != 0, p.ydt);
    };
    for (int i = threadIdx.x; i < total; i += blockDim.x) {
        const int tt = i >> lipt, rp = i & (ipt - 1);
        const int wrr = rp >> lipb, it = rp & (ipb - 1);
        float v[2][2] = {{0.0f, 0.0f}, {0.0f, 0.0f}};
        for (int hf = 0; hf < (p.glu ? 2 : 1); ++hf) {
            const int rl = lrow(wrr, it, 0, hf) - wrr * ROWS;   // even: the pair is one float2
            for (int k = 0; k < p.wk; ++k) {
                const float* part = reinterpret_cast<const float*>(smem + (size_t)(k * p.wr + wrr) * p.ring_bytes);
                const float2 u = *reinterpret_cast<const float2*>(part + tt * RED_PITCH + rl);
                v[0][hf] += u.x;
                v[1][hf] += u.y;
            }
            if (cs > 1)
                *reinterpret_cast<float2*>(cpart + tt * rows_cta + wrr * ROWS + rl) = make_float2(v[0][hf], v[1][hf]);
        }
        if (cs == 1) emit(i, tt, wrr, it, v);
    }
    if (cs > 1) {
        if (p.rms && threadIdx.x < NT) {   // the CTA's sum of squares per token, slices in order
            float s2 = 0.0f;
            for (int k = 0; k < p.wk; ++k) s2 += xsq[k * NT + threadIdx.x];
            xsq[MAX_WARPS * NT + threadIdx.x] = s2;
        }
        // every CTA's partial tile is complete and visible cluster-wide (hardware barrier)
        asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
        // this CTA's share of the tile: the CTAs' partials added in rank order over distributed
        // shared memory
        const uint32_t cp_s = ptx::smem_u32(cpart);
        for (int i = i_lo + threadIdx.x; i < i_hi; i += blockDim.x) {
            const int tt = i >> lipt, rp = i & (ipt - 1);
            const int wrr = rp >> lipb, it = rp & (ipb - 1);
            float v[2][2] = {{0.0f, 0.0f}, {0.0f, 0.0f}};
            for (int hf = 0; hf < (p.glu ? 2 : 1); ++hf) {
                const uint32_t off = (uint32_t)((tt * rows_cta + lrow(wrr, it, 0, hf)) * 4);
                for (int q = 0; q < cs; ++q) {
                    const float2 u = ptx::ld_cluster_f2(ptx::mapa(cp_s + off, (uint32_t)q));
                    v[0][hf] += u.x;
                    v[1][hf] += u.y;
                }
            }
            emit(i, tt, wrr, it, v);
        }
        // no CTA leaves while another may still read its partial tile
        asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    }
}

template <int BITS, typename XT, int G, int NTL>
cudaError_t launch_t(const WParams& p, dim3 grid, int warps, size_t smem, cudaStream_t s) {
    static std::mutex mu;
    static bool done[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!done[dev]) {
            e = cudaFuncSetAttribute(qmm_warp_kernel<BITS, XT, G, NTL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)SMEM_LIMIT);
            if (e != cudaSuccess) return e;
            done[dev] = true;
        }
    }
    // a programmatic dependent of the previous kernel in the stream: it may be scheduled early,
    // but reads nothing before that kernel completed (griddepcontrol.wait at its start)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(32 * warps);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;   // CTAs splitting K of one row block
    attr[1].val.clusterDim.x = (unsigned)p.cs;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.cs > 1 ? 2 : 1;   // a plain launch without a split (measured a little faster)
    return cudaLaunchKernelEx(&cfg, qmm_warp_kernel<BITS, XT, G, NTL>, p);
}

template <int BITS, typename XT, int G>
cudaError_t launch_n(int ntl, const WParams& p, dim3 grid, int warps, size_t smem, cudaStream_t s) {
    switch (ntl) {
        case 1: return launch_t<BITS, XT, G, 1>(p, grid, warps, smem, s);
        case 2: return launch_t<BITS, XT, G, 2>(p, grid, warps, smem, s);
    }
    return cudaErrorInvalidValue;
}

template <int BITS, typename XT>
cudaError_t launch_g(int group, int ntl, const WParams& p, dim3 grid, int warps, size_t smem, cudaStream_t s) {
    switch (group) {
        case 32:
            if constexpr (BITS * 32 >= 128) return launch_n<BITS, XT, 32>(ntl, p, grid, warps, smem, s);
            else return cudaErrorInvalidValue;
        case 64: return launch_n<BITS, XT, 64>(ntl, p, grid, warps, smem, s);
        case 128: return launch_n<BITS, XT, 128>(ntl, p, grid, warps, smem, s);
    }
    return cudaErrorInvalidValue;
}

template <int BITS>
cudaError_t launch(bool bf16, int group, int ntl, const WParams& p, dim3 grid, int warps, size_t smem,
                   cudaStream_t stream) {
    return bf16 ? launch_g<BITS, bf16_t>(group, ntl, p, grid, warps, smem, stream)
                : launch_g<BITS, f16_t>(group, ntl, p, grid, warps, smem, stream);
}

}  // namespace wm
}  // namespace aq
