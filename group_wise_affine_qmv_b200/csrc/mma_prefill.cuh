// mma_prefill.cuh -- tensor-core kernel for many rows of x (prefill, M >= 64): the same exact
// factored arithmetic as mma_kernel.cuh,
//     y[n, t] = sum_g  s[n,g] * D_g[n, t]  +  b[n,g] * X_g[t],   D_g = sum_{k in g} q * x,
// on tiles of 128 W rows x 128 tokens, so that each tcgen05.mma (M = 128, N = 128, K = 16)
// carries four times the work of the decode kernel's and the tensor pipe, not instruction
// issue, sets the pace.  One W stage is one group (G = 64 or 128 codes), so a single fp32
// accumulator of 128 columns per stage is enough and two of them fit tensor memory next to
// the double-buffered A blocks.
//
// Roles (480 threads):
//   warp 0       W producer: TMA of each stage's 128 x G codes onto a ring.
//   warp 14      x producer: TMA of each stage's x block (G/64 boxes of [128 tokens x 64],
//                128-byte swizzle, the UMMA B operand) onto a ring; fold warps free a slot.
//   warp 1       MMA issuer: G/16 tcgen05.mma kind::f16 per stage into accumulator i % 2, one
//                tcgen05.commit (sdone[i % 2]).
//   warps 2..5   code expanders: thread <-> W row, all G codes of the stage (128 + q in bf16 for
//                codes below 128, exact integers otherwise), into A block i % 2.
//   warps 6..13  folds: thread <-> W row, warps q and q + 4 take 64 tokens each.  Per stage,
//                X_g of the 128 tokens is summed from the x block in shared memory (fp32, k
//                order) by all fold threads, then y += s*D' + (b - OFF*s)*X_g; the x slot and
//                the accumulator are released.  Per tile, the store of y: staged in shared
//                memory and stored with one bulk tensor copy (N a multiple of 8, 16-byte aligned
//                rows of y), else element stores.
// Tiles are walked W-tile-fastest, so the CTAs in flight share one token tile (x from L2) and
// the whole packed W stays in L2 across token tiles.
#pragma once

#include "mma_kernel.cuh"

namespace aq {
namespace mma {
namespace pf {

struct PSmem {
    uint64_t* wfull;     // [P_MAX_STAGES]
    uint64_t* wfree;     // [P_MAX_STAGES] (expander warps)
    uint64_t* xfull;     // [P_MAX_XST]
    uint64_t* xfree;     // [P_MAX_XST] (fold warps)
    uint64_t* afull;     // [2] (expander warps)
    uint64_t* sdone;     // [2] (commit)
    uint64_t* dfree;     // [2] (fold warps)
    uint64_t* sbar;      // [2] scale/bias chunk slots (fold threads)
    uint64_t* xgbar;     // [2 token halves][2] sums of x of a stage written (the half's fold threads)
    uint64_t* mdone;
    uint64_t* ybar;      // ytma: the staged y tile is written (fold threads)
    uint32_t* tmem_base;
    int* abort;
    float* xg;           // [2][NTP] sums of x of a stage
    uint16_t* ystg;      // ytma: [NTP tokens][128 rows] of y, the source of the tile's TMA store
    uint8_t* xs;         // [xst][SUB][NTP][128 B]
    uint8_t* ws;         // [stages][128][ROWB]
    uint16_t* sb;        // [2 slots][2 arrays][128][SCP]
};

template <int SUB, int ROWB>
__device__ __forceinline__ PSmem p_carve(uint8_t* base, const Params& p) {
    PSmem s;
    uint8_t* q = base;
    s.xs = q;
    q += (size_t)p.xst * SUB * NTP * 128;
    s.ws = q;
    q += (size_t)p.stages * 128 * ROWB;
    q += (1024u - (uint32_t)((q - base) & 1023)) & 1023u;   // base is 1024-byte aligned
    s.sb = reinterpret_cast<uint16_t*>(q);
    q += 2 * 2 * 128 * SCP * 2;
    s.xg = reinterpret_cast<float*>(q);
    q += 2 * NTP * 4;
    s.ystg = reinterpret_cast<uint16_t*>(q);
    if (p.ytma) q += P_YSTG_BYTES;
    s.wfull = reinterpret_cast<uint64_t*>(q);
    s.wfree = s.wfull + P_MAX_STAGES;
    s.xfull = s.wfree + P_MAX_STAGES;
    s.xfree = s.xfull + P_MAX_XST;
    s.afull = s.xfree + P_MAX_XST;
    s.sdone = s.afull + 2;
    s.dfree = s.sdone + 2;
    s.sbar = s.dfree + 2;
    s.xgbar = s.sbar + 2;
    s.mdone = s.xgbar + 4;
    s.ybar = s.mdone + 1;
    s.tmem_base = reinterpret_cast<uint32_t*>(s.ybar + 1);
    s.abort = reinterpret_cast<int*>(s.tmem_base + 1);
    return s;
}

struct PTile {
    int64_t n0;      // first W row
    int nvalid;      // valid W rows
    int64_t xrow0;   // first token within its batch
    int tvalid;      // valid tokens
    int b0, b1;      // launch batch
};

__device__ __forceinline__ PTile p_tile(const Params& p, int t) {
    PTile ti;
    const int wt = t % p.n_wtiles;
    const int rest = t / p.n_wtiles;
    const int tt = rest % p.n_ttiles;
    const int b = rest / p.n_ttiles;
    ti.n0 = (int64_t)wt * 128;
    ti.nvalid = (int)min64(128, p.N - ti.n0);
    ti.xrow0 = (int64_t)tt * NTP;
    ti.tvalid = (int)min64(NTP, p.M - ti.xrow0);
    ti.b1 = (int)(b % p.nb1);
    ti.b0 = (int)(b / p.nb1);
    return ti;
}

// fold thread tid copies groups [g0, min(g0 + 32, kg)) of row tid % 128 (scales below 128,
// biases above) with 4-byte asynchronous copies
__device__ __forceinline__ void p_issue_sb(const Params& p, const PTile& ti, int g0, uint16_t* slot, int tid) {
    const int pairs = min(SCW, p.kg - g0) >> 1;
    const int r = tid & 127, arr = tid >> 7;
    const int64_t row = ti.n0 + min(r, ti.nvalid - 1);
    const uint16_t* src = (arr ? p.biases : p.scales) + row * p.kg + g0;
    uint16_t* dst = slot + arr * 128 * SCP + r * SCP;
    for (int pr = 0; pr < pairs; ++pr) ptx::cp_async_4(dst + 2 * pr, src + 2 * pr);
}

template <int BITS, typename XT, int G>
__global__ void __launch_bounds__(P_THREADS, 1) qmm_prefill_kernel(const __grid_constant__ Params p) {
    constexpr int WSC = G;                      // one group per stage
    constexpr int ROWB = WSC * BITS / 8;
    constexpr int SUB = WSC / KB;
    constexpr int ACOLS = WSC / 2;
    constexpr int H = NTP / 2;                  // tokens per fold thread
    constexpr float OFF = code_offset<BITS, XT>();
    static_assert(SUB >= 1 && SUB <= 2, "prefill stages hold one group of 64 or 128 codes");

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // aligned by an offset from the shared array itself, so that every pointer derived from it stays
    // in the shared address space (shared loads and stores, not generic ones)
    uint8_t* base = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    const PSmem s = p_carve<SUB, ROWB>(base, p);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.stages, XS = p.xst;
    const int NWS = p.n_wstages;            // == groups per row
    const int ntiles = p.n_wtiles * p.n_ttiles * p.nbatch;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            ptx::mbar_init(&s.wfull[i], 1);
            ptx::mbar_init(&s.wfree[i], P_EXP);
        }
        for (int i = 0; i < XS; ++i) {
            ptx::mbar_init(&s.xfull[i], 1);
            ptx::mbar_init(&s.xfree[i], P_FOLD);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&s.afull[i], P_EXP);
            ptx::mbar_init(&s.sdone[i], 1);
            ptx::mbar_init(&s.dfree[i], P_FOLD);
            ptx::mbar_init(&s.sbar[i], P_FOLD_THREADS);
            ptx::mbar_init(&s.xgbar[i], P_FOLD_THREADS / 2);
            ptx::mbar_init(&s.xgbar[2 + i], P_FOLD_THREADS / 2);
        }
        ptx::mbar_init(s.mdone, 1);
        ptx::mbar_init(s.ybar, P_FOLD_THREADS);
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
    // programmatic dependent launch: nothing an earlier kernel may write is touched before this
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tbase = *s.tmem_base;
    const uint32_t d_tmem = tbase + (uint32_t)WSC;   // two accumulators of NTP columns follow the A blocks

    if (warp == 0) {
        // ======================= W producer =======================
        const bool leader = lane == 0;
        uint32_t wg = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const PTile ti = p_tile(p, t);
            for (int w = 0; w < NWS; ++w, ++wg) {
                const int st = wg % S;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.wfree[st], ((wg / S) & 1) ^ 1, s.abort, WAIT_NS));
                if (!ok) break;
                if (leader) {
                    ptx::mbar_arrive_expect_tx(&s.wfull[st], 128u * ROWB);
                    ptx::tma_load_2d(s.ws + (size_t)st * 128 * ROWB, &p.tw, &s.wfull[st], w * (ROWB / 4),
                                     (int32_t)ti.n0);
                }
            }
        }
        if (leader && !ok) {
            raise_abort(p, s.abort, DEVERR_AT_PF_W);
            volatile int never = 0;
            for (uint32_t j = wg >= (uint32_t)S ? wg - S : 0; j < wg; ++j)
                ptx::mbar_wait(&s.wfull[j % S], (j / S) & 1, &never, 200000000ull);
        }
        __syncwarp();
    } else if (warp == P_XPROD) {
        // ======================= x producer =======================
        const bool leader = lane == 0;
        uint32_t wg = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const PTile ti = p_tile(p, t);
            for (int w = 0; w < NWS; ++w, ++wg) {
                const int xs = wg % XS;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.xfree[xs], ((wg / XS) & 1) ^ 1, s.abort, WAIT_NS));
                if (!ok) break;
                if (leader) {
                    ptx::mbar_arrive_expect_tx(&s.xfull[xs], (uint32_t)SUB * NTP * 128);
#pragma unroll
                    for (int j = 0; j < SUB; ++j)
                        ptx::tma_load_4d(s.xs + ((size_t)xs * SUB + j) * NTP * 128, &p.tx, &s.xfull[xs],
                                         (w * SUB + j) * KB, (int32_t)ti.xrow0, ti.b1, ti.b0);
                }
            }
        }
        if (leader && !ok) {
            raise_abort(p, s.abort, DEVERR_AT_PF_X);
            volatile int never = 0;
            for (uint32_t j = wg >= (uint32_t)XS ? wg - XS : 0; j < wg; ++j)
                ptx::mbar_wait(&s.xfull[j % XS], (j / XS) & 1, &never, 200000000ull);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ======================= MMA issuer =======================
        const bool leader = lane == 0;
        uint32_t wg = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            for (int w = 0; w < NWS; ++w, ++wg) {
                const int slot = wg & 1;
                const uint32_t ph = (wg >> 1) & 1;
                const int xs = wg % XS;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.xfull[xs], (wg / XS) & 1, s.abort, WAIT_NS));
                if (!ok) break;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.afull[slot], ph, s.abort, WAIT_NS));
                if (!ok) break;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.dfree[slot], ph ^ 1, s.abort, WAIT_NS));
                if (!ok) break;
                ptx::tc_fence_after();
                if (leader) {
                    const uint32_t a_blk = tbase + (uint32_t)(slot * ACOLS);
                    const uint32_t d = d_tmem + (uint32_t)(slot * NTP);
                    const uint64_t bdesc = ptx::smem_desc_sw128(ptx::smem_u32(s.xs + (size_t)xs * SUB * NTP * 128));
#pragma unroll
                    for (int j = 0; j < SUB; ++j) {
#pragma unroll
                        for (int kk = 0; kk < KB / 16; ++kk) {
                            const uint32_t a = a_blk + (uint32_t)(j * 32 + kk * 8);
                            const uint64_t b = bdesc + (uint64_t)(j * (NTP * 128 / 16) + 2 * kk);
                            if (j == 0 && kk == 0) ptx::mma_ts_imm<0>(d, a, b, p.idesc);
                            else ptx::mma_ts_imm<1>(d, a, b, p.idesc);
                        }
                    }
                    ptx::mma_commit(&s.sdone[slot]);
                }
                __syncwarp();
            }
        }
        if (!ok && leader) raise_abort(p, s.abort, DEVERR_AT_PF_MMA);
        if (leader) {
            ptx::mma_commit(s.mdone);
            volatile int never = 0;
            ptx::mbar_wait(s.mdone, 0, &never, 200000000ull);
        }
        __syncwarp();
    } else if (warp < 2 + P_EXP) {
        // ======================= code expanders =======================
        const int q = warp & 3;
        const int row = 32 * q + lane;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        uint32_t wg = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            for (int w = 0; w < NWS; ++w, ++wg) {
                const int st = wg % S;
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.wfull[st], (wg / S) & 1, s.abort, WAIT_NS));
                if (!ok) break;
                const uint8_t* wstage = s.ws + (size_t)st * 128 * ROWB;
                uint32_t out[2 * SUB][16];
#pragma unroll
                for (int j = 0; j < SUB; ++j) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t wv[BITS];
                        load_w32<BITS, ROWB>(wstage, row, j, h, wv);
                        expand32<BITS, XT>(wv, out[2 * j + h]);
                    }
                }
                if (wg >= 2) {
                    ok = __all_sync(0xffffffffu,
                                    ptx::mbar_wait(&s.sdone[wg & 1], ((wg >> 1) & 1) ^ 1, s.abort, WAIT_NS));
                    if (!ok) break;
                    ptx::tc_fence_after();
                }
                const uint32_t a_blk = tbase + lane_base + (uint32_t)((wg & 1) * ACOLS);
#pragma unroll
                for (int i = 0; i < 2 * SUB; ++i) ptx::tmem_st16(a_blk + (uint32_t)(16 * i), out[i]);
                ptx::tc_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    ptx::mbar_arrive(&s.wfree[st]);
                    ptx::mbar_arrive(&s.afull[wg & 1]);
                }
            }
        }
        if (!ok) raise_abort(p, s.abort, DEVERR_AT_PF_EXP);
    } else {
        // ======================= folds =======================
        const int q = warp & 3;
        const int th = (warp - 2 - P_EXP) >> 2;   // token half
        const int row = 32 * q + lane;
        const int tid = threadIdx.x - 32 * (2 + P_EXP);   // 0..255
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        uint32_t wg = 0, ytile = 0;
        int unit = 0;
        bool ok = true;
        if ((int)blockIdx.x < ntiles) p_issue_sb(p, p_tile(p, blockIdx.x), 0, s.sb, tid);
        ptx::cp_async_commit();
        const uint16_t* sbslot = s.sb;
        int g_chunk0 = 0;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const PTile ti = p_tile(p, t);
            float2 acc[H / 2];
#pragma unroll
            for (int i = 0; i < H / 2; ++i) acc[i] = make_float2(0.0f, 0.0f);
            for (int w = 0; w < NWS; ++w, ++wg) {
                if (w % SCW == 0) {
                    // this stage opens a scale/bias chunk: its copies were issued a chunk earlier.
                    // (ytma: every tile opens with a chunk, and the store of the previous tile's y has
                    // read the staging tile before any fold thread passes this barrier)
                    ptx::cp_async_wait_all();
                    if (p.ytma && tid == 0) ptx::bulk_wait_read_all();
                    ptx::mbar_arrive(&s.sbar[unit & 1]);
                    ok = __all_sync(0xffffffffu,
                                    ptx::mbar_wait(&s.sbar[unit & 1], (unit >> 1) & 1, s.abort, WAIT_NS));
                    if (!ok) break;
                    sbslot = s.sb + (unit & 1) * 2 * 128 * SCP;
                    g_chunk0 = w;
                    uint16_t* nslot = s.sb + ((unit + 1) & 1) * 2 * 128 * SCP;
                    if (w + SCW < NWS) p_issue_sb(p, ti, w + SCW, nslot, tid);
                    else if (t + (int)gridDim.x < ntiles) p_issue_sb(p, p_tile(p, t + gridDim.x), 0, nslot, tid);
                    ptx::cp_async_commit();
                    ++unit;
                }
                const int slot = wg & 1;
                const int xs = wg % XS;
                // the MMAs of this stage are complete: its x block and accumulator are final
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.sdone[slot], (wg >> 1) & 1, s.abort, WAIT_NS));
                if (!ok) break;
                ptx::tc_fence_after();
                // ---- X_g of the stage's 128 tokens: thread pair (2t, 2t+1) sums token t's codes,
                //      first and second half, from the swizzled x block ----
                {
                    const int tok = tid >> 1, half = tid & 1;
                    const uint8_t* xrow = s.xs + (size_t)xs * SUB * NTP * 128 + (size_t)tok * 128;
                    float sum = 0.0f;
#pragma unroll
                    for (int c = 0; c < 4 * SUB; ++c) {
                        const int cg = half * 4 * SUB + c;                  // 16-byte chunk along the group
                        const int box = cg >> 3, ch = cg & 7;
                        const uint4 v = *reinterpret_cast<const uint4*>(xrow + (size_t)box * NTP * 128 +
                                                                        ((ch ^ (tok & 7)) << 4));
                        float f[8];
                        unpack8(v, f, XT{});
#pragma unroll
                        for (int e = 0; e < 8; ++e) sum += f[e];
                    }
                    const float other = __shfl_xor_sync(0xffffffffu, sum, 1);
                    if (half == 0) s.xg[slot * NTP + tok] = sum + other;
                }
                // the sums of a token half are written and read by that half's four fold warps only
                ptx::mbar_arrive(&s.xgbar[2 * th + slot]);
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(&s.xgbar[2 * th + slot], (wg >> 1) & 1, s.abort, WAIT_NS));
                if (!ok) break;
                if (lane == 0) ptx::mbar_arrive(&s.xfree[xs]);   // x block read by this warp
                // ---- y += s * D' + (b - OFF*s) * X_g ----
                const int gl = w - g_chunk0;
                const float sv = half_bits_to_float(sbslot[row * SCP + gl], XT{});
                const float bv = half_bits_to_float(sbslot[128 * SCP + row * SCP + gl], XT{});
                const float bo = OFF == 0.0f ? bv : fmaf(-OFF, sv, bv);
                const float2 s2 = make_float2(sv, sv), b2 = make_float2(bo, bo);
#pragma unroll
                for (int c0 = 0; c0 < H; c0 += 16) {
                    uint32_t v[16];
                    ptx::tmem_ld16(d_tmem + (uint32_t)(slot * NTP + th * H + c0) + lane_base, v);
                    const float* xg = s.xg + slot * NTP + th * H + c0;
                    ptx::tc_wait_ld();
#pragma unroll
                    for (int c = 0; c < 16; c += 4) {
                        const float4 xv = *reinterpret_cast<const float4*>(xg + c);
                        float2& a0 = acc[(c0 + c) / 2];
                        float2& a1 = acc[(c0 + c) / 2 + 1];
                        a0 = ptx::ffma2(b2, make_float2(xv.x, xv.y), a0);
                        a1 = ptx::ffma2(b2, make_float2(xv.z, xv.w), a1);
                        a0 = ptx::ffma2(s2, make_float2(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), a0);
                        a1 = ptx::ffma2(s2, make_float2(__uint_as_float(v[c + 2]), __uint_as_float(v[c + 3])), a1);
                    }
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&s.dfree[slot]);
            }
            if (!ok) break;
            if (p.ytma) {
                // ---- the tile's y: every fold thread writes its row of its 64 tokens into the
                //      staging tile, then one thread stores the tile with TMA (rows past N and
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
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(s.ybar, ytile & 1, s.abort, WAIT_NS));
                ++ytile;
                if (!ok) break;
                if (tid == 0) {
                    ptx::tma_store_4d(&p.ty, s.ystg, (int32_t)ti.n0, (int32_t)ti.xrow0, ti.b1, ti.b0);
                    ptx::bulk_commit_group();
                }
                continue;
            }
            // ---- this thread's row of y for its 64 tokens ----
            if (row < ti.nvalid) {
                const int64_t off = ti.xrow0 * p.y_row + ti.n0 + row + (int64_t)ti.b0 * p.yb[0] + (int64_t)ti.b1 * p.yb[1];
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
        if (!ok) raise_abort(p, s.abort, DEVERR_AT_PF_FOLD);
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tbase, p.tmem_cols);
    }
}

template <int BITS, typename XT, int G>
cudaError_t launch_pt(const Params& prm, int grid, size_t smem, cudaStream_t s) {
    static std::mutex mu;
    static bool done[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!done[dev]) {
            e = cudaFuncSetAttribute(qmm_prefill_kernel<BITS, XT, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)SMEM_LIMIT);
            if (e != cudaSuccess) return e;
            done[dev] = true;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(P_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, qmm_prefill_kernel<BITS, XT, G>, prm);
}

}  // namespace pf

template <int BITS>
cudaError_t launch_prefill(bool bf16, int group, const Params& prm, int grid, size_t smem, cudaStream_t stream) {
    if (group == 64)
        return bf16 ? pf::launch_pt<BITS, bf16_t, 64>(prm, grid, smem, stream)
                    : pf::launch_pt<BITS, f16_t, 64>(prm, grid, smem, stream);
    if (group == 128)
        return bf16 ? pf::launch_pt<BITS, bf16_t, 128>(prm, grid, smem, stream)
                    : pf::launch_pt<BITS, f16_t, 128>(prm, grid, smem, stream);
    return cudaErrorInvalidValue;
}

}  // namespace mma
}  // namespace aq
