// kernels_warp_mma.cu -- host side of the warp-level tensor-core kernel (warp_mma_kernel.cuh):
// which problems it takes and how a launch is shaped.
#include <cuda_runtime.h>
#include <string.h>

#include "aq_internal.h"
#include "warp_mma.cuh"

namespace aq {

namespace {

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

int tokens_per_tile(int64_t M) { return M <= 8 ? 8 : wm::TILE_TOKENS; }

// scales and biases of a CTA's rows, staged in shared memory
constexpr int64_t SB_MAX_BYTES = 64 * 1024;

struct Shape {
    int ntl, wr, wk, gpw, cs, kgc;
    int rd, ring_bytes;
    int x_pitch;
    bool xsm;
    dim3 grid;
    size_t smem;
};

// Warps of a CTA: wr blocks of 32 W rows while the CTAs still cover every SM, the rest slices
// of K.  The split of K depends on N, K and the total rows only (not on how the rows are
// grouped into launch batches), so a strided view and its contiguous copy sum in the same
// order and give the same bits.
// Row blocks (of wm::ROWS W rows, one per warp) of a launch: the plain W; the fused matrices one
// after another; or, for gate/up, 16 rows of each matrix per block.
int64_t row_blocks(const MmaProblem& p) {
    if (p.nseg <= 1) return (p.N + wm::ROWS - 1) / wm::ROWS;
    if (p.glu) return (p.seg_N[0] + wm::ROWS / 2 - 1) / (wm::ROWS / 2);
    int64_t n = 0;
    for (int s = 0; s < p.nseg; ++s) n += (p.seg_N[s] + wm::ROWS - 1) / wm::ROWS;
    return n;
}

Shape shape_for(const MmaProblem& p, int sms) {
    Shape s;
    const int nt = tokens_per_tile(p.M);
    s.ntl = nt / 8;
    const int64_t kg = p.K / p.group;
    const int64_t nrt = row_blocks(p);
    const int64_t rows_all = p.M * p.nb[0] * p.nb[1];
    const int64_t units = (rows_all + wm::TILE_TOKENS - 1) / wm::TILE_TOKENS;
    int wr = 1;
    while (wr < wm::MAX_WARPS && ((nrt + 2 * wr - 1) / (2 * wr)) * units >= sms &&
           (int64_t)(2 * wr) * wm::ROWS * kg * 4 <= SB_MAX_BYTES)
        wr *= 2;
    // one row block per CTA and still few CTAs: a cluster of cs CTAs splits K of each row block.
    // Not for short K (16 groups or fewer): there the split's two cluster barriers cost more than
    // the second K piece per warp it saves (chained decode launches at K 1024: 7.19 against 7.45 us)
    int cs = 1;
    if (wr == 1 && kg > 16)
        while (cs < wm::MAX_CLUSTER && nrt * units * cs * 2 <= sms && kg >= 4 * cs) cs *= 2;
    const int64_t kgc = (kg + cs - 1) / cs;
    int64_t wk = wm::MAX_WARPS / wr;
    if (wk > kgc) wk = kgc;
    const int64_t gpw = (kgc + wk - 1) / wk;
    wk = (kgc + gpw - 1) / gpw;
    s.wr = wr;
    s.wk = (int)wk;
    s.gpw = (int)gpw;
    s.cs = cs;
    s.kgc = (int)kgc;
    s.grid = dim3((unsigned)(((nrt + wr - 1) / wr) * cs), (unsigned)((p.M + nt - 1) / nt),
                  (unsigned)(p.nb[0] * p.nb[1]));
    s.x_pitch = (int)(2 * kgc * p.group + 16);
    // ring: a warp's sub-blocks, up to the depth RING_BYTES allows; at least the warp's partial tile
    const int ks = p.group < 64 ? p.group : 64, ksb = ks * p.bits / 8, spg = p.group / ks;
    int rdmax = wm::RING_BYTES / (wm::ROWS * ksb);
    if (rdmax > wm::MAX_RD) rdmax = wm::MAX_RD;
    s.rd = (int)(gpw * spg < rdmax ? gpw * spg : rdmax);
    if (s.rd < 1) s.rd = 1;
    s.ring_bytes = s.rd * wm::ROWS * ksb;
    const int red_bytes = nt * wm::RED_PITCH * 4;
    if (s.ring_bytes < red_bytes) s.ring_bytes = (red_bytes + 127) / 128 * 128;
    const bool rms = p.rms_eps > 0.0f;
    const size_t base = wm::smem_bytes(s.wr * s.wk, s.ring_bytes, s.wr, (int)kg, cs, nt, s.x_pitch, false, rms);
    s.xsm = base + (size_t)nt * s.x_pitch <= wm::SMEM_LIMIT;
    s.smem = wm::smem_bytes(s.wr * s.wk, s.ring_bytes, s.wr, (int)kg, cs, nt, s.x_pitch, s.xsm, rms);
    return s;
}

}  // namespace

bool warp_mma_supported(const MmaProblem& p) {
#if defined(AQ_WARP_MMA) && AQ_WARP_MMA == 0
    return false;
#endif
    if (p.offsets) return false;
    // by the total rows, so that a strided view and its contiguous copy run the same kernel
    if (p.M < 1 || p.M * p.nb[0] * p.nb[1] > wm::MAX_TOKENS || p.N < 1) return false;
    if (!(p.bits == 2 || p.bits == 4 || p.bits == 8)) return false;
    if (!(p.group == 32 || p.group == 64 || p.group == 128)) return false;
    if (p.bits * (p.group < 64 ? p.group : 64) < 128) return false;   // a lane's codes fill whole words
    if (p.K % p.group != 0 || p.K < p.group) return false;
    const int64_t kg = p.K / p.group;
    if ((size_t)kg * wm::MAX_TOKENS * sizeof(float) > (size_t)wm::MAX_XTAB_BYTES) return false;
    if ((int64_t)wm::ROWS * kg * 4 > SB_MAX_BYTES) return false;
    if (p.nb[0] * p.nb[1] > 65535 || row_blocks(p) > 0x7fffffff) return false;
    // 16-byte rows of x and W, as the tensor-core kernels require (checked by mma_supported)
    return true;
}

// Whether the warp kernel is the faster choice for a problem it supports.  Measured on B200 at
// 8/16/32 tokens against the tcgen05 small-M kernel (decode shapes, K 1024..3072, N 1024..151936):
// the warp kernel wins every case of up to 8 tokens; at 16 tokens unless the CTA holds the most
// row blocks and a warp more than eight 64-code sub-blocks of K (lm_head: eight row blocks and
// sixteen sub-blocks per warp, 99 us against 64 us on the tcgen05 kernel); at 32 tokens when each warp of a one-row-block CTA has at most four sub-blocks (after
// a cluster split of K); with many row blocks per CTA its serial per-warp work outweighs the
// tcgen05 kernel's fixed costs.
// The choice depends on N, K and the total rows only.
bool warp_mma_preferred(const MmaProblem& p) {
#if defined(AQ_WARP_MMA) && AQ_WARP_MMA == 2
    return true;
#endif
    const Shape s = shape_for(p, sm_count());
    const int64_t rows = p.M * p.nb[0] * p.nb[1];
    const int spg = p.group > 64 ? p.group / 64 : 1;
    if (rows <= 8) return true;
    if (rows <= 16) return !(s.wr == wm::MAX_WARPS && s.gpw * spg > 8);
    return s.wr == 1 && s.gpw * spg <= 4;
}

cudaError_t launch_warp_mma(const MmaProblem& pb, cudaStream_t stream) {
    const Shape s = shape_for(pb, sm_count());
    wm::WParams p;
    memset(&p, 0, sizeof p);
    p.x = static_cast<const uint16_t*>(pb.x);
    const bool fused = pb.nseg > 1;
    p.nseg = fused ? pb.nseg : 1;
    p.glu = fused && pb.glu ? 1 : 0;
    int64_t rb = 0;
    for (int i = 0; i < p.nseg; ++i) {
        wm::WSeg& g = p.seg[i];
        g.wq = fused ? pb.seg_wq[i] : pb.wq;
        g.scales = static_cast<const uint16_t*>(fused ? pb.seg_scales[i] : pb.scales);
        g.biases = static_cast<const uint16_t*>(fused ? pb.seg_biases[i] : pb.biases);
        g.y = fused ? pb.seg_y[i] : pb.y;
        g.N = fused ? pb.seg_N[i] : pb.N;
        g.w_row = fused ? pb.seg_w_row[i] : pb.w_row;
        g.y_row = fused ? pb.seg_y_row[i] : pb.y_row;
        g.rb0 = p.glu ? 0 : rb;
        g.r = fused ? nullptr : pb.r;
        g.r_row = pb.r_row;
        rb += (g.N + wm::ROWS - 1) / wm::ROWS;
    }
    p.nrb = row_blocks(pb);
    p.M = pb.M;
    p.K = pb.K;
    p.x_row = pb.x_row;
    for (int i = 0; i < 2; ++i) {
        p.xb[i] = pb.nb[i] > 1 ? pb.xb[i] : 0;
        p.yb[i] = pb.nb[i] > 1 ? pb.yb[i] : 0;
    }
    p.nb1 = pb.nb[1] > 0 ? pb.nb[1] : 1;
    p.kg = (int)(pb.K / pb.group);
    p.cs = s.cs;
    p.kgc = s.kgc;
    p.gpw = s.gpw;
    p.wr = s.wr;
    p.wk = s.wk;
    p.ydt = (int)pb.ydt;
    const size_t ysz = pb.ydt == DT::F32 ? 4 : 2;
    bool yvec = true, sb16 = p.kg % 8 == 0;
    for (int i = 0; i < p.nseg; ++i) {
        if (((uintptr_t)p.seg[i].y % (2 * ysz)) != 0 || (pb.M > 1 && p.seg[i].y_row % 2 != 0)) yvec = false;
        if (((uintptr_t)p.seg[i].scales & 15) || ((uintptr_t)p.seg[i].biases & 15)) sb16 = false;
    }
    for (int i = 0; i < 2; ++i)
        if (pb.nb[i] > 1 && pb.yb[i] % 2 != 0) yvec = false;
    p.yvec = yvec ? 1 : 0;
    p.xsm = s.xsm ? 1 : 0;
    p.x_pitch = s.x_pitch;
    p.sb16 = sb16 ? 1 : 0;
    p.rd = s.rd;
    p.ring_bytes = s.ring_bytes;
    p.rms = pb.rms_eps > 0.0f ? 1 : 0;
    p.rms_eps = pb.rms_eps;
    cudaError_t e = device_error_ptr(&p.err);
    if (e != cudaSuccess) return e;
    // W boxes: one ring sub-block (min(G, 64) codes) of 32 rows, or 16 rows per matrix for gate/up
    const int ks = pb.group < 64 ? pb.group : 64;
    const int box_words = ks * pb.bits / 32;
    for (int i = 0; i < p.nseg; ++i)
        if (!encode_w_rows(&p.tw[i], p.seg[i].wq, pb.K * pb.bits / 32, p.seg[i].N, p.seg[i].w_row, box_words,
                           p.glu ? wm::ROWS / 2 : wm::ROWS))
            return cudaErrorInvalidValue;
    const bool bf = pb.xdt == DT::BF16;
    const int warps = s.wr * s.wk;
    switch (pb.bits) {
        case 2: return wm::launch<2>(bf, pb.group, s.ntl, p, s.grid, warps, s.smem, stream);
        case 4: return wm::launch<4>(bf, pb.group, s.ntl, p, s.grid, warps, s.smem, stream);
        case 8: return wm::launch<8>(bf, pb.group, s.ntl, p, s.grid, warps, s.smem, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace aq
