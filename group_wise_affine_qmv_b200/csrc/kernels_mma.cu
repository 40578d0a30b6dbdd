// kernels_mma.cu -- host side of the tensor-core kernel (mma_kernel.cuh): shared-memory and
// x-residency planning, TMA descriptors, grid size, and the device error word.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "aq_internal.h"
#include "mma_common.cuh"
#include "sm100_ptx.cuh"

namespace aq {

// Error bits set on the device (DEVERR_TIMEOUT by any tensor-core CTA whose bounded wait expired,
// DEVERR_INDEX by a row gather given an id out of range); read and cleared by aq_device_error().
// Kernels receive its address in their parameters.
__device__ int g_device_error = 0;

namespace {

using namespace mma;

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

// device address of a __device__ symbol, looked up once per device
template <typename T>
cudaError_t symbol_address(const T& sym, void** cache, void** out) {
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu);
    if (!cache[dev]) {
        e = cudaGetSymbolAddress(&cache[dev], sym);
        if (e != cudaSuccess) return e;
    }
    *out = cache[dev];
    return cudaSuccess;
}

constexpr size_t SMEM_LIMIT = 227 * 1024;
constexpr int MIN_STAGES = 3;

struct Geom {
    int wsc, rowb, sub;   // codes, bytes per W row and 64-code sub-steps of one W stage
};
Geom geometry(int bits, int group) {
    Geom g;
    g.wsc = stage_codes(bits, group);
    g.rowb = stage_rowb(bits, group);
    g.sub = g.wsc / KB;
    return g;
}

// Shared memory of one CTA whose K range spans at most `ms` W stages: x (that range when
// resident, else `xst` x stages of SUB boxes), the sum-of-x table of the range, the partial
// tile of a split, the staged y tile (`ystg` bytes, 0 without), and the fixed part.
size_t fixed_bytes(int64_t K, int64_t kg, int ms, int split, int xres, int xst, const Geom& g, size_t ystg) {
    const int64_t boxes = std::min<int64_t>((int64_t)ms * g.sub, K / KB);
    const int64_t groups = std::min<int64_t>((int64_t)ms * (g.wsc / (K / kg)), kg);
    return (xres ? (size_t)boxes * NT * 128 : (size_t)xst * g.sub * NT * 128) + (size_t)groups * NT * 4 +
           (split > 1 ? (size_t)RED_BYTES : 0) + ystg + smem_fixed_bytes();
}
size_t smem_for(int stages, int64_t K, int64_t kg, int ms, int split, int xres, int xst, const Geom& g, size_t ystg) {
    return (size_t)stages * 128 * g.rowb + fixed_bytes(K, kg, ms, split, xres, xst, g, ystg);
}
int pick_stages(int64_t K, int64_t kg, int ms, int split, int xres, int xst, const Geom& g, size_t ystg = 0) {
    const size_t fixed = fixed_bytes(K, kg, ms, split, xres, xst, g, ystg);
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
XPlan pick_x(const MmaProblem& p, int64_t kg, int ms, int split, const Geom& g, size_t ystg) {
    XPlan r{0, 2, 0};
    if (!p.offsets && p.M <= NT && p.nb[0] * p.nb[1] == 1 && pick_stages(p.K, kg, ms, split, 1, 0, g, ystg) >= 6) {
        r.xres = 1;
        r.xst = 0;
    } else {
        for (int xst = MAX_XST; xst > 2; --xst)
            if (pick_stages(p.K, kg, ms, split, 0, xst, g, ystg) >= 4) {
                r.xst = xst;
                break;
            }
    }
    r.stages = pick_stages(p.K, kg, ms, split, r.xres, r.xst, g, ystg);
    return r;
}

// CTAs per cluster splitting each tile's K: when the tiles alone would leave most SMs idle,
// the largest power of two <= 8 that keeps the grid within the SMs and gives every rank
// at least one W stage (two when a stage holds one group).  Clusters of 8 only while the grid
// stays within 64 CTAs: more of them than that could not all be placed at once next to the
// tail of the previous kernel (a cluster needs its SMs free in one GPC).
int pick_split(int64_t tiles, int nws, int gps, int sms) {
    const int u = gps == 1 ? 2 : 1;
    const int nu = (nws + u - 1) / u;
    int cs = 1;
    while (cs < 8 && tiles * cs * 2 <= sms && cs * 2 <= nu && (cs < 4 || tiles * cs * 2 <= 64)) cs *= 2;
    return cs;
}

}  // namespace

bool mma_supported(const MmaProblem& p, const char** why) {
    auto no = [&](const char* r) { if (why) *why = r; return false; };
    if (!(p.bits == 2 || p.bits == 4 || p.bits == 6 || p.bits == 8)) return no("tensor-core kernel takes bits 2/4/6/8");
    if (!(p.group == 32 || p.group == 64 || p.group == 128)) return no("tensor-core kernel takes groups 32/64/128");
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
    const Geom g = geometry(p.bits, p.group);
    if ((size_t)kg * NT * 4 > XTAB_MAX_BYTES ||
        pick_stages(p.K, kg, (int)((p.K + g.wsc - 1) / g.wsc), 1, 0, 2, g) < MIN_STAGES)
        return no("K/group too large for the sum-of-x table of the tensor-core kernel");
    if (!get_encode()) return no("driver entry point cuTensorMapEncodeTiled unavailable");
    return true;
}

namespace {

CUtensorMapSwizzle swizzle_for(int rowb) {
    switch (rowb) {
        case 128: return CU_TENSOR_MAP_SWIZZLE_128B;
        case 64: return CU_TENSOR_MAP_SWIZZLE_64B;
        case 32: return CU_TENSOR_MAP_SWIZZLE_32B;
        default: return CU_TENSOR_MAP_SWIZZLE_NONE;
    }
}

// x viewed as {K, rows, nb1, nb0} bf16/f16 bits, box {64 codes, `box_rows` tokens}, 128-byte swizzle
CUresult encode_x(PFN_cuTensorMapEncodeTiled_v12000 encode, CUtensorMap* m, const MmaProblem& pb, int box_rows) {
    const int64_t rows_total = pb.M;
    cuuint64_t dims[4] = {(cuuint64_t)pb.K, (cuuint64_t)rows_total, (cuuint64_t)pb.nb[1], (cuuint64_t)pb.nb[0]};
    const int64_t rowb = rows_total > 1 ? pb.x_row * 2 : (pb.K * 2 + 15) / 16 * 16;
    const int64_t s1 = pb.nb[1] > 1 ? pb.xb[1] * 2 : rowb * rows_total;
    const int64_t s2 = pb.nb[0] > 1 ? pb.xb[0] * 2 : s1 * (int64_t)pb.nb[1];
    cuuint64_t strides[3] = {(cuuint64_t)rowb, (cuuint64_t)((s1 + 15) / 16 * 16), (cuuint64_t)((s2 + 15) / 16 * 16)};
    cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, const_cast<void*>(pb.x), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// W viewed as {K*bits/32 words, rows}, box {rowb/4 words, 128 rows}
CUresult encode_w(PFN_cuTensorMapEncodeTiled_v12000 encode, CUtensorMap* m, const MmaProblem& pb, int rowb) {
    const int64_t wrows = pb.offsets ? pb.N * pb.n_experts : pb.N;
    cuuint64_t dims[2] = {(cuuint64_t)(pb.K * pb.bits / 32), (cuuint64_t)wrows};
    cuuint64_t strides[1] = {(cuuint64_t)(pb.w_row * 4)};
    cuuint32_t box[2] = {(cuuint32_t)(rowb / 4), 128};
    cuuint32_t estr[2] = {1, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(pb.wq), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_for(rowb), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// y viewed as {N, rows, nb1, nb0} bf16/f16 bits, box {128 rows of W, `box_rows` tokens}: the store of
// one tile (TMA writes nothing outside the tensor, so a tile's rows past N and tokens past M are dropped)
CUresult encode_y(PFN_cuTensorMapEncodeTiled_v12000 encode, CUtensorMap* m, const MmaProblem& pb, int box_rows) {
    const int64_t rows_total = pb.M;
    cuuint64_t dims[4] = {(cuuint64_t)pb.N, (cuuint64_t)rows_total, (cuuint64_t)pb.nb[1], (cuuint64_t)pb.nb[0]};
    const int64_t rowb = rows_total > 1 ? pb.y_row * 2 : (pb.N * 2 + 15) / 16 * 16;
    const int64_t s1 = pb.nb[1] > 1 ? pb.yb[1] * 2 : rowb * rows_total;
    const int64_t s2 = pb.nb[0] > 1 ? pb.yb[0] * 2 : s1 * (int64_t)pb.nb[1];
    cuuint64_t strides[3] = {(cuuint64_t)rowb, (cuuint64_t)((s1 + 15) / 16 * 16), (cuuint64_t)((s2 + 15) / 16 * 16)};
    cuuint32_t box[4] = {128, (cuuint32_t)box_rows, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, pb.y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// Whether the tiles of y can go out as TMA stores: plain (not grouped, no split of K) calls whose y
// has x's 16-bit type, 16-byte aligned rows and batch strides, and N a multiple of 8 (a tile store
// writes whole 16-byte pieces of a row: on this B200 a piece that straddles N was written in full,
// past the end of the row)
bool y_tma_ok(const MmaProblem& pb, int split) {
    if (pb.offsets || split > 1 || pb.ydt != pb.xdt || pb.N % 8 != 0) return false;
    if (((uintptr_t)pb.y & 15) || (pb.M > 1 && pb.y_row % 8 != 0)) return false;
    for (int i = 0; i < 2; ++i)
        if (pb.nb[i] > 1 && pb.yb[i] % 8 != 0) return false;
    return true;
}

void fill_common(Params& prm, const MmaProblem& pb) {
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
    prm.nbatch = (int)(pb.nb[0] * pb.nb[1]);
    prm.kg = (int)(pb.K / pb.group);
    prm.ydt = (int)pb.ydt;
    prm.offsets = pb.offsets;
    prm.n_experts = pb.n_experts;
    prm.ksplit = 1;
}

cudaError_t device_pointers(Params& prm) {
    static void* cache[64] = {nullptr};
    void* a = nullptr;
    cudaError_t e = symbol_address(g_device_error, cache, &a);
    if (e != cudaSuccess) return e;
    prm.err = static_cast<int*>(a);
    return cudaSuccess;
}

// Prefill: 128 W rows x 128 tokens per tile, one group per W stage (groups of 64 or 128)
bool prefill_eligible(const MmaProblem& pb) {
    return !pb.offsets && pb.M >= 64 && (pb.group == 64 || pb.group == 128);
}

// Shared memory plan of the prefill kernel for a problem: x ring depth, W ring depth and whether
// the tiles of y are staged for bulk tensor stores
struct PrefillPlan {
    bool ok;
    int xst, stages;
    size_t fixed, wstage;
    bool ytma;
};
PrefillPlan plan_prefill(const MmaProblem& pb) {
    using namespace pf;
    PrefillPlan r{};
    const int sub = pb.group / KB;
    const int rowb = pb.group * pb.bits / 8;
    const size_t xstage = (size_t)sub * NTP * 128;
    r.wstage = (size_t)128 * rowb;
    r.xst = sub == 1 ? 4 : 3;
    r.fixed = (size_t)r.xst * xstage + p_fixed_bytes();
    if (r.fixed + 4 * r.wstage > SMEM_LIMIT) return r;
    r.ok = true;
    r.stages = (int)((SMEM_LIMIT - r.fixed) / r.wstage);
    if (r.stages > P_MAX_STAGES) r.stages = P_MAX_STAGES;
    // the staged y tile (32 KB) takes shared memory from the W ring where that leaves it at least
    // 8 stages deep (or as deep as without it)
    r.ytma = y_tma_ok(pb, 1);
    if (r.ytma) {
        const size_t f1 = r.fixed + P_YSTG_BYTES;
        int s1 = f1 + 4 * r.wstage <= SMEM_LIMIT ? (int)((SMEM_LIMIT - f1) / r.wstage) : 0;
        if (s1 > P_MAX_STAGES) s1 = P_MAX_STAGES;
        r.ytma = s1 >= 4 && (s1 == r.stages || s1 >= 8);
        if (r.ytma) {
            r.fixed = f1;
            r.stages = s1;
        }
    }
    return r;
}

cudaError_t launch_prefill_problem(const MmaProblem& pb, cudaStream_t stream) {
    auto encode = get_encode();
    if (!encode) return cudaErrorNotSupported;
    using namespace pf;
    Params prm;
    memset(&prm, 0, sizeof prm);
    const int rowb = pb.group * pb.bits / 8;
    const PrefillPlan pl = plan_prefill(pb);
    if (!pl.ok) return cudaErrorInvalidValue;
    const int xst = pl.xst, stages = pl.stages;
    const bool ytma = pl.ytma;
    const size_t fixed = pl.fixed, wstage = pl.wstage;
    if (encode_x(encode, &prm.tx, pb, NTP) != CUDA_SUCCESS) return cudaErrorInvalidValue;
    if (encode_w(encode, &prm.tw, pb, rowb) != CUDA_SUCCESS) return cudaErrorInvalidValue;
    fill_common(prm, pb);
    prm.n_ttiles = (int)((pb.M + NTP - 1) / NTP);
    prm.n_wstages = (int)(pb.K / pb.group);
    prm.stages = stages;
    prm.xst = xst;
    prm.ytma = ytma ? 1 : 0;
    if (ytma && encode_y(encode, &prm.ty, pb, NTP) != CUDA_SUCCESS) return cudaErrorInvalidValue;
    prm.tmem_cols = 512;   // [A block 0 | A block 1 | 2 accumulators of 128 columns]
    prm.idesc = ptx::idesc_f16(NTP, pb.xdt == DT::BF16 ? 1 : 0);
    cudaError_t e = device_pointers(prm);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (int64_t)prm.n_wtiles * prm.n_ttiles * prm.nbatch;
    const int sms = num_sms();
    const int grid = (int)(tiles < sms ? tiles : sms);
    const size_t smem = fixed + (size_t)stages * wstage;
    const bool bf = pb.xdt == DT::BF16;
    switch (pb.bits) {
        case 2: return launch_prefill<2>(bf, pb.group, prm, grid, smem, stream);
        case 4: return launch_prefill<4>(bf, pb.group, prm, grid, smem, stream);
        case 6: return launch_prefill<6>(bf, pb.group, prm, grid, smem, stream);
        case 8: return launch_prefill<8>(bf, pb.group, prm, grid, smem, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

MmaKernel mma_kernel_for(const MmaProblem& pb) {
    if (prefill_eligible(pb)) return MmaKernel::PREFILL;
    if (warp_mma_supported(pb) && warp_mma_preferred(pb)) return MmaKernel::WARP;
    return MmaKernel::SMALL_M;
}

namespace {

// Plan of the small-M kernel for a problem: split of K over a cluster, x residency and ring
// depths, and whether the tiles of y are staged for bulk tensor stores
struct SmallMPlan {
    int split, ms;
    XPlan xp;
    bool ytma;
};
SmallMPlan plan_small_m(const MmaProblem& pb) {
    SmallMPlan r{};
    const int64_t kg = pb.K / pb.group;
    const Geom geo = geometry(pb.bits, pb.group);
    const int nws = (int)((pb.K + geo.wsc - 1) / geo.wsc);
    const int gps = geo.wsc / pb.group;
    // The split depends on the total rows, not on how they are grouped into launch batches, so
    // that a strided view and its contiguous copy take the same split (and give the same bits).
    const int64_t rows_all = pb.M * pb.nb[0] * pb.nb[1];
    r.split = pb.offsets ? 1 : pick_split(((pb.N + 127) / 128) * ((rows_all + NT - 1) / NT), nws, gps, num_sms());
    r.ms = r.split > 1 ? split_max_stages(nws, gps, r.split) : nws;
    // the staged y tile takes shared memory from the W ring: only where that keeps x resident (if it
    // was) and the ring at least 4 stages deep (or as deep as without it)
    const XPlan xp0 = pick_x(pb, kg, r.ms, r.split, geo, 0);
    r.ytma = y_tma_ok(pb, r.split);
    r.xp = xp0;
    if (r.ytma) {
        const XPlan xp1 = pick_x(pb, kg, r.ms, r.split, geo, YSTG_BYTES);
        r.ytma = xp1.xres == xp0.xres && (xp1.stages == xp0.stages || xp1.stages >= 4);
        if (r.ytma) r.xp = xp1;
    }
    return r;
}

}  // namespace

bool mma_y_tiles(const MmaProblem& pb) {
    switch (mma_kernel_for(pb)) {
        case MmaKernel::PREFILL: {
            const PrefillPlan pl = plan_prefill(pb);
            return pl.ok && pl.ytma;
        }
        case MmaKernel::SMALL_M: return plan_small_m(pb).ytma;
        default: return false;
    }
}

cudaError_t launch_mma(const MmaProblem& pb, cudaStream_t stream) {
    const MmaKernel kind = mma_kernel_for(pb);
    if (kind == MmaKernel::PREFILL) return launch_prefill_problem(pb, stream);
    if (kind == MmaKernel::WARP) return launch_warp_mma(pb, stream);
    auto encode = get_encode();
    if (!encode) return cudaErrorNotSupported;
    Params prm;
    memset(&prm, 0, sizeof prm);
    const int bits = pb.bits;
    const int64_t kg = pb.K / pb.group;
    const Geom geo = geometry(bits, pb.group);
    const int nws = (int)((pb.K + geo.wsc - 1) / geo.wsc);
    const int sms = num_sms();
    const int64_t tiles = pb.offsets ? 0 : ((pb.N + 127) / 128) * ((pb.M + NT - 1) / NT) * pb.nb[0] * pb.nb[1];
    const SmallMPlan pl = plan_small_m(pb);
    const int split = pl.split, ms = pl.ms;
    const XPlan xp = pl.xp;
    const bool ytma = pl.ytma;
    const int stages = xp.stages;
    if (stages < MIN_STAGES) return cudaErrorInvalidValue;
    if (encode_x(encode, &prm.tx, pb, NT) != CUDA_SUCCESS) return cudaErrorInvalidValue;
    if (encode_w(encode, &prm.tw, pb, geo.rowb) != CUDA_SUCCESS) return cudaErrorInvalidValue;
    fill_common(prm, pb);
    prm.n_ttiles = (int)((pb.M + NT - 1) / NT);
    prm.n_wstages = nws;
    prm.ksplit = split;
    prm.stages = stages;
    prm.xres = xp.xres;
    prm.xst = xp.xst;
    prm.ytma = ytma ? 1 : 0;
    if (ytma && encode_y(encode, &prm.ty, pb, NT) != CUDA_SUCCESS) return cudaErrorInvalidValue;
    // [A block 0 | A block 1 | 2 x (WSC / group) accumulators of NT columns], a power of two >= 32
    uint32_t cols = (uint32_t)(geo.wsc + 2 * (geo.wsc / pb.group) * NT), pw = 32;
    while (pw < cols) pw <<= 1;
    prm.tmem_cols = pw;
    prm.idesc = ptx::idesc_f16(NT, pb.xdt == DT::BF16 ? 1 : 0);
    {
        cudaError_t e = device_pointers(prm);
        if (e != cudaSuccess) return e;
    }

    int grid;
    if (pb.offsets) grid = sms;
    else if (split > 1) grid = (int)tiles * split;   // one tile per cluster
    else grid = (int)(tiles < sms ? tiles : sms);
    const size_t smem = smem_for(stages, pb.K, kg, ms, split, xp.xres, xp.xst, geo, ytma ? YSTG_BYTES : 0);
    const bool bf = pb.xdt == DT::BF16;
    switch (bits) {
        case 2: return launch<2>(bf, pb.group, prm, grid, smem, stream);
        case 4: return launch<4>(bf, pb.group, prm, grid, smem, stream);
        case 6: return launch<6>(bf, pb.group, prm, grid, smem, stream);
        case 8: return launch<8>(bf, pb.group, prm, grid, smem, stream);
    }
    return cudaErrorInvalidValue;
}

// Check of the bounded waits every pipeline kernel uses: one warp waits, with the same bounded
// wait, on an mbarrier that nothing arrives on (no copy or MMA is tied to it), for `budget_ns`,
// and records DEVERR_TIMEOUT as a pipeline kernel whose wait expired does.
__global__ void __launch_bounds__(32) bounded_wait_check_kernel(int* err, uint64_t budget_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        abort_flag = 0;
        ptx::fence_mbar_init();
    }
    __syncwarp();
    const bool done = ptx::mbar_wait(&bar, 0, &abort_flag, budget_ns);
    if (!done && threadIdx.x == 0) atomicOr(err, DEVERR_TIMEOUT | DEVERR_AT_CHECK);
}

cudaError_t launch_bounded_wait_check(uint64_t budget_ns, cudaStream_t s) {
    int* err = nullptr;
    cudaError_t e = device_error_ptr(&err);
    if (e != cudaSuccess) return e;
    bounded_wait_check_kernel<<<1, 32, 0, s>>>(err, budget_ns);
    return cudaGetLastError();
}

bool encode_w_rows(void* map, const uint32_t* wq, int64_t words, int64_t rows, int64_t row_stride_words,
                   int box_words, int box_rows) {
    auto encode = get_encode();
    if (!encode) return false;
    cuuint64_t dims[2] = {(cuuint64_t)words, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(row_stride_words * 4)};
    cuuint32_t box[2] = {(cuuint32_t)box_words, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return encode(static_cast<CUtensorMap*>(map), CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(wq), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t device_error_ptr(int** out) {
    static void* cache[64] = {nullptr};
    void* a = nullptr;
    cudaError_t e = symbol_address(g_device_error, cache, &a);
    if (e != cudaSuccess) return e;
    *out = static_cast<int*>(a);
    return cudaSuccess;
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
