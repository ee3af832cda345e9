// api.cu -- the C ABI of libtriattn.so (declared in include/tri_attn.h):
// host-side validation, TMA descriptor encoding and kernel launches.
//
// Validation happens entirely on the host before any CUDA call, so argument
// errors are reported without touching the device.  The driver's tensor-map
// encoder is fetched through the runtime's driver entry point, so the library
// has no link-time dependency on libcuda.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/tri_attn.h"
#include "sm100.cuh"
#include "fwd.cuh"
#include "bwd.cuh"
#include "dbias.cuh"
#include "tri_mul.cuh"
#include "tri_gate.cuh"

namespace {

std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};

constexpr int kMaxN = 4096;
constexpr int kMaxDevices = 64;

// ---------------------------------------------------------------------------
// validation helpers
// ---------------------------------------------------------------------------
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

tri_attn_status check_t5(const tri_attn_tensor5& t) {
    if (!t.ptr) return TRI_ATTN_ERR_NULL;
    if (t.stride[4] != 1) return TRI_ATTN_ERR_STRIDE;
    for (int a = 0; a < 4; ++a)
        if (t.stride[a] < 0 || (t.stride[a] % 8) != 0) return TRI_ATTN_ERR_STRIDE;
    if (!aligned16(t.ptr)) return TRI_ATTN_ERR_ALIGN;
    return TRI_ATTN_OK;
}
tri_attn_status check_t4(const tri_attn_tensor4& t) {
    if (!t.ptr) return TRI_ATTN_ERR_NULL;
    if (t.stride[3] != 1) return TRI_ATTN_ERR_STRIDE;
    for (int a = 0; a < 3; ++a)
        if (t.stride[a] < 0 || (t.stride[a] % 8) != 0) return TRI_ATTN_ERR_STRIDE;
    if (!aligned16(t.ptr)) return TRI_ATTN_ERR_ALIGN;
    return TRI_ATTN_OK;
}

tri_attn_status check_sizes(int B, int N, int H, int d) {
    if (B < 1 || N < 1 || H < 1) return TRI_ATTN_ERR_SHAPE;
    if (d != 32 && d != 64) return TRI_ATTN_ERR_UNSUPPORTED;
    if (N > kMaxN) return TRI_ATTN_ERR_UNSUPPORTED;
    // 32-bit work-item and index arithmetic inside the kernels
    const double items = static_cast<double>(B) * H * N * ((N + 127) / 128);
    if (items > 2.0e9) return TRI_ATTN_ERR_SHAPE;
    return TRI_ATTN_OK;
}

tri_attn_status check_fwd_args(const tri_attn_fwd_args* a) {
    if (!a) return TRI_ATTN_ERR_NULL;
    tri_attn_status st = check_sizes(a->B, a->N, a->H, a->d);
    if (st) return st;
    const tri_attn_tensor5* t5[] = {&a->q, &a->k, &a->v, &a->o, &a->resid};
    for (const auto* t : t5)
        if ((st = check_t5(*t))) return st;
    if ((st = check_t4(a->bias))) return st;
    if (!a->lse) return TRI_ATTN_ERR_NULL;
    if (!aligned16(a->lse)) return TRI_ATTN_ERR_ALIGN;
    if (a->mask.ptr && (reinterpret_cast<uintptr_t>(a->mask.ptr) & 3u)) return TRI_ATTN_ERR_ALIGN;
    if (!std::isfinite(a->scale)) return TRI_ATTN_ERR_SHAPE;
    return TRI_ATTN_OK;
}

// ---------------------------------------------------------------------------
// device checks and the driver's tensor-map encoder
// ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// 0 unknown, 1 ok (sm_100 and kernel attributes set), 2 wrong arch
std::atomic<int> g_dev_state[kMaxDevices];

tri_attn_status ensure_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
        cudaGetLastError();
        return TRI_ATTN_ERR_CUDA;
    }
    if (dev >= kMaxDevices) return TRI_ATTN_ERR_CUDA;
    int s = g_dev_state[dev].load();
    if (s == 1) return TRI_ATTN_OK;
    if (s == 2) return TRI_ATTN_ERR_ARCH;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return TRI_ATTN_ERR_CUDA;
    }
    if (major != 10 || minor != 0) {
        g_dev_state[dev].store(2);
        return TRI_ATTN_ERR_ARCH;
    }
    bool ok = true;
    ok &= cudaFuncSetAttribute(tri::tri_attn_fwd_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               tri::FwdLayout<32>::SMEM) == cudaSuccess;
    ok &= cudaFuncSetAttribute(tri::tri_attn_fwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               tri::FwdLayout<64>::SMEM) == cudaSuccess;
    ok &= tri::bwd_set_attributes();
    ok &= cudaFuncSetAttribute(tri::tri_mul_gemm_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               tri::TriMulLayout::SMEM) == cudaSuccess;
    ok &= cudaFuncSetAttribute(tri::tri_mul_gemm_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               tri::TriMulLayout::SMEM) == cudaSuccess;
    ok &= cudaFuncSetAttribute(tri::tri_mul_gemm_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               tri::TriMulLayout::SMEM) == cudaSuccess;
    ok &= cudaFuncSetAttribute(tri::tri_gate_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               tri::TriGateLayout::SMEM) == cudaSuccess;
    ok &= cudaFuncSetAttribute(tri::tri_gate_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               tri::TriGateBwdLayout::SMEM) == cudaSuccess;
    if (!ok || !encoder()) {
        cudaGetLastError();
        return TRI_ATTN_ERR_CUDA;
    }
    g_dev_state[dev].store(1);
    return TRI_ATTN_OK;
}

// Encode a tiled BF16 map with the outer dimensions in the given (fixed) order.
// Strides need not be monotonic (an ending-node view swaps the j and i
// strides); a size-1 dimension's stride is irrelevant and is replaced by a
// harmless 16-byte multiple.
bool encode_map(CUtensorMap* m, void* ptr, uint64_t inner, uint32_t inner_box, const uint64_t* size,
                const uint64_t* stride_bytes, const uint32_t* box, int nouter, CUtensorMapSwizzle swz) {
    cuuint64_t dims[5], strides[4];
    cuuint32_t boxd[5], estr[5] = {1, 1, 1, 1, 1};
    dims[0] = inner;
    boxd[0] = inner_box;
    for (int a = 0; a < nouter; ++a) {
        dims[a + 1] = size[a];
        boxd[a + 1] = box[a];
        uint64_t st = stride_bytes[a];
        if (size[a] == 1) st = 16;
        if (st == 0 || st % 16 || st >= (1ull << 40)) return false;
        strides[a] = st;
    }
    CUresult r = encoder()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 1 + nouter, ptr, dims, strides, boxd, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS && std::getenv("TRI_ATTN_DEBUG")) {
        std::fprintf(stderr, "tri_attn: tensor-map encode failed (CUresult %d): rank %d ptr %p dims", static_cast<int>(r),
                     1 + nouter, ptr);
        for (int a = 0; a <= nouter; ++a) std::fprintf(stderr, " %llu", static_cast<unsigned long long>(dims[a]));
        std::fprintf(stderr, " strides");
        for (int a = 0; a < nouter; ++a) std::fprintf(stderr, " %llu", static_cast<unsigned long long>(strides[a]));
        std::fprintf(stderr, "\n");
    }
    return r == CUDA_SUCCESS;
}

// Pair tensor [B,N,N,H,d] map: coordinates (c, h, j, i, b), box d x 1 x 128 x 1 x 1.
// R: the rows i the map covers (N, or a row shard); the j extent is always N
bool map_pair(CUtensorMap* m, const tri_attn_tensor5& t, int B, int R, int N, int H, int d) {
    const uint64_t size[4] = {static_cast<uint64_t>(H), static_cast<uint64_t>(N), static_cast<uint64_t>(R),
                              static_cast<uint64_t>(B)};
    const uint64_t st[4] = {static_cast<uint64_t>(t.stride[3]) * 2, static_cast<uint64_t>(t.stride[2]) * 2,
                            static_cast<uint64_t>(t.stride[1]) * 2, static_cast<uint64_t>(t.stride[0]) * 2};
    const uint32_t box[4] = {1, 128, 1, 1};
    return encode_map(m, t.ptr, d, d, size, st, box, 4, d == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
}

// Bias [B,H,N,N] map: coordinates (k, j, h, b), box 64 keys x 128 rows, 128-byte swizzle.
bool map_bias(CUtensorMap* m, const tri_attn_tensor4& t, int B, int N, int H) {
    const uint64_t size[3] = {static_cast<uint64_t>(N), static_cast<uint64_t>(H), static_cast<uint64_t>(B)};
    const uint64_t st[3] = {static_cast<uint64_t>(t.stride[2]) * 2, static_cast<uint64_t>(t.stride[1]) * 2,
                            static_cast<uint64_t>(t.stride[0]) * 2};
    const uint32_t box[3] = {128, 1, 1};
    return encode_map(m, t.ptr, N, 64, size, st, box, 3, CU_TENSOR_MAP_SWIZZLE_128B);
}

float eff_scale(float s, int d) { return s == 0.f ? 1.0f / std::sqrt(static_cast<float>(d)) : s; }

// ---------------------------------------------------------------------------
// triangle multiplicative contraction
// ---------------------------------------------------------------------------
// 4-D map over a BF16 [B, C, rows, cols] tensor: inner = cols (box 64, 128-byte
// swizzle), then rows (box box_rows), c and b (box 1).
bool map_bcrc(CUtensorMap* m, const tri_attn_tensor4& t, int B, int C, int N, uint32_t box_rows) {
    const uint64_t size[3] = {static_cast<uint64_t>(N), static_cast<uint64_t>(C), static_cast<uint64_t>(B)};
    const uint64_t st[3] = {static_cast<uint64_t>(t.stride[2]) * 2, static_cast<uint64_t>(t.stride[1]) * 2,
                            static_cast<uint64_t>(t.stride[0]) * 2};
    const uint32_t box[3] = {box_rows, 1, 1};
    return encode_map(m, t.ptr, N, 64, size, st, box, 3, CU_TENSOR_MAP_SWIZZLE_128B);
}

// 2-D map over a BF16 [rows, 128] matrix with the given row stride: box 64 x box_rows,
// 128-byte swizzle
bool map_rows128(CUtensorMap* m, const void* ptr, int64_t rows, int64_t row_stride, uint32_t box_rows) {
    const uint64_t size[1] = {static_cast<uint64_t>(rows)};
    const uint64_t st[1] = {static_cast<uint64_t>(row_stride) * 2};
    const uint32_t box[1] = {box_rows};
    return encode_map(m, const_cast<void*>(ptr), 128, 64, size, st, box, 1, CU_TENSOR_MAP_SWIZZLE_128B);
}

tri_attn_status check_mul_sizes(int B, int C, int N) {
    if (B < 1 || C < 1 || N < 1 || static_cast<int64_t>(B) * C > 65535) return TRI_ATTN_ERR_SHAPE;
    if (N > 16384) return TRI_ATTN_ERR_UNSUPPORTED;
    return TRI_ATTN_OK;
}

// out[z][m][n] = sum_k A(m, k) B(n, k); an operand flagged MN is stored with m (n)
// contiguous, otherwise with k contiguous
template <bool A_MN, bool B_MN>
tri_attn_status tri_mul_gemm(const tri_attn_tensor4& A, const tri_attn_tensor4& Bt, const tri_attn_tensor4& out, int Bn,
                             int C, int N, cudaStream_t s) {
    using L = tri::TriMulLayout;
    CUtensorMap ma, mb;
    if (!map_bcrc(&ma, A, Bn, C, N, A_MN ? 64 : L::BM) || !map_bcrc(&mb, Bt, Bn, C, N, B_MN ? 64 : L::BN))
        return TRI_ATTN_ERR_STRIDE;
    tri::TriMulGemmParams p{};
    p.N = N;
    p.C = C;
    p.Z = Bn * C;
    p.out = static_cast<__nv_bfloat16*>(out.ptr);
    for (int x = 0; x < 4; ++x) p.os[x] = out.stride[x];
    p.wait_limit_ns = g_wait_limit_ns.load();
    // persistent grid: one CTA per SM (148 on B200) walking the output tiles
    const int64_t tiles = static_cast<int64_t>((N + L::BM - 1) / L::BM) * ((N + L::BN - 1) / L::BN) * Bn * C;
    const dim3 grid(static_cast<unsigned>(std::min<int64_t>(tiles, 148)));
    tri::tri_mul_gemm_kernel<A_MN, B_MN><<<grid, L::THREADS, L::SMEM, s>>>(ma, mb, p);
    return cudaGetLastError() == cudaSuccess ? TRI_ATTN_OK : TRI_ATTN_ERR_CUDA;
}

}  // namespace

// ===========================================================================
// backward launch (declared in bwd.cuh)
// ===========================================================================
namespace tri {

bool bwd_set_attributes() {
    bool ok = true;
    ok &= cudaFuncSetAttribute(tri_attn_bwd_main_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               MainLayout<32>::SMEM) == cudaSuccess;
    ok &= cudaFuncSetAttribute(tri_attn_bwd_main_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               MainLayout<64>::SMEM) == cudaSuccess;
    ok &= cudaFuncSetAttribute(tri_attn_bwd_dbias_kernel<32, TRI_DBIAS_FMA_PAIRS>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, DbLayout<32>::SMEM) == cudaSuccess;
    ok &= cudaFuncSetAttribute(tri_attn_bwd_dbias_kernel<64, TRI_DBIAS_FMA_PAIRS>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, DbLayout<64>::SMEM) == cudaSuccess;
    return ok;
}

tri_attn_status bwd_launch(const tri_attn_bwd_args* a, int R, float* parts, const BwdWorkspace& ws, float scale,
                           uint64_t wait_ns, cudaStream_t stream, void* const* markers) {
    auto mark = [&](int m) {
        if (markers && markers[m]) cudaEventRecord(static_cast<cudaEvent_t>(markers[m]), stream);
    };
    const tri_attn_fwd_args& f = a->f;
    const int B = f.B, N = f.N, H = f.H, d = f.d;
    CUtensorMap mq, mk, mv, mdo;
    if (!map_pair(&mq, f.q, B, R, N, H, d) || !map_pair(&mk, f.k, B, R, N, H, d) ||
        !map_pair(&mv, f.v, B, R, N, H, d) || !map_pair(&mdo, a->dout, B, R, N, H, d))
        return TRI_ATTN_ERR_STRIDE;
    uint8_t* wsb = static_cast<uint8_t*>(a->workspace);
    BwdParams p{};
    p.B = B; p.N = N; p.H = H;
    p.R = R;
    p.nt = (N + 127) / 128;
    p.Np = ws.Np;
    p.dq_tmem = (256 + 2 * d + p.nt * d <= 512) ? 1 : 0;
    p.scale = scale;
    float* Dv = reinterpret_cast<float*>(wsb + ws.off_D);
    float* Lv = reinterpret_cast<float*>(wsb + ws.off_L);
    float* Mv = reinterpret_cast<float*>(wsb + ws.off_M);
    int* Fv = reinterpret_cast<int*>(wsb + ws.off_F);
    p.Dv = Dv; p.Lv = Lv; p.Mv = Mv; p.Fv = Fv;
    p.bias = static_cast<const __nv_bfloat16*>(f.bias.ptr);
    p.bs0 = f.bias.stride[0]; p.bs1 = f.bias.stride[1]; p.bs2 = f.bias.stride[2];
    p.bias_tiles = reinterpret_cast<const uint4*>(wsb + ws.off_BT);
    p.dq_slots = reinterpret_cast<float*>(wsb + ws.off_dq);
    p.part = parts ? parts : reinterpret_cast<float*>(wsb + ws.off_part);
    p.part_out = parts ? 1 : 0;
    p.chunks = ws.chunks;
    p.dq = static_cast<__nv_bfloat16*>(a->dq.ptr);
    p.dk = static_cast<__nv_bfloat16*>(a->dk.ptr);
    p.dv = static_cast<__nv_bfloat16*>(a->dv.ptr);
    p.dbias = static_cast<__nv_bfloat16*>(a->dbias.ptr);
    for (int x = 0; x < 5; ++x) { p.dqs[x] = a->dq.stride[x]; p.dks[x] = a->dk.stride[x]; p.dvs[x] = a->dv.stride[x]; }
    for (int x = 0; x < 4; ++x) p.dbs[x] = a->dbias.stride[x];
    p.wait_limit_ns = wait_ns;

    const int64_t rows = static_cast<int64_t>(B) * H * N * N;
    const int64_t prep_items = static_cast<int64_t>(B) * H * R * ws.Np + static_cast<int64_t>(B) * R * ws.Np +
                               static_cast<int64_t>(B) * R * 32;
    const unsigned prep_grid = static_cast<unsigned>(std::min<int64_t>((prep_items + 255) / 256, 148 * 16));
    const auto& sm = f.mask.stride;
    const int use_resid = (a->flags & TRI_ATTN_BWD_NO_RESIDUAL) ? 0 : 1;
    const unsigned db_grid = static_cast<unsigned>(B) * H * p.nt * p.nt * ws.chunks;
    const __nv_bfloat16* bias = static_cast<const __nv_bfloat16*>(f.bias.ptr);
    const auto& so = f.o.stride; const auto& sr = f.resid.stride; const auto& sd = a->dout.stride;
    // pre-pass 1b: the bias in the main kernel's read order
    auto launch_bias_tiles = [&]() {
        const int64_t chunks16 = static_cast<int64_t>(B) * H * ws.Np * (ws.Np / 8);
        const unsigned g = static_cast<unsigned>(std::min<int64_t>((chunks16 + 255) / 256, 148 * 16));
        tri_attn_bwd_bias_tiles_kernel<<<g, 256, 0, stream>>>(bias, f.bias.stride[0], f.bias.stride[1],
                                                              f.bias.stride[2], B, H, N, p.nt,
                                                              reinterpret_cast<uint4*>(wsb + ws.off_BT));
    };
    mark(0);
    if (d == 32) {
        tri_attn_bwd_prep_kernel<32><<<prep_grid, 256, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(a->dout.ptr), sd[0], sd[1], sd[2], sd[3],
            static_cast<const __nv_bfloat16*>(f.o.ptr), so[0], so[1], so[2], so[3],
            static_cast<const __nv_bfloat16*>(f.resid.ptr), sr[0], sr[1], sr[2], sr[3], use_resid, f.lse, f.mask.ptr,
            sm[0], sm[1], sm[2], Dv, Lv, Mv, Fv, B, N, R, H, ws.Np, p.nt);
        launch_bias_tiles();
        mark(1);
        tri_attn_bwd_main_kernel<32><<<ws.grid_main, MainLayout<32>::THREADS, MainLayout<32>::SMEM, stream>>>(mq, mk, mv, mdo, p);
        mark(2);
        tri_attn_bwd_dbias_kernel<32, TRI_DBIAS_FMA_PAIRS><<<db_grid, DbLayout<32>::THREADS, DbLayout<32>::SMEM, stream>>>(
            mq, mk, mv, mdo, bias, f.bias.stride[0], f.bias.stride[1], f.bias.stride[2], p);
    } else {
        tri_attn_bwd_prep_kernel<64><<<prep_grid, 256, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(a->dout.ptr), sd[0], sd[1], sd[2], sd[3],
            static_cast<const __nv_bfloat16*>(f.o.ptr), so[0], so[1], so[2], so[3],
            static_cast<const __nv_bfloat16*>(f.resid.ptr), sr[0], sr[1], sr[2], sr[3], use_resid, f.lse, f.mask.ptr,
            sm[0], sm[1], sm[2], Dv, Lv, Mv, Fv, B, N, R, H, ws.Np, p.nt);
        launch_bias_tiles();
        mark(1);
        tri_attn_bwd_main_kernel<64><<<ws.grid_main, MainLayout<64>::THREADS, MainLayout<64>::SMEM, stream>>>(mq, mk, mv, mdo, p);
        mark(2);
        tri_attn_bwd_dbias_kernel<64, TRI_DBIAS_FMA_PAIRS><<<db_grid, DbLayout<64>::THREADS, DbLayout<64>::SMEM, stream>>>(
            mq, mk, mv, mdo, bias, f.bias.stride[0], f.bias.stride[1], f.bias.stride[2], p);
    }
    if (ws.chunks > 1 && !parts) {
        const unsigned rg = static_cast<unsigned>(std::min<int64_t>((rows + 255) / 256, 148 * 16));
        tri_attn_bwd_dbias_reduce_kernel<<<rg, 256, 0, stream>>>(p.part, ws.chunks, B, H, N, p.dbias,
                                                                  a->dbias.stride[0], a->dbias.stride[1],
                                                                  a->dbias.stride[2]);
    }
    mark(3);
    return cudaGetLastError() == cudaSuccess ? TRI_ATTN_OK : TRI_ATTN_ERR_CUDA;
}

}  // namespace tri

// ===========================================================================
// exported entry points
// ===========================================================================
extern "C" {

int tri_attn_abi_version(void) { return TRI_ATTN_ABI_VERSION; }

#ifdef TRI_TRACE
// instrumentation builds only: where the kernels write their phase cycles
int tri_attn_trace_set(void* p) { return cudaMemcpyToSymbol(tri::g_trace, &p, sizeof(p)) == cudaSuccess ? 0 : 1; }
#endif

const char* tri_attn_strerror(tri_attn_status s) {
    switch (s) {
        case TRI_ATTN_OK: return "ok";
        case TRI_ATTN_ERR_NULL: return "a required pointer is NULL";
        case TRI_ATTN_ERR_SHAPE: return "B, N or H out of range";
        case TRI_ATTN_ERR_STRIDE: return "innermost stride must be 1 and other strides non-negative multiples of 8 elements";
        case TRI_ATTN_ERR_ALIGN: return "a data pointer is not 16-byte aligned";
        case TRI_ATTN_ERR_DTYPE: return "wrong element type";
        case TRI_ATTN_ERR_UNSUPPORTED: return "unsupported size (d must be 32 or 64, N <= 4096)";
        case TRI_ATTN_ERR_WORKSPACE: return "workspace missing or too small";
        case TRI_ATTN_ERR_ARCH: return "current device is not compute capability 10.0 (sm_100)";
        case TRI_ATTN_ERR_CUDA: return "a CUDA call failed";
        case TRI_ATTN_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel expired";
        case TRI_ATTN_ERR_SCRATCH_LIMIT: return "sizes need more scratch than the 64 MiB static scratch area holds";
    }
    return "unknown status";
}

void tri_attn_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns ? ns : 1); }

}  // extern "C"

namespace {

// the forward over rows 0 .. R-1 of the given tensors (R = N: the whole problem)
tri_attn_status fwd_impl(const tri_attn_fwd_args* a, int R, tri_attn_stream_t stream) {
    tri_attn_status st = check_fwd_args(a);
    if (st) return st;
    if (R < 1 || R > a->N) return TRI_ATTN_ERR_SHAPE;
    if ((st = ensure_device())) return st;
    const int B = a->B, N = a->N, H = a->H, d = a->d;
    CUtensorMap mq, mk, mv, mb;
    if (!map_pair(&mq, a->q, B, R, N, H, d) || !map_pair(&mk, a->k, B, R, N, H, d) ||
        !map_pair(&mv, a->v, B, R, N, H, d) || !map_bias(&mb, a->bias, B, N, H))
        return TRI_ATTN_ERR_STRIDE;
    tri::FwdParams p{};
    p.B = B; p.N = N; p.H = H;
    p.R = R;
    p.nt = (N + 127) / 128;
    p.npairs = (R + 1) / 2;
    p.scale = eff_scale(a->scale, d);
    p.mask = a->mask.ptr;
    p.ms0 = a->mask.stride[0]; p.ms1 = a->mask.stride[1]; p.ms2 = a->mask.stride[2];
    p.o = static_cast<__nv_bfloat16*>(a->o.ptr);
    p.r = static_cast<__nv_bfloat16*>(a->resid.ptr);
    for (int x = 0; x < 5; ++x) { p.os[x] = a->o.stride[x]; p.rs[x] = a->resid.stride[x]; }
    p.lse = a->lse;
    p.wait_limit_ns = g_wait_limit_ns.load();
    // persistent grid: one CTA per SM (148 on B200), each walking work items
    const int64_t items = static_cast<int64_t>(B) * p.npairs * H * p.nt;
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(items, 148));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (d == 32)
        tri::tri_attn_fwd_kernel<32><<<grid, 384, tri::FwdLayout<32>::SMEM, s>>>(mq, mk, mv, mb, p);
    else
        tri::tri_attn_fwd_kernel<64><<<grid, 384, tri::FwdLayout<64>::SMEM, s>>>(mq, mk, mv, mb, p);
    return cudaGetLastError() == cudaSuccess ? TRI_ATTN_OK : TRI_ATTN_ERR_CUDA;
}

// host-side argument checks of the backward over rows 0 .. R-1 (everything but the
// workspace); no CUDA call
tri_attn_status bwd_check_args(const tri_attn_bwd_args* a, int R, const float* parts) {
    if (!a) return TRI_ATTN_ERR_NULL;
    tri_attn_status st = check_fwd_args(&a->f);
    if (st) return st;
    if (R < 1 || R > a->f.N) return TRI_ATTN_ERR_SHAPE;
    const tri_attn_tensor5* t5[] = {&a->dout, &a->dq, &a->dk, &a->dv};
    for (const auto* t : t5)
        if ((st = check_t5(*t))) return st;
    if (parts) {
        if (!aligned16(parts)) return TRI_ATTN_ERR_ALIGN;
    } else if ((st = check_t4(a->dbias))) {
        return st;
    }
    return TRI_ATTN_OK;
}

// the backward over rows 0 .. R-1; parts == nullptr: dBias (BF16) for those rows
// as the whole sum over i; otherwise dBias leaves as FP32 partial sums in parts
tri_attn_status bwd_impl(const tri_attn_bwd_args* a, int R, float* parts, tri_attn_stream_t stream,
                         void* const* markers) {
    tri_attn_status st = bwd_check_args(a, R, parts);
    if (st) return st;
    const int B = a->f.B, N = a->f.N, H = a->f.H, d = a->f.d;
    const tri::BwdWorkspace ws = tri::bwd_workspace_layout(B, R, N, H, d);
    const size_t need = parts ? ws.off_part : ws.total;  // shard calls keep no partials of their own
    if (!a->workspace || a->workspace_bytes < need) return TRI_ATTN_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(a->workspace) & 255u) return TRI_ATTN_ERR_ALIGN;
    if ((st = ensure_device())) return st;
    return tri::bwd_launch(a, R, parts, ws, eff_scale(a->f.scale, d), g_wait_limit_ns.load(),
                           reinterpret_cast<cudaStream_t>(stream), markers);
}

}  // namespace

// argument checks of tri_attn_bwd, shared with the static-scratch entry point
// (csrc/bwd_static.cu) so that it rejects bad arguments before any CUDA call
namespace tri {
tri_attn_status bwd_validate(const tri_attn_bwd_args* a) { return bwd_check_args(a, a ? a->f.N : 0, nullptr); }
}  // namespace tri

extern "C" {

tri_attn_status tri_attn_fwd(const tri_attn_fwd_args* a, tri_attn_stream_t stream) {
    return fwd_impl(a, a ? a->N : 0, stream);
}

tri_attn_status tri_attn_fwd_rows(const tri_attn_fwd_args* a, int rows, tri_attn_stream_t stream) {
    return fwd_impl(a, rows, stream);
}

size_t tri_attn_bwd_workspace_bytes(int B, int N, int H, int d) {
    if (check_sizes(B, N, H, d)) return 0;
    return tri::bwd_workspace_layout(B, N, N, H, d).total;
}

size_t tri_attn_bwd_rows_workspace_bytes(int B, int rows, int N, int H, int d) {
    if (check_sizes(B, N, H, d) || rows < 1 || rows > N) return 0;
    return tri::bwd_workspace_layout(B, rows, N, H, d).off_part;
}

int tri_attn_bwd_rows_dbias_parts(int B, int rows, int N, int H, int d) {
    if (check_sizes(B, N, H, d) || rows < 1 || rows > N) return 0;
    return tri::bwd_workspace_layout(B, rows, N, H, d).chunks;
}

tri_attn_status tri_attn_bwd(const tri_attn_bwd_args* a, tri_attn_stream_t stream) {
    return bwd_impl(a, a ? a->f.N : 0, nullptr, stream, nullptr);
}

tri_attn_status tri_attn_bwd_marked(const tri_attn_bwd_args* a, tri_attn_stream_t stream, void* const* markers) {
    return bwd_impl(a, a ? a->f.N : 0, nullptr, stream, markers);
}

tri_attn_status tri_attn_bwd_rows(const tri_attn_bwd_args* a, int rows, float* dbias_parts,
                                  tri_attn_stream_t stream) {
    if (!dbias_parts) return TRI_ATTN_ERR_NULL;
    return bwd_impl(a, rows, dbias_parts, stream, nullptr);
}

tri_attn_status tri_attn_dbias_sum(const float* parts, int nparts, int B, int H, int N, tri_attn_tensor4 dbias,
                                   tri_attn_stream_t stream) {
    if (!parts) return TRI_ATTN_ERR_NULL;
    if (!aligned16(parts)) return TRI_ATTN_ERR_ALIGN;
    if (nparts < 1 || B < 1 || H < 1 || N < 1 || N > kMaxN) return TRI_ATTN_ERR_SHAPE;
    tri_attn_status st = check_t4(dbias);
    if (st) return st;
    if ((st = ensure_device())) return st;
    const int64_t total = static_cast<int64_t>(B) * H * N * N;
    const unsigned rg = static_cast<unsigned>(std::min<int64_t>((total + 255) / 256, 148 * 16));
    tri::tri_attn_bwd_dbias_reduce_kernel<<<rg, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        parts, nparts, B, H, N, static_cast<__nv_bfloat16*>(dbias.ptr), dbias.stride[0], dbias.stride[1],
        dbias.stride[2]);
    return cudaGetLastError() == cudaSuccess ? TRI_ATTN_OK : TRI_ATTN_ERR_CUDA;
}

tri_attn_status tri_mul_fwd(const tri_mul_fwd_args* a, tri_attn_stream_t stream) {
    if (!a) return TRI_ATTN_ERR_NULL;
    tri_attn_status st = check_mul_sizes(a->B, a->C, a->N);
    if (st) return st;
    if ((st = check_t4(a->a)) || (st = check_t4(a->b)) || (st = check_t4(a->x))) return st;
    if (a->flags & ~TRI_MUL_INCOMING) return TRI_ATTN_ERR_UNSUPPORTED;
    if ((st = ensure_device())) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (a->flags & TRI_MUL_INCOMING)  // x[i,j] = sum_k a[k,i] b[k,j]: both operands i/j-contiguous
        return tri_mul_gemm<true, true>(a->a, a->b, a->x, a->B, a->C, a->N, s);
    return tri_mul_gemm<false, false>(a->a, a->b, a->x, a->B, a->C, a->N, s);  // sum_k a[i,k] b[j,k]
}

tri_attn_status tri_mul_bwd(const tri_mul_bwd_args* a, tri_attn_stream_t stream) {
    if (!a) return TRI_ATTN_ERR_NULL;
    const tri_mul_fwd_args& f = a->f;
    tri_attn_status st = check_mul_sizes(f.B, f.C, f.N);
    if (st) return st;
    if ((st = check_t4(f.a)) || (st = check_t4(f.b)) || (st = check_t4(a->dx)) || (st = check_t4(a->da)) ||
        (st = check_t4(a->db)))
        return st;
    if (f.flags & ~TRI_MUL_INCOMING) return TRI_ATTN_ERR_UNSUPPORTED;
    if ((st = ensure_device())) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (f.flags & TRI_MUL_INCOMING) {
        // da[k,i] = sum_j b[k,j] dx[i,j];  db[k,j] = sum_i a[k,i] dx[i,j]
        if ((st = tri_mul_gemm<false, false>(f.b, a->dx, a->da, f.B, f.C, f.N, s))) return st;
        return tri_mul_gemm<false, true>(f.a, a->dx, a->db, f.B, f.C, f.N, s);
    }
    // da[i,k] = sum_j dx[i,j] b[j,k];  db[j,k] = sum_i dx[i,j] a[i,k]
    if ((st = tri_mul_gemm<false, true>(a->dx, f.b, a->da, f.B, f.C, f.N, s))) return st;
    return tri_mul_gemm<true, true>(a->dx, f.a, a->db, f.B, f.C, f.N, s);
}

tri_attn_status tri_gate_fwd(const tri_gate_fwd_args* a, tri_attn_stream_t stream) {
    if (!a) return TRI_ATTN_ERR_NULL;
    if (!a->z || !a->o || !a->wg || !a->wo || !a->y) return TRI_ATTN_ERR_NULL;
    if (a->R < 1) return TRI_ATTN_ERR_SHAPE;
    for (int64_t st : {a->z_stride, a->o_stride, a->y_stride})
        if (st < 128 || st % 8) return TRI_ATTN_ERR_STRIDE;
    for (const void* ptr : {a->z, a->o, a->wg, a->wo, static_cast<const void*>(a->y)})
        if (!aligned16(ptr)) return TRI_ATTN_ERR_ALIGN;
    tri_attn_status st = ensure_device();
    if (st) return st;
    using L = tri::TriGateLayout;
    CUtensorMap mz, mo, mwg, mwo, my;
    if (!map_rows128(&mz, a->z, a->R, a->z_stride, L::BM) || !map_rows128(&mo, a->o, a->R, a->o_stride, L::BM) ||
        !map_rows128(&mwg, a->wg, 128, 128, 128) || !map_rows128(&mwo, a->wo, 128, 128, 128) ||
        !map_rows128(&my, a->y, a->R, a->y_stride, 32))
        return TRI_ATTN_ERR_STRIDE;
    tri::TriGateParams p{};
    p.R = a->R;
    p.wait_limit_ns = g_wait_limit_ns.load();
    const int64_t tiles = (static_cast<int64_t>(a->R) + L::BM - 1) / L::BM;
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(tiles, 148));  // persistent, one CTA per SM
    tri::tri_gate_fwd_kernel<<<grid, L::THREADS, L::SMEM, reinterpret_cast<cudaStream_t>(stream)>>>(mz, mo, mwg, mwo,
                                                                                                   my, p);
    return cudaGetLastError() == cudaSuccess ? TRI_ATTN_OK : TRI_ATTN_ERR_CUDA;
}

namespace {
constexpr int kGateMaxCtas = 148;  // persistent grid: one CTA per SM
int64_t gate_ctas(int R) {
    return std::min<int64_t>((static_cast<int64_t>(R) + tri::TriGateBwdLayout::BM - 1) / tri::TriGateBwdLayout::BM,
                             kGateMaxCtas);
}
}  // namespace

size_t tri_gate_bwd_workspace_bytes(int R) {
    if (R < 1) return 0;
    return static_cast<size_t>(gate_ctas(R)) * tri::TriGateBwdLayout::PARTIAL_FLOATS * sizeof(float);
}

tri_attn_status tri_gate_bwd(const tri_gate_bwd_args* a, tri_attn_stream_t stream) {
    if (!a) return TRI_ATTN_ERR_NULL;
    const tri_gate_fwd_args& f = a->f;
    if (!f.z || !f.o || !f.wg || !f.wo || !a->dy || !a->dz || !a->d_o || !a->dwg || !a->dwo) return TRI_ATTN_ERR_NULL;
    if (f.R < 1) return TRI_ATTN_ERR_SHAPE;
    for (int64_t st : {f.z_stride, f.o_stride, a->dy_stride, a->dz_stride, a->do_stride})
        if (st < 128 || st % 8) return TRI_ATTN_ERR_STRIDE;
    for (const void* ptr : {f.z, f.o, f.wg, f.wo, a->dy, static_cast<const void*>(a->dz),
                            static_cast<const void*>(a->d_o), static_cast<const void*>(a->dwg),
                            static_cast<const void*>(a->dwo)})
        if (!aligned16(ptr)) return TRI_ATTN_ERR_ALIGN;
    if (!a->workspace || !aligned16(a->workspace) || a->workspace_bytes < tri_gate_bwd_workspace_bytes(f.R))
        return TRI_ATTN_ERR_WORKSPACE;
    tri_attn_status st = ensure_device();
    if (st) return st;
    using L = tri::TriGateBwdLayout;
    CUtensorMap mz, mdy, mwg, mwo, mdz, mdo;
    if (!map_rows128(&mz, f.z, f.R, f.z_stride, L::BM) || !map_rows128(&mdy, a->dy, f.R, a->dy_stride, L::BM) ||
        !map_rows128(&mwg, f.wg, 128, 128, 128) || !map_rows128(&mwo, f.wo, 128, 128, 128) ||
        !map_rows128(&mdz, a->dz, f.R, a->dz_stride, 32) || !map_rows128(&mdo, a->d_o, f.R, a->do_stride, 32))
        return TRI_ATTN_ERR_STRIDE;
    tri::TriGateBwdParams p{};
    p.R = f.R;
    p.o = static_cast<const __nv_bfloat16*>(f.o);
    p.os = f.o_stride;
    p.partial = static_cast<float*>(a->workspace);
    p.wait_limit_ns = g_wait_limit_ns.load();
    const int grid = static_cast<int>(gate_ctas(f.R));
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    tri::tri_gate_bwd_kernel<<<grid, L::THREADS, L::SMEM, s>>>(mz, mdy, mwg, mwo, mdz, mdo, p);
    constexpr int n4 = L::PARTIAL_FLOATS / 4, per_block = tri::kWsumThreads / 8;
    tri::tri_gate_wsum_kernel<<<(n4 + per_block - 1) / per_block, tri::kWsumThreads, 0, s>>>(p.partial, grid, a->dwg,
                                                                                             a->dwo);
    return cudaGetLastError() == cudaSuccess ? TRI_ATTN_OK : TRI_ATTN_ERR_CUDA;
}

tri_attn_status tri_attn_device_error(int clear, uint32_t* word) {
    uint32_t w = 0;
    if (cudaMemcpyFromSymbol(&w, tri::g_error_word, sizeof w) != cudaSuccess) {
        cudaGetLastError();
        return TRI_ATTN_ERR_CUDA;
    }
    if (word) *word = w;
    if (clear) {
        const uint32_t z = 0;
        if (cudaMemcpyToSymbol(tri::g_error_word, &z, sizeof z) != cudaSuccess) {
            cudaGetLastError();
            return TRI_ATTN_ERR_CUDA;
        }
    }
    return w ? TRI_ATTN_ERR_DEVICE_TIMEOUT : TRI_ATTN_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// self-test of the bounded-wait path: a barrier that nothing ever completes
// ---------------------------------------------------------------------------
namespace tri {
__global__ void selftest_expire_kernel(uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(smem_addr(&bar), 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const WaitCtx wc{limit_ns, KERNEL_SELFTEST, &abort_flag};
        (void)mbar_wait(smem_addr(&bar), 0, wc, 1);
    }
    __syncthreads();
}
}  // namespace tri

extern "C" tri_attn_status tri_attn_selftest_expire_wait(tri_attn_stream_t stream) {
    tri_attn_status st = ensure_device();
    if (st) return st;
    tri::selftest_expire_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(g_wait_limit_ns.load());
    return cudaGetLastError() == cudaSuccess ? TRI_ATTN_OK : TRI_ATTN_ERR_CUDA;
}
