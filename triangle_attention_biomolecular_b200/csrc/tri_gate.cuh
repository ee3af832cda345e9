// tri_gate.cuh -- the gated output projection around triangle attention, sm_100a.
//
// The pages describe the attention itself; the steps on either side of it are
// the model's.  Read the AlphaFold way, the attention output o (heads
// concatenated) leaves through a sigmoid gate computed from the pair
// representation z and a linear output projection, position by position:
//   g = sigmoid(z Wg),   y = (g * o) Wo        (cz = co = 128, no biases)
// Per pair position this is 2 x 128 x 128 multiply-adds against 768 bytes of
// traffic (z, o in, y out), so the step is HBM-bound; the kernel keeps both
// weight matrices resident and streams 128-position tiles through two
// tcgen05 contractions with the gate in between.
//
// B200 mapping (one persistent CTA per SM, 192 threads):
//  * warp 4 TMA producer: Wg, Wo once (MN-major B operands, 32 KB each), then
//    per tile z (K-major A operand) and o (read by the epilogue) through a
//    two-stage ring, 64 KB per stage;
//  * warp 5 MMA issuer: G = z Wg into one of two 128-column TMEM accumulators,
//    later Y = a Wo into one of two more;
//  * warps 0-3 (one row per thread): sigmoid of G (exp2 and reciprocal on the
//    MUFU unit), a = g * o, BF16 a written to shared memory in the 128-byte-
//    swizzled K-major layout the second MMA reads; then Y -> BF16 -> global,
//    one tile behind, so the tensor cores, the MUFU unit and the stores of
//    neighbouring tiles overlap.
#pragma once

#include "sm100.cuh"

namespace tri {

constexpr uint32_t KERNEL_TRIGATE = 5u << 16;   // device error word: kernel field of this kernel's waits

// 2-D tiled TMA load, completion counted on an mbarrier (no multicast).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* m, uint32_t bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

struct TriGateParams {
    int R;                  // pair positions
    __nv_bfloat16* y;       // [R, 128]
    int64_t ys;             // row stride (elements)
    uint64_t wait_limit_ns;
};

struct TriGateLayout {
    static constexpr int C = 128, BM = 128;
    static constexpr int W_TILE = C * C * 2;          // 32 KB
    static constexpr int X_TILE = BM * C * 2;         // 32 KB (two 64-column halves of 16 KB)
    static constexpr int NS = 2;
    static constexpr int OFF_WG = 0, OFF_WO = W_TILE;
    static constexpr int OFF_STAGE = 2 * W_TILE;      // [NS][z, o]
    static constexpr int STAGE = 2 * X_TILE;
    static constexpr int OFF_A = OFF_STAGE + NS * STAGE;  // gated a, K-major, two halves
    static constexpr int OFF_BAR = OFF_A + X_TILE;
    static constexpr int B_W = 0, B_FULL = 1, B_XEMPTY = 1 + NS, B_GFULL = 1 + 2 * NS, B_GFREE = B_GFULL + 2,
                         B_AFULL = B_GFREE + 2, B_AFREE = B_AFULL + 1, B_YFULL = B_AFREE + 1, B_YFREE = B_YFULL + 2,
                         B_DRAIN = B_YFREE + 2, NBAR = B_DRAIN + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + slack for 1 KB alignment
    static constexpr int THREADS = 192;
    static_assert(SMEM <= 232448, "shared memory budget");
};

__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__global__ void __launch_bounds__(192, 1)
    tri_gate_fwd_kernel(const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_o,
                        const __grid_constant__ CUtensorMap tm_wg, const __grid_constant__ CUtensorMap tm_wo,
                        const TriGateParams p) {
    using L = TriGateLayout;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sb - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto BAR = [&](int idx) -> uint32_t { return sb + L::OFF_BAR + idx * 8; };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
    const int tiles = (p.R + L::BM - 1) / L::BM;

    if (threadIdx.x == 0) {
        *abort_flag = device_error_pending() ? 1 : 0;
        mbar_init(BAR(L::B_W), 1);
        for (int s = 0; s < L::NS; ++s) {
            mbar_init(BAR(L::B_FULL + s), 1);
            mbar_init(BAR(L::B_XEMPTY + s), 1 + 4);  // MMA done with z + epilogue done with o
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(BAR(L::B_GFULL + x), 1);
            mbar_init(BAR(L::B_GFREE + x), 4);
            mbar_init(BAR(L::B_YFULL + x), 1);
            mbar_init(BAR(L::B_YFREE + x), 4);
        }
        mbar_init(BAR(L::B_AFULL), 4);
        mbar_init(BAR(L::B_AFREE), 1);
        mbar_init(BAR(L::B_DRAIN), 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(const_cast<uint32_t*>(tmem_slot)), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtx wc{p.wait_limit_ns, KERNEL_TRIGATE, abort_flag};
    const bool aborted_early = *abort_flag != 0;

    if (warp == 4) {
        // =========================== TMA producer ===========================
        const bool leader = elect_one();
        int armed[L::NS] = {};
        bool w_armed = false;
        if (!aborted_early) {
            if (leader) {
                tma_prefetch_map(&tm_z);
                tma_prefetch_map(&tm_o);
                mbar_arrive_expect_tx(BAR(L::B_W), 2 * L::W_TILE);
                // weights: [k rows][n cols] with n contiguous -> two 64-column chunks each
                tma_load_2d(sb + L::OFF_WG, &tm_wg, BAR(L::B_W), 0, 0);
                tma_load_2d(sb + L::OFF_WG + L::W_TILE / 2, &tm_wg, BAR(L::B_W), 64, 0);
                tma_load_2d(sb + L::OFF_WO, &tm_wo, BAR(L::B_W), 0, 0);
                tma_load_2d(sb + L::OFF_WO + L::W_TILE / 2, &tm_wo, BAR(L::B_W), 64, 0);
            }
            w_armed = true;
            int gt = 0;
            for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++gt) {
                const int s = gt % L::NS;
                if (gt >= L::NS && !mbar_wait_warp(BAR(L::B_XEMPTY + s), ((gt / L::NS) - 1) & 1, wc, 1)) break;
                if (leader) {
                    const uint32_t bar = BAR(L::B_FULL + s);
                    const uint32_t st = sb + L::OFF_STAGE + s * L::STAGE;
                    mbar_arrive_expect_tx(bar, L::STAGE);
                    tma_load_2d(st, &tm_z, bar, 0, t * L::BM);
                    tma_load_2d(st + L::X_TILE / 2, &tm_z, bar, 64, t * L::BM);
                    tma_load_2d(st + L::X_TILE, &tm_o, bar, 0, t * L::BM);
                    tma_load_2d(st + L::X_TILE + L::X_TILE / 2, &tm_o, bar, 64, t * L::BM);
                }
                armed[s]++;
            }
        }
        if (leader) {
            if (w_armed) drain_wait(BAR(L::B_W), 0, 100000000ull);
#pragma unroll
            for (int s = 0; s < L::NS; ++s)
                if (armed[s] > 0) drain_wait(BAR(L::B_FULL + s), (armed[s] - 1) & 1, 100000000ull);
        }
    } else if (warp == 5) {
        // =========================== MMA issuer =============================
        const bool leader = elect_one();
        if (!aborted_early) {
            constexpr uint32_t IDESC = idesc_bf16_f32(128, 128, false, true);
            // A (z, a): K-major, two 64-column halves 16 KB apart; B (Wg, Wo): MN-major,
            // 64-column chunks 16 KB apart (LBO), 8-k-row groups 1 KB apart (SBO)
            const uint64_t dz0 = smem_desc(sb + L::OFF_STAGE, 16, 1024, SWZ_128B);
            const uint64_t da0 = smem_desc(sb + L::OFF_A, 16, 1024, SWZ_128B);
            const uint64_t dwg = smem_desc(sb + L::OFF_WG, L::W_TILE / 2, 1024, SWZ_128B);
            const uint64_t dwo = smem_desc(sb + L::OFF_WO, L::W_TILE / 2, 1024, SWZ_128B);
            bool ok = mbar_wait_warp(BAR(L::B_W), 0, wc, 2);
            int lt = 0;
            for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++lt) {
                const int x = lt & 1, s = lt % L::NS;
                if (!mbar_wait_warp(BAR(L::B_FULL + s), (lt / L::NS) & 1, wc, 3)) { ok = false; break; }
                if (lt >= 2 && !mbar_wait_warp(BAR(L::B_GFREE + x), ((lt >> 1) - 1) & 1, wc, 4)) { ok = false; break; }
                tc_fence_after();
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss(tmem + x * 128, desc_add(dz0, s * L::STAGE + (kk >> 2) * (L::X_TILE / 2) + (kk & 3) * 32),
                               desc_add(dwg, kk * 2048), IDESC, kk > 0 ? 1u : 0u);
                    mma_commit(BAR(L::B_GFULL + x));
                    mma_commit(BAR(L::B_XEMPTY + s));
                }
                __syncwarp();
                // the gated a of this tile is in shared memory; Y[x] was read two tiles ago
                if (!mbar_wait_warp(BAR(L::B_AFULL), lt & 1, wc, 5)) { ok = false; break; }
                if (lt >= 2 && !mbar_wait_warp(BAR(L::B_YFREE + x), ((lt >> 1) - 1) & 1, wc, 6)) { ok = false; break; }
                tc_fence_after();
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss(tmem + 256 + x * 128, desc_add(da0, (kk >> 2) * (L::X_TILE / 2) + (kk & 3) * 32),
                               desc_add(dwo, kk * 2048), IDESC, kk > 0 ? 1u : 0u);
                    mma_commit(BAR(L::B_YFULL + x));
                    mma_commit(BAR(L::B_AFREE));
                }
                __syncwarp();
            }
            if (leader) {
                mma_commit(BAR(L::B_DRAIN));
                drain_wait(BAR(L::B_DRAIN), 0, 100000000ull);
            }
            __syncwarp();
        }
    } else {
        // =========================== gate + epilogue (warps 0-3) =============
        if (!aborted_early) {
            constexpr float LOG2E = 1.4426950408889634f;
            const int row = warp * 32 + lane;
            const uint32_t tl = tmem + (static_cast<uint32_t>(warp * 32) << 16);
            bool ok = true;
            // Y of tile lt (local index) -> BF16 -> global
            auto store_y = [&](int lt, int t) -> bool {
                const int x = lt & 1;
                if (!mbar_wait_warp(BAR(L::B_YFULL + x), (lt >> 1) & 1, wc, 9)) return false;
                tc_fence_after();
                const int r = t * L::BM + row;
                __nv_bfloat16* dst = p.y + static_cast<int64_t>(r) * p.ys;
#pragma unroll 1
                for (int c0 = 0; c0 < L::C; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld32(tl + 256 + x * 128 + c0, v);
                    tmem_wait_ld();
                    if (c0 == L::C - 32) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(BAR(L::B_YFREE + x));
                    }
                    if (r < p.R) {
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            uint4 q;
                            q.x = pack_bf16(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                            q.y = pack_bf16(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                            q.z = pack_bf16(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]));
                            q.w = pack_bf16(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7]));
                            *reinterpret_cast<uint4*>(dst + c0 + e) = q;
                        }
                    }
                }
                return true;
            };
            int lt = 0, prev_t = -1;
            for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
                const int x = lt & 1, s = lt % L::NS;
                if (!mbar_wait_warp(BAR(L::B_GFULL + x), (lt >> 1) & 1, wc, 7)) { ok = false; break; }
                tc_fence_after();
                // o of this tile arrived with z (the MMA has already waited for the stage)
                if (!mbar_wait_warp(BAR(L::B_FULL + s), (lt / L::NS) & 1, wc, 8)) { ok = false; break; }
                const uint32_t orow = sb + L::OFF_STAGE + s * L::STAGE + L::X_TILE + row * 128;
                const uint32_t arow = sb + L::OFF_A + row * 128;
#pragma unroll
                for (int h = 0; h < 2; ++h) {  // 64-column halves
                    uint32_t ga[32], gb[32];
                    tmem_ld32(tl + x * 128 + h * 64, ga);
                    tmem_ld32(tl + x * 128 + h * 64 + 32, gb);
                    tmem_wait_ld();
                    if (h == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(BAR(L::B_GFREE + x));
                    }
                    uint32_t aw[32];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {  // 16-byte chunks of 8 channels
                        const uint4 ob = lds128(orow + h * (L::X_TILE / 2) + ((c ^ (row & 7)) << 4));
                        const uint32_t ow[4] = {ob.x, ob.y, ob.z, ob.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int k = c * 8 + 2 * e;
                            // sigmoid(G) = 1 / (1 + 2^(-G log2 e))
                            const float l0 = __uint_as_float(k < 32 ? ga[k] : gb[k - 32]);
                            const float l1 = __uint_as_float(k + 1 < 32 ? ga[k + 1] : gb[k + 1 - 32]);
                            const float g0 = rcp_approx(1.f + ex2(-l0 * LOG2E));
                            const float g1 = rcp_approx(1.f + ex2(-l1 * LOG2E));
                            aw[c * 4 + e] = pack_bf16(g0 * bf16lo(ow[e]), g1 * bf16hi(ow[e]));
                        }
                    }
                    if (h == 0 && lt > 0 && !mbar_wait_warp(BAR(L::B_AFREE), (lt - 1) & 1, wc, 10)) {
                        ok = false;
                        break;
                    }
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        sts128(arow + h * (L::X_TILE / 2) + ((c ^ (row & 7)) << 4),
                               make_uint4(aw[4 * c], aw[4 * c + 1], aw[4 * c + 2], aw[4 * c + 3]));
                }
                if (!ok) break;
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(BAR(L::B_AFULL));
                    mbar_arrive(BAR(L::B_XEMPTY + s));
                }
                // the previous tile's output, while the tensor cores work on this one
                if (prev_t >= 0 && !(ok = store_y(lt - 1, prev_t))) break;
                prev_t = t;
            }
            if (ok && prev_t >= 0) store_y(lt - 1, prev_t);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ===========================================================================
// Backward.  For the upstream gradient dy (a = g * o as in the forward):
//   dA  = dy Wo^T                      do  = dA * g
//   dl  = dA * o * g * (1 - g)         (gradient of the gate logits z Wg)
//   dz  = dl Wg^T
//   dWo = sum_r a^T dy,   dWg = sum_r z^T dl
// One persistent CTA per SM walks 128-row tiles; five 128 x 128 x 128
// contractions per tile on the tensor cores:
//   MMA1  G   = z  Wg      A z  (K-major)      B Wg (MN-major)
//   MMA2  dA  = dy Wo^T    A dy (K-major)      B Wo (K-major: rows of Wo)
//   MMA5  dWo += a^T dy    A a  (MN-major)     B dy (MN-major)
//   MMA3  dz  = dl Wg^T    A dl (K-major)      B Wg (K-major: rows of Wg)
//   MMA4  dWg += z^T dl    A z  (MN-major)     B dl (MN-major)
// The same swizzled shared-memory tile serves as a K-major operand of one
// contraction and an MN-major operand of another, so nothing is transposed.
// TMEM: two 128-column slots P, Q for the per-tile products and 2 x 128 columns
// for the weight-gradient accumulators, which stay resident across all the
// CTA's tiles.  Even tiles put G and dz in P and dA in Q, odd tiles the other
// way round, so that the next tile's G is computed while this tile's dz is
// drained, and its dA while its G is being gated.
// Each CTA writes its FP32 dWg, dWo partial sums to a workspace; a second
// kernel adds the partials in CTA order (deterministic for a given R).
//
// Warps 0-7 (epilogue; warp w reads TMEM lanes 32 (w % 4) .. +31, i.e. rows,
// and channel half w / 4), warp 8 TMA producer, warp 9 MMA issuer.
// Per tile, each epilogue thread: A1 reads G, writes a = g * o (BF16) into
// the shared tile X and keeps g and s = o g (1 - g), both rounded to BF16, in
// registers (s is formed in FP32 from the FP32 g, so 1 - g keeps its relative
// accuracy for saturated gates); A2 reads dA, stores do = dA g, forms
// dl = dA s, and once MMA5 has finished with a overwrites X with dl; B reads
// dz and stores it.  o comes straight from global memory into
// registers, prefetched one tile ahead.
// ===========================================================================
struct TriGateBwdParams {
    int R;
    const __nv_bfloat16* o;
    int64_t os;
    __nv_bfloat16* dz;
    int64_t dzs;
    __nv_bfloat16* d_o;
    int64_t dos;
    float* partial;  // [gridDim.x][2][128][128]: dWg, dWo partial sums of each CTA
    uint64_t wait_limit_ns;
};

struct TriGateBwdLayout {
    static constexpr int C = 128, BM = 128;
    static constexpr int W_TILE = C * C * 2;   // 32 KB
    static constexpr int X_TILE = BM * C * 2;  // 32 KB, two 64-column halves of 16 KB
    static constexpr int HALF = X_TILE / 2;
    static constexpr int NS = 2;
    static constexpr int OFF_WG = 0, OFF_WO = W_TILE;
    static constexpr int OFF_STAGE = 2 * W_TILE;  // [NS][z, dy]
    static constexpr int STAGE = 2 * X_TILE;
    static constexpr int OFF_X = OFF_STAGE + NS * STAGE;  // a, then dl
    static constexpr int OFF_BAR = OFF_X + X_TILE;
    static constexpr int B_W = 0, B_FULL = 1, B_XEMPTY = 1 + NS, B_GFULL = 1 + 2 * NS, B_DAFULL = B_GFULL + 1,
                         B_A1DONE = B_DAFULL + 1, B_AFREE = B_A1DONE + 1, B_A2DONE = B_AFREE + 1,
                         B_DLFULL = B_A2DONE + 1, B_DZFULL = B_DLFULL + 1, B_BDONE = B_DZFULL + 1,
                         B_ACC = B_BDONE + 1, NBAR = B_ACC + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + slack for 1 KB alignment
    static constexpr int EPI_WARPS = 8, W_PRODUCER = 8, W_MMA = 9, THREADS = 320;
    static constexpr int PARTIAL_FLOATS = 2 * C * C;  // per CTA
    static_assert(SMEM <= 232448, "shared memory budget");
};

__device__ __forceinline__ uint4 ldg128_nc(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__global__ void __launch_bounds__(320, 1)
    tri_gate_bwd_kernel(const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_dy,
                        const __grid_constant__ CUtensorMap tm_wg, const __grid_constant__ CUtensorMap tm_wo,
                        const TriGateBwdParams p) {
    using L = TriGateBwdLayout;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sb - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto BAR = [&](int idx) -> uint32_t { return sb + L::OFF_BAR + idx * 8; };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
    const int tiles = (p.R + L::BM - 1) / L::BM;

    if (threadIdx.x == 0) {
        *abort_flag = device_error_pending() ? 1 : 0;
        mbar_init(BAR(L::B_W), 1);
        for (int s = 0; s < L::NS; ++s) {
            mbar_init(BAR(L::B_FULL + s), 1);
            mbar_init(BAR(L::B_XEMPTY + s), 1);
        }
        for (int b : {L::B_GFULL, L::B_DAFULL, L::B_AFREE, L::B_DZFULL, L::B_ACC}) mbar_init(BAR(b), 1);
        for (int b : {L::B_A1DONE, L::B_A2DONE, L::B_DLFULL, L::B_BDONE}) mbar_init(BAR(b), L::EPI_WARPS);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(const_cast<uint32_t*>(tmem_slot)), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtx wc{p.wait_limit_ns, KERNEL_TRIGATE, abort_flag};
    const bool aborted_early = *abort_flag != 0;

    if (warp == L::W_PRODUCER) {
        // =========================== TMA producer ===========================
        const bool leader = elect_one();
        int armed[L::NS] = {};
        bool w_armed = false;
        if (!aborted_early) {
            if (leader) {
                tma_prefetch_map(&tm_z);
                tma_prefetch_map(&tm_dy);
                mbar_arrive_expect_tx(BAR(L::B_W), 2 * L::W_TILE);
                tma_load_2d(sb + L::OFF_WG, &tm_wg, BAR(L::B_W), 0, 0);
                tma_load_2d(sb + L::OFF_WG + L::W_TILE / 2, &tm_wg, BAR(L::B_W), 64, 0);
                tma_load_2d(sb + L::OFF_WO, &tm_wo, BAR(L::B_W), 0, 0);
                tma_load_2d(sb + L::OFF_WO + L::W_TILE / 2, &tm_wo, BAR(L::B_W), 64, 0);
            }
            w_armed = true;
            int gt = 0;
            for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++gt) {
                const int s = gt % L::NS;
                if (gt >= L::NS && !mbar_wait_warp(BAR(L::B_XEMPTY + s), ((gt / L::NS) - 1) & 1, wc, 1)) break;
                if (leader) {
                    const uint32_t bar = BAR(L::B_FULL + s);
                    const uint32_t st = sb + L::OFF_STAGE + s * L::STAGE;
                    mbar_arrive_expect_tx(bar, L::STAGE);
                    tma_load_2d(st, &tm_z, bar, 0, t * L::BM);
                    tma_load_2d(st + L::HALF, &tm_z, bar, 64, t * L::BM);
                    tma_load_2d(st + L::X_TILE, &tm_dy, bar, 0, t * L::BM);
                    tma_load_2d(st + L::X_TILE + L::HALF, &tm_dy, bar, 64, t * L::BM);
                }
                armed[s]++;
            }
        }
        if (leader) {
            if (w_armed) drain_wait(BAR(L::B_W), 0, 100000000ull);
#pragma unroll
            for (int s = 0; s < L::NS; ++s)
                if (armed[s] > 0) drain_wait(BAR(L::B_FULL + s), (armed[s] - 1) & 1, 100000000ull);
        }
    } else if (warp == L::W_MMA) {
        // =========================== MMA issuer =============================
        const bool leader = elect_one();
        if (!aborted_early) {
            constexpr uint32_t ID_KM = idesc_bf16_f32(128, 128, false, true);
            constexpr uint32_t ID_KK = idesc_bf16_f32(128, 128, false, false);
            constexpr uint32_t ID_MM = idesc_bf16_f32(128, 128, true, true);
            // K-major view of a [128 rows][128] swizzled tile: 8-row groups 1 KB apart,
            // k steps of 16 are 32 bytes, the second 64-column half 16 KB on.
            // MN-major view of the same tile: 64-wide m/n chunks 16 KB apart (LBO),
            // 8-k-row groups 1 KB apart, k steps of 16 rows are 2 KB.
            auto kmaj = [&](uint32_t base, int kk) {
                return desc_add(smem_desc(base, 16, 1024, SWZ_128B), (kk >> 2) * L::HALF + (kk & 3) * 32);
            };
            auto mnmaj = [&](uint32_t base, int kk) {
                return desc_add(smem_desc(base, L::HALF, 1024, SWZ_128B), kk * 2048);
            };
            const uint32_t wg = sb + L::OFF_WG, wo = sb + L::OFF_WO, xb = sb + L::OFF_X;
            bool ok = mbar_wait_warp(BAR(L::B_W), 0, wc, 2);
            int lt = 0;
            for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++lt) {
                const int s = lt % L::NS, par = lt & 1;
                const uint32_t slot_g = tmem + (par ? 128u : 0u), slot_d = tmem + (par ? 0u : 128u);
                const uint32_t zt = sb + L::OFF_STAGE + s * L::STAGE, dyt = zt + L::X_TILE;
                // MMA1: G into the slot last holding the previous tile's dA
                if (!mbar_wait_warp(BAR(L::B_FULL + s), (lt / L::NS) & 1, wc, 3)) { ok = false; break; }
                if (lt > 0 && !mbar_wait_warp(BAR(L::B_A2DONE), (lt - 1) & 1, wc, 4)) { ok = false; break; }
                tc_fence_after();
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) mma_ss(slot_g, kmaj(zt, kk), mnmaj(wg, kk), ID_KM, kk > 0 ? 1u : 0u);
                    mma_commit(BAR(L::B_GFULL));
                }
                __syncwarp();
                // MMA2: dA into the slot last holding the previous tile's dz
                if (lt > 0 && !mbar_wait_warp(BAR(L::B_BDONE), (lt - 1) & 1, wc, 5)) { ok = false; break; }
                tc_fence_after();
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) mma_ss(slot_d, kmaj(dyt, kk), kmaj(wo, kk), ID_KK, kk > 0 ? 1u : 0u);
                    mma_commit(BAR(L::B_DAFULL));
                }
                __syncwarp();
                // MMA5: dWo += a^T dy
                if (!mbar_wait_warp(BAR(L::B_A1DONE), lt & 1, wc, 6)) { ok = false; break; }
                tc_fence_after();
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss(tmem + 384, mnmaj(xb, kk), mnmaj(dyt, kk), ID_MM, (lt > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(BAR(L::B_AFREE));
                }
                __syncwarp();
                // MMA3: dz into G's slot (read by A1 before dl was written);  MMA4: dWg += z^T dl
                if (!mbar_wait_warp(BAR(L::B_DLFULL), lt & 1, wc, 7)) { ok = false; break; }
                tc_fence_after();
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) mma_ss(slot_g, kmaj(xb, kk), kmaj(wg, kk), ID_KK, kk > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss(tmem + 256, mnmaj(zt, kk), mnmaj(xb, kk), ID_MM, (lt > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(BAR(L::B_DZFULL));
                    mma_commit(BAR(L::B_XEMPTY + s));
                }
                __syncwarp();
            }
            if (leader) mma_commit(BAR(L::B_ACC));  // every contraction above has completed
            __syncwarp();
        }
    } else {
        // =========================== epilogue (warps 0-7) =====================
        if (!aborted_early) {
            constexpr float LOG2E = 1.4426950408889634f;
            const int q = warp & 3, h = warp >> 2;
            const int row = q * 32 + lane;
            const uint32_t tl = tmem + (static_cast<uint32_t>(q * 32) << 16) + h * 64;
            const uint32_t xrow = sb + L::OFF_X + h * L::HALF + row * 128;
            const int ch0 = h * 64;  // first channel of this thread
            uint4 ov[8];             // o[r, ch0 .. ch0 + 63] of the current tile
            auto load_o = [&](int t) {
                const int r = t * L::BM + row;
                const __nv_bfloat16* src = p.o + static_cast<int64_t>(r) * p.os + ch0;
#pragma unroll
                for (int c = 0; c < 8; ++c) ov[c] = r < p.R ? ldg128_nc(src + 8 * c) : make_uint4(0, 0, 0, 0);
            };
            bool ok = true;
            int lt = 0;
            if (blockIdx.x < tiles) load_o(blockIdx.x);
            for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
                const int par = lt & 1;
                const uint32_t slot_g = tl + (par ? 128u : 0u), slot_d = tl + (par ? 0u : 128u);
                const int r = t * L::BM + row;
                const bool live = r < p.R;
                // ---- A1: g = sigmoid(G), a = g * o -> X; keep g and s = o g (1 - g) ----
                if (!mbar_wait_warp(BAR(L::B_GFULL), lt & 1, wc, 8)) { ok = false; break; }
                tc_fence_after();
                uint32_t gw[32], sw[32];  // BF16 pairs of g and s for the 64 channels
#pragma unroll
                for (int j = 0; j < 4; ++j) {  // 16-column chunks
                    uint32_t v[16];
                    tmem_ld16(slot_g + 16 * j, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 2; ++c) {  // 8 channels
                        const uint4 o4 = ov[2 * j + c];
                        const uint32_t ow[4] = {o4.x, o4.y, o4.z, o4.w};
                        uint32_t aw[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int k = 8 * c + 2 * e;
                            const float g0 = rcp_approx(1.f + ex2(-__uint_as_float(v[k]) * LOG2E));
                            const float g1 = rcp_approx(1.f + ex2(-__uint_as_float(v[k + 1]) * LOG2E));
                            const float o0 = bf16lo(ow[e]), o1 = bf16hi(ow[e]);
                            aw[e] = pack_bf16(g0 * o0, g1 * o1);
                            gw[8 * j + 4 * c + e] = pack_bf16(g0, g1);
                            sw[8 * j + 4 * c + e] = pack_bf16(o0 * (g0 * (1.f - g0)), o1 * (g1 * (1.f - g1)));
                        }
                        const int cc = 2 * j + c;  // 16-byte chunk within the 128-byte row
                        sts128(xrow + ((cc ^ (row & 7)) << 4), make_uint4(aw[0], aw[1], aw[2], aw[3]));
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(L::B_A1DONE));
                // ---- A2: dA -> do = dA g (global), dl = dA s (registers) ----
                if (!mbar_wait_warp(BAR(L::B_DAFULL), lt & 1, wc, 9)) { ok = false; break; }
                tc_fence_after();
                uint32_t dlw[32];
                __nv_bfloat16* dodst = p.d_o + static_cast<int64_t>(r) * p.dos + ch0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t v[16];
                    tmem_ld16(slot_d + 16 * j, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        uint32_t dw[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int k = 8 * c + 2 * e, w = 8 * j + 4 * c + e;
                            const float da0 = __uint_as_float(v[k]), da1 = __uint_as_float(v[k + 1]);
                            dw[e] = pack_bf16(da0 * bf16lo(gw[w]), da1 * bf16hi(gw[w]));
                            dlw[w] = pack_bf16(da0 * bf16lo(sw[w]), da1 * bf16hi(sw[w]));
                        }
                        if (live)
                            *reinterpret_cast<uint4*>(dodst + 16 * j + 8 * c) = make_uint4(dw[0], dw[1], dw[2], dw[3]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(L::B_A2DONE));
                // ---- dl -> X once MMA5 has read a ----
                if (!mbar_wait_warp(BAR(L::B_AFREE), lt & 1, wc, 10)) { ok = false; break; }
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    sts128(xrow + ((c ^ (row & 7)) << 4), make_uint4(dlw[4 * c], dlw[4 * c + 1], dlw[4 * c + 2], dlw[4 * c + 3]));
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(L::B_DLFULL));
                // fetch the next tile's o while this tile's dz is formed and drained
                if (t + static_cast<int>(gridDim.x) < tiles) load_o(t + gridDim.x);
                // ---- B: dz -> global ----
                if (!mbar_wait_warp(BAR(L::B_DZFULL), lt & 1, wc, 11)) { ok = false; break; }
                tc_fence_after();
                __nv_bfloat16* dzdst = p.dz + static_cast<int64_t>(r) * p.dzs + ch0;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    uint32_t v[32];
                    tmem_ld32(slot_g + 32 * j, v);
                    tmem_wait_ld();
                    if (j == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(BAR(L::B_BDONE));
                    }
                    if (live) {
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            uint4 w;
                            w.x = pack_bf16(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                            w.y = pack_bf16(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                            w.z = pack_bf16(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]));
                            w.w = pack_bf16(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7]));
                            *reinterpret_cast<uint4*>(dzdst + 32 * j + e) = w;
                        }
                    }
                }
            }
            // ---- weight-gradient partial sums -> workspace ----
            if (ok && mbar_wait_warp(BAR(L::B_ACC), 0, wc, 12)) {
                tc_fence_after();
                float* dst = p.partial + static_cast<int64_t>(blockIdx.x) * L::PARTIAL_FLOATS + row * L::C + ch0;
#pragma unroll 1
                for (int w = 0; w < 2; ++w) {  // 0: dWg (columns 256..), 1: dWo (384..)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        uint32_t v[32];
                        tmem_ld32(tl + 256 + 128 * w + 32 * j, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            *reinterpret_cast<uint4*>(dst + w * L::C * L::C + 32 * j + e) =
                                make_uint4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// dW[w][i][j] = sum over CTAs b = 0, 1, ... of partial[b][w][i][j], in that order
// (four interleaved running sums, combined at the end, so the result is the same
// on every run for the same number of partials).
__global__ void __launch_bounds__(256) tri_gate_wsum_kernel(const float* __restrict__ partial, int nparts,
                                                             float* __restrict__ dwg, float* __restrict__ dwo) {
    if (device_error_pending()) return;
    constexpr int N4 = TriGateBwdLayout::PARTIAL_FLOATS / 4;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;  // float4 index in [0, N4)
    if (i >= N4) return;
    const float4* src = reinterpret_cast<const float4*>(partial) + i;
    float4 acc[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    int b = 0;
    for (; b + 4 <= nparts; b += 4) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float4 x = src[static_cast<int64_t>(b + u) * N4];
            acc[u].x += x.x;
            acc[u].y += x.y;
            acc[u].z += x.z;
            acc[u].w += x.w;
        }
    }
#pragma unroll
    for (int u = 0; u < 3; ++u) {
        if (b + u < nparts) {
            const float4 x = src[static_cast<int64_t>(b + u) * N4];
            acc[u].x += x.x;
            acc[u].y += x.y;
            acc[u].z += x.z;
            acc[u].w += x.w;
        }
    }
    float4 r;
    r.x = (acc[0].x + acc[1].x) + (acc[2].x + acc[3].x);
    r.y = (acc[0].y + acc[1].y) + (acc[2].y + acc[3].y);
    r.z = (acc[0].z + acc[1].z) + (acc[2].z + acc[3].z);
    r.w = (acc[0].w + acc[1].w) + (acc[2].w + acc[3].w);
    constexpr int HALF4 = N4 / 2;
    if (i < HALF4)
        reinterpret_cast<float4*>(dwg)[i] = r;
    else
        reinterpret_cast<float4*>(dwo)[i - HALF4] = r;
}

}  // namespace tri
