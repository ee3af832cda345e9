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
// B200 mapping (one persistent CTA per SM, 320 threads):
//  * warp 8 TMA producer: Wg, Wo once (MN-major B operands, 32 KB each), then
//    per tile z (K-major A operand) into one of two slots and o into one of
//    three slots;
//  * warp 9 MMA issuer: G = z Wg into one of two 128-column TMEM accumulators,
//    later Y = a Wo into one of two more;
//  * warps 0-7 (warp w: rows 32 (w % 4) .. +31, one per thread, channel half
//    w / 4): sigmoid of G (exp2 on the FMA pipe, reciprocal on the MUFU unit),
//    a = g * o written in place over o -- whose 128-byte-swizzled K-major tile
//    is exactly the A operand the second MMA reads -- then, one tile behind,
//    Y -> BF16 into the same slot and out with a TMA store, so the tensor
//    cores, the MUFU unit and the stores of neighbouring tiles overlap.
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
    int R;  // pair positions
    uint64_t wait_limit_ns;
};

struct TriGateLayout {
    static constexpr int C = 128, BM = 128;
    static constexpr int W_TILE = C * C * 2;   // 32 KB
    static constexpr int X_TILE = BM * C * 2;  // 32 KB (two 64-column halves of 16 KB)
    static constexpr int HALF = X_TILE / 2;
    static constexpr int NZ = 2, NO = 3;       // z slots, o slots
    static constexpr int OFF_WG = 0, OFF_WO = W_TILE;
    static constexpr int OFF_Z = 2 * W_TILE;                // [NZ] z
    static constexpr int OFF_O = OFF_Z + NZ * X_TILE;       // [NO] o, then a, then y
    static constexpr int OFF_BAR = OFF_O + NO * X_TILE;
    static constexpr int B_W = 0, B_ZFULL = 1, B_ZEMPTY = B_ZFULL + NZ, B_OFULL = B_ZEMPTY + NZ,
                         B_OEMPTY = B_OFULL + NO, B_GFULL = B_OEMPTY + NO, B_GFREE = B_GFULL + 2,
                         B_AFULL = B_GFREE + 2, B_YFULL = B_AFULL + 1, B_YFREE = B_YFULL + 2, B_DRAIN = B_YFREE + 2,
                         NBAR = B_DRAIN + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int OFF_TRACE = (OFF_MISC + 16 + 7) & ~7;  // phase timing (TRI_TRACE builds only)
    static constexpr int TRACE_BYTES = (OFF_TRACE + kTraceBytes + 1024 <= 232448) ? kTraceBytes : 0;
    static constexpr int SMEM = OFF_TRACE + TRACE_BYTES + 1024;  // + slack for 1 KB alignment
    static constexpr int EPI_WARPS = 8, W_PRODUCER = 8, W_MMA = 9, THREADS = 320;
    static_assert(SMEM <= 232448, "shared memory budget");
};

__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// g = sigmoid(x) = 1 / (1 + e), e = 2^(-x log2 e), and h = 1 - g = e g (formed as a
// product, so it keeps its relative accuracy when the gate saturates at 1), for a pair
// of logits.  e comes from the FMA-pipe exp2 (relative error 1.4e-4), leaving the MUFU
// unit only the reciprocal; its argument is clamped to [-125, 126], where the result
// stays a normal number (g then rounds to 1 or to about 1e-38).
__device__ __forceinline__ void sigmoid2(float x0, float x1, float2& g, float2& h) {
    constexpr float NLOG2E = -1.4426950408889634f;
    const float2 e = ex2_fma2(make_float2(fminf(x0 * NLOG2E, 126.f), fminf(x1 * NLOG2E, 126.f)));
    g = make_float2(rcp_approx(1.f + e.x), rcp_approx(1.f + e.y));
    h = make_float2(e.x * g.x, e.y * g.y);
}

// 2-D tiled TMA store from shared memory, tracked by the issuing thread's bulk group.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, uint32_t src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(src), "r"(c0), "r"(c1)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// every bulk store this thread committed has finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// ... and has completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__global__ void __launch_bounds__(320, 1)
    tri_gate_fwd_kernel(const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_o,
                        const __grid_constant__ CUtensorMap tm_wg, const __grid_constant__ CUtensorMap tm_wo,
                        const __grid_constant__ CUtensorMap tm_y, const TriGateParams p) {
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
        for (int i = 0; i < L::NZ; ++i) {
            mbar_init(BAR(L::B_ZFULL + i), 1);
            mbar_init(BAR(L::B_ZEMPTY + i), 1);
        }
        for (int i = 0; i < L::NO; ++i) {
            mbar_init(BAR(L::B_OFULL + i), 1);
            mbar_init(BAR(L::B_OEMPTY + i), L::EPI_WARPS);  // every warp's y box read out
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(BAR(L::B_GFULL + x), 1);
            mbar_init(BAR(L::B_GFREE + x), L::EPI_WARPS);
            mbar_init(BAR(L::B_YFULL + x), 1);
            mbar_init(BAR(L::B_YFREE + x), L::EPI_WARPS);
        }
        mbar_init(BAR(L::B_AFULL), L::EPI_WARPS);
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

    if (warp == L::W_PRODUCER) {
        // =========================== TMA producer ===========================
        const bool leader = elect_one();
        int zarmed[L::NZ] = {}, oarmed[L::NO] = {};
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
                const int zs = gt % L::NZ, os = gt % L::NO;
                if (gt >= L::NZ && !mbar_wait_warp(BAR(L::B_ZEMPTY + zs), ((gt / L::NZ) - 1) & 1, wc, 1)) break;
                if (leader) {
                    const uint32_t bar = BAR(L::B_ZFULL + zs), dst = sb + L::OFF_Z + zs * L::X_TILE;
                    mbar_arrive_expect_tx(bar, L::X_TILE);
                    tma_load_2d(dst, &tm_z, bar, 0, t * L::BM);
                    tma_load_2d(dst + L::HALF, &tm_z, bar, 64, t * L::BM);
                }
                zarmed[zs]++;
                if (gt >= L::NO && !mbar_wait_warp(BAR(L::B_OEMPTY + os), ((gt / L::NO) - 1) & 1, wc, 11)) break;
                if (leader) {
                    const uint32_t bar = BAR(L::B_OFULL + os), dst = sb + L::OFF_O + os * L::X_TILE;
                    mbar_arrive_expect_tx(bar, L::X_TILE);
                    tma_load_2d(dst, &tm_o, bar, 0, t * L::BM);
                    tma_load_2d(dst + L::HALF, &tm_o, bar, 64, t * L::BM);
                }
                oarmed[os]++;
            }
        }
        if (leader) {
            if (w_armed) drain_wait(BAR(L::B_W), 0, 100000000ull);
#pragma unroll
            for (int i = 0; i < L::NZ; ++i)
                if (zarmed[i] > 0) drain_wait(BAR(L::B_ZFULL + i), (zarmed[i] - 1) & 1, 100000000ull);
#pragma unroll
            for (int i = 0; i < L::NO; ++i)
                if (oarmed[i] > 0) drain_wait(BAR(L::B_OFULL + i), (oarmed[i] - 1) & 1, 100000000ull);
        }
    } else if (warp == L::W_MMA) {
        // =========================== MMA issuer =============================
        const bool leader = elect_one();
        if (!aborted_early) {
            constexpr uint32_t IDESC = idesc_bf16_f32(128, 128, false, true);
            // A (z, a): K-major, two 64-column halves 16 KB apart; B (Wg, Wo): MN-major,
            // 64-column chunks 16 KB apart (LBO), 8-k-row groups 1 KB apart (SBO)
            const uint64_t dz0 = smem_desc(sb + L::OFF_Z, 16, 1024, SWZ_128B);
            const uint64_t da0 = smem_desc(sb + L::OFF_O, 16, 1024, SWZ_128B);
            const uint64_t dwg = smem_desc(sb + L::OFF_WG, L::HALF, 1024, SWZ_128B);
            const uint64_t dwo = smem_desc(sb + L::OFF_WO, L::HALF, 1024, SWZ_128B);
            bool ok = mbar_wait_warp(BAR(L::B_W), 0, wc, 2);
            TRI_TRACE_DECL
            int lt = 0;
            for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++lt) {
                const int x = lt & 1, zs = lt % L::NZ, os = lt % L::NO;
                TRI_TP(5)
                if (!mbar_wait_warp(BAR(L::B_ZFULL + zs), (lt / L::NZ) & 1, wc, 3)) { ok = false; break; }
                TRI_TP(0)
                if (lt >= 2 && !mbar_wait_warp(BAR(L::B_GFREE + x), ((lt >> 1) - 1) & 1, wc, 4)) { ok = false; break; }
                TRI_TP(1)
                tc_fence_after();
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss(tmem + x * 128, desc_add(dz0, zs * L::X_TILE + (kk >> 2) * L::HALF + (kk & 3) * 32),
                               desc_add(dwg, kk * 2048), IDESC, kk > 0 ? 1u : 0u);
                    mma_commit(BAR(L::B_GFULL + x));
                    mma_commit(BAR(L::B_ZEMPTY + zs));
                }
                __syncwarp();
                // the gated a of this tile is in its o slot; Y[x] was read two tiles ago
                TRI_TP(5)
                if (!mbar_wait_warp(BAR(L::B_AFULL), lt & 1, wc, 5)) { ok = false; break; }
                TRI_TP(2)
                if (lt >= 2 && !mbar_wait_warp(BAR(L::B_YFREE + x), ((lt >> 1) - 1) & 1, wc, 6)) { ok = false; break; }
                TRI_TP(3)
                tc_fence_after();
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss(tmem + 256 + x * 128,
                               desc_add(da0, os * L::X_TILE + (kk >> 2) * L::HALF + (kk & 3) * 32),
                               desc_add(dwo, kk * 2048), IDESC, kk > 0 ? 1u : 0u);
                    mma_commit(BAR(L::B_YFULL + x));
                }
                __syncwarp();
            }
            TRI_TP(5)
            TRI_TRACE_FLUSH_AT(0)
            if (leader) {
                mma_commit(BAR(L::B_DRAIN));
                drain_wait(BAR(L::B_DRAIN), 0, 100000000ull);
            }
            __syncwarp();
        }
    } else {
        // =========================== gate + epilogue (warps 0-7) =============
        if (!aborted_early) {
            const int q = warp & 3, h = warp >> 2;
            const int row = q * 32 + lane;
            const uint32_t tl = tmem + (static_cast<uint32_t>(q * 32) << 16) + h * 64;
            const uint32_t box = h * L::HALF + q * 32 * 128;  // this warp's 32 x 64 box within a slot
            bool ok = true;
            TRI_TRACE_DECL
            // Y of tile lt (local index) -> BF16 into its o slot -> TMA store
            auto store_y = [&](int lt, int t) -> bool {
                const int x = lt & 1;
                TRI_TP(6)
                if (!mbar_wait_warp(BAR(L::B_YFULL + x), (lt >> 1) & 1, wc, 9)) return false;
                TRI_TP(4)
                tc_fence_after();
                const uint32_t slot = sb + L::OFF_O + (lt % L::NO) * L::X_TILE + h * L::HALF;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    uint32_t v[32];
                    tmem_ld32(tl + 256 + x * 128 + 32 * j, v);
                    tmem_wait_ld();
                    if (j == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(BAR(L::B_YFREE + x));
                    }
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                        w.y = pack_bf16(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                        w.z = pack_bf16(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]));
                        w.w = pack_bf16(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7]));
                        const int c = 4 * j + (e >> 3);
                        sts128(slot + row * 128 + ((c ^ (row & 7)) << 4), w);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                const int box_row = t * L::BM + q * 32;
                if (lane == 0 && box_row < p.R) {
                    tma_store_2d(&tm_y, sb + L::OFF_O + (lt % L::NO) * L::X_TILE + box, h * 64, box_row);
                    bulk_commit();
                }
                TRI_TP(5)
                return true;
            };
            int lt = 0, prev_t = -1;
            for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
                const int x = lt & 1, os = lt % L::NO;
                TRI_TP(6)
                if (!mbar_wait_warp(BAR(L::B_GFULL + x), (lt >> 1) & 1, wc, 7)) { ok = false; break; }
                if (lt >= 2) {  // the y box of tile lt - 2 has left its slot
                    if (lane == 0) {
                        bulk_wait_read_all();
                        mbar_arrive(BAR(L::B_OEMPTY + (lt - 2) % L::NO));
                    }
                    __syncwarp();
                }
                TRI_TP(0)
                if (!mbar_wait_warp(BAR(L::B_OFULL + os), (lt / L::NO) & 1, wc, 8)) { ok = false; break; }
                tc_fence_after();
                const uint32_t orow = sb + L::OFF_O + os * L::X_TILE + h * L::HALF + row * 128;
#pragma unroll
                for (int j = 0; j < 2; ++j) {  // 32-column chunks
                    uint32_t gv[32];
                    tmem_ld32(tl + x * 128 + 32 * j, gv);
                    tmem_wait_ld();
                    if (j == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(BAR(L::B_GFREE + x));
                    }
#pragma unroll
                    for (int c = 0; c < 4; ++c) {  // 16-byte chunks of 8 channels
                        const int cc = 4 * j + c;
                        const uint32_t addr = orow + ((cc ^ (row & 7)) << 4);
                        const uint4 ob = lds128(addr);
                        const uint32_t ow[4] = {ob.x, ob.y, ob.z, ob.w};
                        uint32_t aw[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            float2 g, hh;
                            sigmoid2(__uint_as_float(gv[8 * c + 2 * e]), __uint_as_float(gv[8 * c + 2 * e + 1]), g, hh);
                            aw[e] = pack_bf16(g.x * bf16lo(ow[e]), g.y * bf16hi(ow[e]));
                        }
                        sts128(addr, make_uint4(aw[0], aw[1], aw[2], aw[3]));  // a over o, in place
                    }
                }
                TRI_TP(1)
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(L::B_AFULL));
                TRI_TP(3)
                // the previous tile's output, while the tensor cores work on this one
                if (prev_t >= 0 && !(ok = store_y(lt - 1, prev_t))) break;
                prev_t = t;
            }
            if (ok && prev_t >= 0) store_y(lt - 1, prev_t);
            if (lane == 0) bulk_wait_all();  // every y box has reached global memory
            TRI_TP(6)
            TRI_TRACE_FLUSH_AT(0)
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
// do and dz leave through shared memory and TMA stores (one 32-row x 64-column
// box per epilogue warp): do in the dy slot of the tile's stage once MMA5 has
// consumed dy, dz in the z slot once MMA4 has consumed z; the epilogue then
// hands the stage back to the producer.
// Each CTA writes its FP32 dWg, dWo partial sums to a workspace; a second
// kernel adds the partials in CTA order (deterministic for a given R).
//
// Warps 0-7 (epilogue; warp w reads TMEM lanes 32 (w % 4) .. +31, i.e. rows,
// and channel half w / 4), warp 8 TMA producer, warp 9 MMA issuer.
// Per tile, each epilogue thread: A1 reads G, writes a = g * o (BF16) into
// the shared tile X and keeps g and s = o g (1 - g), both rounded to BF16, in
// registers (s is formed in FP32 from the FP32 g, so 1 - g keeps its relative
// accuracy for saturated gates); A2 reads dA and forms do = dA g and
// dl = dA s, and once MMA5 has finished with a and dy writes dl over a in X and
// do into the dy slot; B reads dz into the z slot.  o comes straight from
// global memory into registers, prefetched one tile ahead.
// ===========================================================================
struct TriGateBwdParams {
    int R;
    const __nv_bfloat16* o;
    int64_t os;
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
    static constexpr int OFF_TRACE = (OFF_MISC + 16 + 7) & ~7;  // phase timing (TRI_TRACE builds only)
    static constexpr int TRACE_BYTES = (OFF_TRACE + kTraceBytes + 1024 <= 232448) ? kTraceBytes : 0;
    static constexpr int SMEM = OFF_TRACE + TRACE_BYTES + 1024;  // + slack for 1 KB alignment
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
                        const __grid_constant__ CUtensorMap tm_dz, const __grid_constant__ CUtensorMap tm_do,
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
            mbar_init(BAR(L::B_XEMPTY + s), L::EPI_WARPS);  // both output boxes of every warp read out
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
            TRI_TRACE_DECL
            int lt = 0;
            for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++lt) {
                const int s = lt % L::NS, par = lt & 1;
                const uint32_t slot_g = tmem + (par ? 128u : 0u), slot_d = tmem + (par ? 0u : 128u);
                const uint32_t zt = sb + L::OFF_STAGE + s * L::STAGE, dyt = zt + L::X_TILE;
                // MMA1: G into the slot last holding the previous tile's dA
                TRI_TP(5)
                if (!mbar_wait_warp(BAR(L::B_FULL + s), (lt / L::NS) & 1, wc, 3)) { ok = false; break; }
                TRI_TP(0)
                if (lt > 0 && !mbar_wait_warp(BAR(L::B_A2DONE), (lt - 1) & 1, wc, 4)) { ok = false; break; }
                TRI_TP(1)
                tc_fence_after();
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) mma_ss(slot_g, kmaj(zt, kk), mnmaj(wg, kk), ID_KM, kk > 0 ? 1u : 0u);
                    mma_commit(BAR(L::B_GFULL));
                }
                __syncwarp();
                // MMA2: dA into the slot last holding the previous tile's dz
                TRI_TP(5)
                if (lt > 0 && !mbar_wait_warp(BAR(L::B_BDONE), (lt - 1) & 1, wc, 5)) { ok = false; break; }
                TRI_TP(2)
                tc_fence_after();
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) mma_ss(slot_d, kmaj(dyt, kk), kmaj(wo, kk), ID_KK, kk > 0 ? 1u : 0u);
                    mma_commit(BAR(L::B_DAFULL));
                }
                __syncwarp();
                // MMA5: dWo += a^T dy
                TRI_TP(5)
                if (!mbar_wait_warp(BAR(L::B_A1DONE), lt & 1, wc, 6)) { ok = false; break; }
                TRI_TP(3)
                tc_fence_after();
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss(tmem + 384, mnmaj(xb, kk), mnmaj(dyt, kk), ID_MM, (lt > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(BAR(L::B_AFREE));
                }
                __syncwarp();
                // MMA3: dz into G's slot (read by A1 before dl was written);  MMA4: dWg += z^T dl
                TRI_TP(5)
                if (!mbar_wait_warp(BAR(L::B_DLFULL), lt & 1, wc, 7)) { ok = false; break; }
                TRI_TP(4)
                tc_fence_after();
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) mma_ss(slot_g, kmaj(xb, kk), kmaj(wg, kk), ID_KK, kk > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss(tmem + 256, mnmaj(zt, kk), mnmaj(xb, kk), ID_MM, (lt > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(BAR(L::B_DZFULL));
                }
                __syncwarp();
            }
            TRI_TP(5)
            TRI_TRACE_FLUSH_AT(0)
            if (leader) mma_commit(BAR(L::B_ACC));  // every contraction above has completed
            __syncwarp();
        }
    } else {
        // =========================== epilogue (warps 0-7) =====================
        if (!aborted_early) {
            const int q = warp & 3, h = warp >> 2;
            const int row = q * 32 + lane;
            const uint32_t tl = tmem + (static_cast<uint32_t>(q * 32) << 16) + h * 64;
            const uint32_t xrow = sb + L::OFF_X + h * L::HALF + row * 128;
            const int ch0 = h * 64;  // first channel of this thread
            // o[r, ch0 .. ch0 + 63] of the current tile as eight 16-byte chunks.  Loaded
            // coalesced -- lane 8a + b, load i fetches chunk b of warp row 8a + i, so one load
            // covers four whole 128-byte lines -- then transposed within each group of
            // eight lanes (three butterfly exchange steps) so that lane L holds row L.
            uint32_t ov[8][4];
            auto load_o = [&](int t) {
                const int a8 = lane >> 3, b8 = lane & 7;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = t * L::BM + q * 32 + 8 * a8 + i;
                    const uint4 v = r < p.R ? ldg128_nc(p.o + static_cast<int64_t>(r) * p.os + ch0 + 8 * b8)
                                            : make_uint4(0, 0, 0, 0);
                    ov[i][0] = v.x;
                    ov[i][1] = v.y;
                    ov[i][2] = v.z;
                    ov[i][3] = v.w;
                }
            };
            auto transpose_o = [&]() {
#pragma unroll
                for (int k = 0; k < 3; ++k) {
                    const int m = 1 << k;
                    const bool up = (lane & m) != 0;
#pragma unroll
                    for (int i0 = 0; i0 < 8; ++i0) {
                        if (i0 & m) continue;
                        const int i1 = i0 | m;
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            const uint32_t recv = __shfl_xor_sync(0xffffffffu, up ? ov[i0][w] : ov[i1][w], m);
                            if (up)
                                ov[i0][w] = recv;
                            else
                                ov[i1][w] = recv;
                        }
                    }
                }
            };
            bool ok = true;
            int lt = 0;
            if (blockIdx.x < tiles) load_o(blockIdx.x);
            TRI_TRACE_DECL
            for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
                const int par = lt & 1;
                const uint32_t slot_g = tl + (par ? 128u : 0u), slot_d = tl + (par ? 0u : 128u);
                TRI_TP(7)
#ifdef TRI_TRACE
                {  // time the wait for this tile's o on its own
                    uint32_t x_ = 0;
#pragma unroll
                    for (int c = 0; c < 8; ++c) x_ ^= ov[c][0] ^ ov[c][3];
                    if (x_ == 0x9e3779b9u) asm volatile("" ::: "memory");
                }
                TRI_TP(9)
#endif
                // ---- A1: g = sigmoid(G), a = g * o -> X; keep g and s = o g (1 - g) ----
                if (!mbar_wait_warp(BAR(L::B_GFULL), lt & 1, wc, 8)) { ok = false; break; }
                if (lt > 0) {  // the previous tile's do and dz boxes have left its stage
                    if (lane == 0) {
                        bulk_wait_read_all();
                        mbar_arrive(BAR(L::B_XEMPTY + (lt - 1) % L::NS));
                    }
                    __syncwarp();
                }
                TRI_TP(0)
                tc_fence_after();
                transpose_o();
                uint32_t gw[32], sw[32];  // BF16 pairs of g and s for the 64 channels
#pragma unroll
                for (int j = 0; j < 4; ++j) {  // 16-column chunks
                    uint32_t v[16];
                    tmem_ld16(slot_g + 16 * j, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 2; ++c) {  // 8 channels
                        const uint32_t* ow = ov[2 * j + c];
                        uint32_t aw[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int k = 8 * c + 2 * e;
                            float2 g, h;  // g and 1 - g
                            sigmoid2(__uint_as_float(v[k]), __uint_as_float(v[k + 1]), g, h);
                            const float o0 = bf16lo(ow[e]), o1 = bf16hi(ow[e]);
                            aw[e] = pack_bf16(g.x * o0, g.y * o1);
                            gw[8 * j + 4 * c + e] = pack_bf16(g.x, g.y);
                            sw[8 * j + 4 * c + e] = pack_bf16(o0 * (g.x * h.x), o1 * (g.y * h.y));
                        }
                        const int cc = 2 * j + c;  // 16-byte chunk within the 128-byte row
                        sts128(xrow + ((cc ^ (row & 7)) << 4), make_uint4(aw[0], aw[1], aw[2], aw[3]));
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(L::B_A1DONE));
                TRI_TP(1)
                // ---- A2: dA -> do = dA g, dl = dA s (registers) ----
                if (!mbar_wait_warp(BAR(L::B_DAFULL), lt & 1, wc, 9)) { ok = false; break; }
                TRI_TP(2)
                tc_fence_after();
                uint32_t dlw[32], dow[32];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t v[16];
                    tmem_ld16(slot_d + 16 * j, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int k = 8 * c + 2 * e, w = 8 * j + 4 * c + e;
                            const float da0 = __uint_as_float(v[k]), da1 = __uint_as_float(v[k + 1]);
                            dow[w] = pack_bf16(da0 * bf16lo(gw[w]), da1 * bf16hi(gw[w]));
                            dlw[w] = pack_bf16(da0 * bf16lo(sw[w]), da1 * bf16hi(sw[w]));
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(L::B_A2DONE));
                TRI_TP(3)
                // ---- dl -> X, do -> dy slot, once MMA5 has read a and dy ----
                if (!mbar_wait_warp(BAR(L::B_AFREE), lt & 1, wc, 10)) { ok = false; break; }
                TRI_TP(4)
                const uint32_t zslot = sb + L::OFF_STAGE + (lt % L::NS) * L::STAGE, dyslot = zslot + L::X_TILE;
                const uint32_t box = h * L::HALF + q * 32 * 128;  // this warp's 32 x 64 box in a slot
                const int box_row = t * L::BM + q * 32;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint32_t off = row * 128 + ((c ^ (row & 7)) << 4);
                    sts128(xrow + ((c ^ (row & 7)) << 4), make_uint4(dlw[4 * c], dlw[4 * c + 1], dlw[4 * c + 2], dlw[4 * c + 3]));
                    sts128(dyslot + h * L::HALF + off,
                           make_uint4(dow[4 * c], dow[4 * c + 1], dow[4 * c + 2], dow[4 * c + 3]));
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(BAR(L::B_DLFULL));
                    if (box_row < p.R) {
                        tma_store_2d(&tm_do, dyslot + box, ch0, box_row);
                        bulk_commit();
                    }
                }
                // fetch the next tile's o while this tile's dz is formed and drained
                if (t + static_cast<int>(gridDim.x) < tiles) load_o(t + gridDim.x);
                TRI_TP(5)
                // ---- B: dz -> z slot -> global ----
                if (!mbar_wait_warp(BAR(L::B_DZFULL), lt & 1, wc, 11)) { ok = false; break; }
                TRI_TP(6)
                tc_fence_after();
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
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                        w.y = pack_bf16(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                        w.z = pack_bf16(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]));
                        w.w = pack_bf16(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7]));
                        const int c = 4 * j + (e >> 3);
                        sts128(zslot + h * L::HALF + row * 128 + ((c ^ (row & 7)) << 4), w);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && box_row < p.R) {
                    tma_store_2d(&tm_dz, zslot + box, ch0, box_row);
                    bulk_commit();
                }
            }
            if (lane == 0) bulk_wait_all();  // every output box has reached global memory
            TRI_TP(7)
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
            TRI_TP(8)
            TRI_TRACE_FLUSH_AT(0)
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// dW[w][i][j] = sum over CTAs b of partial[b][w][i][j].  Eight threads share each
// float4 of the result: thread k adds partials k, k + 8, k + 16, ... in that order,
// then the eight partial sums are combined by a butterfly (pairwise sums are
// commutative, so every lane ends with the same bits).  The association is fixed
// by the number of partials alone, so repeated runs give identical results.
constexpr int kWsumThreads = 256;
__global__ void __launch_bounds__(kWsumThreads) tri_gate_wsum_kernel(const float* __restrict__ partial, int nparts,
                                                                      float* __restrict__ dwg, float* __restrict__ dwo) {
    if (device_error_pending()) return;
    constexpr int N4 = TriGateBwdLayout::PARTIAL_FLOATS / 4;
    const int i = blockIdx.x * (kWsumThreads / 8) + (threadIdx.x >> 3);  // float4 index in [0, N4)
    const int k = threadIdx.x & 7;
    if (i >= N4) return;  // whole groups of eight leave together
    const float4* src = reinterpret_cast<const float4*>(partial) + i;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int b = k;
    for (; b + 24 < nparts; b += 32) {
        float4 x[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) x[u] = src[static_cast<int64_t>(b + 8 * u) * N4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            acc.x += x[u].x;
            acc.y += x[u].y;
            acc.z += x[u].z;
            acc.w += x[u].w;
        }
    }
    for (; b < nparts; b += 8) {
        const float4 x = src[static_cast<int64_t>(b) * N4];
        acc.x += x.x;
        acc.y += x.y;
        acc.z += x.z;
        acc.w += x.w;
    }
#pragma unroll
    for (int m = 1; m < 8; m <<= 1) {
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, m);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, m);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, m);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, m);
    }
    if (k != 0) return;
    constexpr int HALF4 = N4 / 2;
    if (i < HALF4)
        reinterpret_cast<float4*>(dwg)[i] = acc;
    else
        reinterpret_cast<float4*>(dwo)[i - HALF4] = acc;
}

}  // namespace tri
