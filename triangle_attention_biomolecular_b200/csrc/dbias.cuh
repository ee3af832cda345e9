// dbias.cuh -- the dBias pass of the triangle-attention backward (sm_100a).
//
// dBias[b,h,j,k] = sum_i dS[b,i,j,h,k]: the pair bias is shared by every row i
// ("16张H100，训练步提速1.73倍：TurboPairFormer…", section "它优化了什么": the
// four gradients include the shared pair bias; no floating-point atomics), so
// this pass is tile-stationary: one CTA per (b, h, query tile jt, key tile kt)
// and row chunk walks the rows i in ascending order, recomputes the score and
// score-gradient tiles with tcgen05 and accumulates dS in FP32 registers.
//
// The per-row softmax statistics enter the contractions instead of the
// element-wise arithmetic.  The MMA warp adds one more K=16 step to each
// product, an augmentation block times a block of ones:
//     S'  = Q K^T  + A_L 1^T,   A_L[j] = -(lse_j / scale)  as hi + mid + lo BF16
//     dP' = dO V^T + A_D 1^T,   A_D[j] = -D_j              as hi + mid + lo BF16
// (three BF16 terms carry the FP32 value to within 2^-24 relative, the
// products are exact and accumulate in FP32).  Then per score, in base 2,
//     p = 2^(c S' + bias log2 e [+ mask log2 e]),  c = scale log2 e,
//     acc += p * dP'                                   (= dS)
// i.e. two packed FP32 instructions and one exponential per pair of scores.  The
// tile's bias (log2 units) stays in each softmax thread's registers for the whole
// row walk, and S', dP' come from TMEM 16 keys at a time to leave room for it.
//
// Roles (640 threads): warps 0-15 four softmax warpgroups (warpgroup w owns
// keys 32w..32w+31 of the tile, warp%4 the TMEM lane quarter); warp 16 TMA
// producer; warp 17 MMA issuer; warp 18 writes the augmentation blocks of
// each stage from the bulk-loaded lse / D vectors; warp 19 idle.
#pragma once

#include <type_traits>

#include "sm100.cuh"
#include "bwd.cuh"

// pairs of every eight that take the FMA-pipe exponential (key tiles without a mask)
#ifndef TRI_DBIAS_FMA_PAIRS
#define TRI_DBIAS_FMA_PAIRS 2
#endif

namespace tri {

template <int D>
struct DbLayout {
    static constexpr int NS = (D == 32) ? 3 : 2;  // row stages
    static constexpr int ROWB = D * 2;
    static constexpr int QKV_TILE = 128 * ROWB;
    // augmentation blocks: 128 rows x 16 BF16, K-major without swizzle: 8x8 core
    // matrices, the two K-halves 128 B apart (LBO), 8-row groups 256 B apart (SBO)
    static constexpr int AUG_TILE = 128 * 32, AUG_LBO = 128, AUG_SBO = 256;
    static constexpr int OFF_Q = 0, OFF_DO = QKV_TILE, OFF_K = 2 * QKV_TILE, OFF_V = 3 * QKV_TILE;
    static constexpr int OFF_AL = 4 * QKV_TILE, OFF_AD = OFF_AL + AUG_TILE;
    static constexpr int STAGE = 4 * QKV_TILE + 2 * AUG_TILE;
    static constexpr int THREADS = 640, SOFTMAX_WARPS = 16, W_PRODUCER = 16, W_MMA = 17, W_AUG = 18;
    static constexpr int OFF_ONES = NS * STAGE;  // B block of ones (keys x 16), AUG layout
    // per-row vectors, in a deeper ring of their own so that a row's tiles are
    // released as soon as its products finish: lse*log2e 128, D 128,
    // mask*log2e 128 (fp32), key-tile flags 32 (int)
    static constexpr int NV = 6;
    static constexpr int OFF_VEC = OFF_ONES + AUG_TILE;
    static constexpr int VEC = 1664;
    static constexpr int OFF_BAR = OFF_VEC + NV * VEC;
    static constexpr int B_FULL = 0, B_EMPTY = NS, B_AUG = 2 * NS, B_VFULL = 3 * NS, B_VEMPTY = 3 * NS + NV,
                         B_SDPFULL = 3 * NS + 2 * NV, B_SDPFREE = B_SDPFULL + 2, B_DRAIN = B_SDPFULL + 4,
                         NBAR = B_DRAIN + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort
    static constexpr int OFF_TRACE = (OFF_MISC + 16 + 7) & ~7;  // phase timing (TRI_TRACE builds only)
    static constexpr int TRACE_BYTES = (OFF_TRACE + kTraceBytes <= 232448) ? kTraceBytes : 0;
    static constexpr int SMEM = OFF_TRACE + TRACE_BYTES;
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(STAGE % 1024 == 0 && QKV_TILE % 1024 == 0, "swizzled tiles need 1 KB alignment");
    static_assert(OFF_BAR % 8 == 0, "mbarrier alignment");
};

// byte offset of element e (0..15) of row r in an augmentation / ones block
__device__ __forceinline__ uint32_t aug_offset(int r, int e) {
    return static_cast<uint32_t>((r >> 3) * 256 + (e >> 3) * 128 + (r & 7) * 16 + (e & 7) * 2);
}

// x as hi + mid + lo, each BF16 round-to-nearest of what the previous terms
// left (the differences are exact in FP32)
__device__ __forceinline__ uint4 split3_bf16(float x) {
    const uint32_t hi_w = pack_bf16(x, 0.f);
    const float r1 = x - bf16lo(hi_w);
    const uint32_t mid_w = pack_bf16(r1, 0.f);
    const float r2 = r1 - bf16lo(mid_w);
    const uint32_t lo_w = pack_bf16(r2, 0.f);
    return make_uint4((hi_w & 0xFFFFu) | (mid_w << 16), lo_w & 0xFFFFu, 0u, 0u);
}

// FMA_PAIRS: how many of every eight score pairs take the FMA-pipe exponential
// in key tiles without a mask (the rest, and every masked tile, use MUFU)
template <int D, int FMA_PAIRS>
__global__ void __launch_bounds__(640, 1)
    tri_attn_bwd_dbias_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                              const __nv_bfloat16* __restrict__ bias, int64_t bs0, int64_t bs1, int64_t bs2,
                              const BwdParams p) {
    using L = DbLayout<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sb = smem_addr(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto BAR = [&](int idx) -> uint32_t { return sb + L::OFF_BAR + idx * 8; };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

    const int nt = p.nt;
    int item = blockIdx.x;
    const int chunk = item % p.chunks;
    item /= p.chunks;
    const int kt = item % nt;
    item /= nt;
    const int jt = item % nt;
    item /= nt;
    const int h = item % p.H;
    const int b = item / p.H;
    const int rows_per = (p.R + p.chunks - 1) / p.chunks;
    const int i_begin = chunk * rows_per;
    const int i_end = min(p.R, i_begin + rows_per);
    const int nrows = max(0, i_end - i_begin);
    constexpr float LOG2E = 1.4426950408889634f;

    if (threadIdx.x == 0) {
        *abort_flag = device_error_pending() ? 1 : 0;
        if (sb & 1023u) {
            atomicCAS(&g_error_word, 0u, ERR_TIMEOUT_BIT | KERNEL_BWD_DBIAS | 0xFFu);
            *abort_flag = 1;
        }
        for (int s = 0; s < L::NS; ++s) {
            mbar_init(BAR(L::B_FULL + s), 1);
            mbar_init(BAR(L::B_EMPTY + s), 1);  // the MMA commit alone: the tiles are read only by MMAs
            mbar_init(BAR(L::B_AUG + s), 1);
        }
        for (int v = 0; v < L::NV; ++v) {
            mbar_init(BAR(L::B_VFULL + v), 1);
            mbar_init(BAR(L::B_VEMPTY + v), L::SOFTMAX_WARPS + 1);  // softmax warps + augmentation writer
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(BAR(L::B_SDPFULL + x), 1);
            mbar_init(BAR(L::B_SDPFREE + x), L::SOFTMAX_WARPS);
        }
        mbar_init(BAR(L::B_DRAIN), 1);
        fence_mbar_init();
    }
    // augmentation blocks start as zeros (only elements 0..2 of each row are ever
    // rewritten); the ones block holds 1 in elements 0..2 of every key row
    for (int idx = threadIdx.x; idx < L::NS * 2 * (L::AUG_TILE / 16); idx += blockDim.x) {
        const int s = idx / (2 * (L::AUG_TILE / 16)), r = idx % (2 * (L::AUG_TILE / 16));
        sts128(sb + s * L::STAGE + L::OFF_AL + r * 16, make_uint4(0u, 0u, 0u, 0u));
    }
    for (int r = threadIdx.x; r < 128; r += blockDim.x) {
        sts128(sb + L::OFF_ONES + aug_offset(r, 0), make_uint4(0x3F803F80u, 0x3F80u, 0u, 0u));
        sts128(sb + L::OFF_ONES + aug_offset(r, 8), make_uint4(0u, 0u, 0u, 0u));
    }
    fence_proxy_async_smem();
    if (warp == 0) {
        tmem_alloc(smem_addr(const_cast<uint32_t*>(tmem_slot)), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtx wc{p.wait_limit_ns, KERNEL_BWD_DBIAS, abort_flag};
    const bool aborted_early = *abort_flag != 0;

    if (warp == L::W_PRODUCER) {
        regs_shrink640w();
        int armed[L::NS], varmed[L::NV];
#pragma unroll
        for (int s = 0; s < L::NS; ++s) armed[s] = 0;
#pragma unroll
        for (int v = 0; v < L::NV; ++v) varmed[v] = 0;
        const bool leader = elect_one();
        if (!aborted_early) {
            if (leader) {
                tma_prefetch_map(&tm_q);
                tma_prefetch_map(&tm_k);
                tma_prefetch_map(&tm_v);
                tma_prefetch_map(&tm_do);
            }
            for (int n = 0; n < nrows; ++n) {
                const int i = i_begin + n;
                const int s = n % L::NS, v = n % L::NV;
                if (n >= L::NV && !mbar_wait_warp(BAR(L::B_VEMPTY + v), ((n / L::NV) - 1) & 1, wc, 8)) break;
                if (leader) {
                    const uint32_t bar = BAR(L::B_VFULL + v);
                    const uint32_t vec = sb + L::OFF_VEC + v * L::VEC;
                    const int64_t vrow = ((static_cast<int64_t>(b) * p.H + h) * p.R + i) * p.Np + jt * 128;
                    const int64_t mrow = (static_cast<int64_t>(b) * p.R + i) * p.Np + kt * 128;
                    mbar_arrive_expect_tx(bar, L::VEC);
                    bulk_load(vec, p.Lv + vrow, 512, bar);
                    bulk_load(vec + 512, p.Dv + vrow, 512, bar);
                    bulk_load(vec + 1024, p.Mv + mrow, 512, bar);
                    bulk_load(vec + 1536, p.Fv + (static_cast<int64_t>(b) * p.R + i) * 32, 128, bar);
                }
                varmed[v]++;
                if (n >= L::NS && !mbar_wait_warp(BAR(L::B_EMPTY + s), ((n / L::NS) - 1) & 1, wc, 1)) break;
                if (leader) {
                    const uint32_t bar = BAR(L::B_FULL + s);
                    const uint32_t base = sb + s * L::STAGE;
                    mbar_arrive_expect_tx(bar, 4 * L::QKV_TILE);
                    auto ld = [&](uint32_t dst, const CUtensorMap* m, int row0) {
                        tma_load_5d(dst, m, bar, 0, h, row0, i, b);
                    };
                    ld(base + L::OFF_Q, &tm_q, jt * 128);
                    ld(base + L::OFF_DO, &tm_do, jt * 128);
                    ld(base + L::OFF_K, &tm_k, kt * 128);
                    ld(base + L::OFF_V, &tm_v, kt * 128);
                }
                armed[s]++;
            }
        }
        if (leader) {
#pragma unroll
            for (int s = 0; s < L::NS; ++s)
                if (armed[s] > 0) drain_wait(BAR(L::B_FULL + s), (armed[s] - 1) & 1, 100000000ull);
#pragma unroll
            for (int v = 0; v < L::NV; ++v)
                if (varmed[v] > 0) drain_wait(BAR(L::B_VFULL + v), (varmed[v] - 1) & 1, 100000000ull);
        }
    } else if (warp == L::W_AUG) {
        // ====== augmentation blocks: -(lse/scale) and -D as hi + mid + lo BF16 ======
        regs_shrink640w();
        if (!aborted_early) {
            // Lv holds -lse * log2(e); -lse / scale = Lv / c.  Padded query rows (Lv = -inf)
            // get a large finite negative term so that their scores underflow to 0.
            const float inv_c = 1.0f / (p.scale * LOG2E);
            for (int n = 0; n < nrows; ++n) {
                const int s = n % L::NS, v = n % L::NV;
                if (!mbar_wait_warp(BAR(L::B_VFULL + v), (n / L::NV) & 1, wc, 6)) break;
                // the stage's tiles have landed, so the products of row n - NS that read its
                // augmentation blocks are done (the producer waited for them)
                if (!mbar_wait_warp(BAR(L::B_FULL + s), (n / L::NS) & 1, wc, 9)) break;
                const float* vec = reinterpret_cast<const float*>(smem + L::OFF_VEC + v * L::VEC);
                const uint32_t al = sb + s * L::STAGE + L::OFF_AL, ad = sb + s * L::STAGE + L::OFF_AD;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int r = q * 32 + lane;
                    const float lv = vec[r];
                    const float xl = (lv > -3.0e38f) ? lv * inv_c : -3.0e38f;
                    sts128(al + aug_offset(r, 0), split3_bf16(xl));
                    sts128(ad + aug_offset(r, 0), split3_bf16(vec[128 + r]));
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(BAR(L::B_AUG + s));
                    mbar_arrive(BAR(L::B_VEMPTY + v));
                }
            }
        }
    } else if (warp == L::W_MMA) {
        regs_shrink640w();
        const bool leader = elect_one();
        if (!aborted_early) {
            constexpr uint32_t SW = (D == 32) ? SWZ_64B : SWZ_128B;
            constexpr uint32_t SBO = 8 * L::ROWB;
            constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false, false);
            const uint64_t d0 = smem_desc(sb, 16, SBO, SW);
            const uint64_t daug = smem_desc(sb + L::OFF_AL, L::AUG_LBO, L::AUG_SBO, SWZ_NONE);
            const uint64_t dones = smem_desc(sb + L::OFF_ONES, L::AUG_LBO, L::AUG_SBO, SWZ_NONE);
            TRI_TRACE_DECL
            for (int n = 0; n < nrows; ++n) {
                const int s = n % L::NS, x = n & 1;
                TRI_TP(2)
                if (!mbar_wait_warp(BAR(L::B_AUG + s), (n / L::NS) & 1, wc, 2)) break;
                // (the augmentation writer saw this stage's loads land; waiting here too
                // makes the tensor-map writes visible to this thread's MMAs directly)
                if (!mbar_wait_warp(BAR(L::B_FULL + s), (n / L::NS) & 1, wc, 7)) break;
                TRI_TP(0)
                if (n >= 2 && !mbar_wait_warp(BAR(L::B_SDPFREE + x), ((n >> 1) - 1) & 1, wc, 3)) break;
                TRI_TP(1)
                tc_fence_after();
                const uint64_t qd = desc_add(d0, s * L::STAGE);
                const uint64_t ad = desc_add(daug, s * L::STAGE);
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        mma_ss(tmem + x * 256, desc_add(qd, L::OFF_Q + kk * 32), desc_add(qd, L::OFF_K + kk * 32),
                               IDESC_S, kk > 0 ? 1u : 0u);
                        mma_ss(tmem + x * 256 + 128, desc_add(qd, L::OFF_DO + kk * 32),
                               desc_add(qd, L::OFF_V + kk * 32), IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    mma_ss(tmem + x * 256, ad, dones, IDESC_S, 1u);
                    mma_ss(tmem + x * 256 + 128, desc_add(ad, L::AUG_TILE), dones, IDESC_S, 1u);
                    mma_commit(BAR(L::B_SDPFULL + x));
                    mma_commit(BAR(L::B_EMPTY + s));
                }
                __syncwarp();
            }
            TRI_TP(2)
            TRI_TRACE_FLUSH_AT(30000)
            if (leader) mma_commit(BAR(L::B_DRAIN));
            __syncwarp();
            drain_wait(BAR(L::B_DRAIN), 0, 100000000ull);
        }
        __syncwarp();
    } else if (warp >= L::SOFTMAX_WARPS) {
        regs_shrink640w();  // spare warp of the control warpgroup
    } else {
        regs_grow640w();
        if (!aborted_early) {
        const int w = warp >> 2;  // key quarter of the tile
        const int qd = warp & 3;  // TMEM lane quarter = query rows 32qd..32qd+31
        const int row = qd * 32 + lane;
        const uint32_t tl = tmem + (static_cast<uint32_t>(qd * 32) << 16);
        const int j = jt * 128 + row;
        const float c2 = p.scale * LOG2E;
        // this thread's 32 bias values (row j, keys kt*128 + 32w ..), log2 units, kept in
        // registers for the whole row walk (the tile is fixed; S' and dP' are taken from TMEM
        // 16 keys at a time, which leaves room for them)
        float bl[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int k = kt * 128 + w * 32 + e;
            float bv = 0.f;
            if (j < p.N && k < p.N) bv = __bfloat162float(bias[b * bs0 + h * bs1 + static_cast<int64_t>(j) * bs2 + k]);
            bl[e] = bv * LOG2E;
        }
        float acc[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[e] = 0.f;
        bool ok = true;
        TRI_TRACE_DECL
        for (int n = 0; n < nrows; ++n) {
            const int x = n & 1, v = n % L::NV;
            if (!mbar_wait_warp(BAR(L::B_SDPFULL + x), (n >> 1) & 1, wc, 4)) { ok = false; break; }
            TRI_TP(0)
            tc_fence_after();
            if (!mbar_wait_warp(BAR(L::B_VFULL + v), (n / L::NV) & 1, wc, 5)) { ok = false; break; }
            const float* vec = reinterpret_cast<const float*>(smem + L::OFF_VEC + v * L::VEC);
            const bool has_mask = reinterpret_cast<const int*>(vec + 384)[kt] != 0;
            const uint32_t ma = sb + L::OFF_VEC + v * L::VEC + 1024 + w * 128;
            const float2 c22 = make_float2(c2, c2);
            TRI_TP(1)
            // dS = p dP', p = 2^(c S' + bias [+ mask]), summed over rows
            auto row_step = [&](auto masked) {
                constexpr bool kMasked = decltype(masked)::value;
                // S' and dP' of this warpgroup's 32 keys, 16 keys at a time; the columns go back
                // to the MMA warp once the second half is in registers
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t sv[16], dv[16];
                    tmem_ld16(tl + x * 256 + w * 32 + hf * 16, sv);
                    tmem_ld16(tl + x * 256 + 128 + w * 32 + hf * 16, dv);
                    tmem_wait_ld();
                    reg_fence16(sv);
                    reg_fence16(dv);
                    if (hf == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(BAR(L::B_SDPFREE + x));
                    }
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const int cc = 4 * hf + c4;  // 4-key chunk of the thread's 32 keys
                        float2 b01 = make_float2(bl[4 * cc], bl[4 * cc + 1]), b23 = make_float2(bl[4 * cc + 2], bl[4 * cc + 3]);
                        if constexpr (kMasked) {
                            const float4 mq = lds128f(ma + cc * 16);
                            b01 = fadd2(b01, make_float2(mq.x, mq.y));
                            b23 = fadd2(b23, make_float2(mq.z, mq.w));
                        }
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int xh = 4 * c4 + 2 * e;  // within the half
                            const int xl = 4 * cc + 2 * e;  // within the thread's 32 keys
                            const float2 y = ffma2(make_float2(__uint_as_float(sv[xh]), __uint_as_float(sv[xh + 1])),
                                                   c22, e ? b23 : b01);
                            const int pair = (xl >> 1) & 7;  // position of this pair within eight
                            const float2 pv = (!kMasked && pair < FMA_PAIRS) ? ex2_fma2(y)
                                                                             : make_float2(ex2(y.x), ex2(y.y));
                            const float2 a = ffma2(pv, make_float2(__uint_as_float(dv[xh]), __uint_as_float(dv[xh + 1])),
                                                   make_float2(acc[xl], acc[xl + 1]));
                            acc[xl] = a.x;
                            acc[xl + 1] = a.y;
                        }
                    }
                }
            };
            if (has_mask) row_step(std::true_type{});
            else row_step(std::false_type{});
            TRI_TP(2)
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(L::B_VEMPTY + v));
        }
        TRI_TP(3)
        if (ok && j < p.N) {
            const int k0 = kt * 128 + w * 32;
            if (p.chunks == 1 && !p.part_out) {
                __nv_bfloat16* dst = p.dbias + b * p.dbs[0] + h * p.dbs[1] + static_cast<int64_t>(j) * p.dbs[2] + k0;
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    if (k0 + e + 8 <= p.N) {
                        uint4 v;
                        v.x = pack_bf16(acc[e], acc[e + 1]);
                        v.y = pack_bf16(acc[e + 2], acc[e + 3]);
                        v.z = pack_bf16(acc[e + 4], acc[e + 5]);
                        v.w = pack_bf16(acc[e + 6], acc[e + 7]);
                        *reinterpret_cast<uint4*>(dst + e) = v;
                    } else {
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            if (k0 + e + u < p.N) dst[e + u] = __float2bfloat16_rn(acc[e + u]);
                    }
                }
            } else {
                float* dst = p.part + (((static_cast<int64_t>(chunk) * p.B + b) * p.H + h) * p.N + j) * p.N + k0;
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    if (k0 + e < p.N) dst[e] = acc[e];
            }
        }
        TRI_TP(4)
        TRI_TRACE_FLUSH_AT(30000)
    }

    }

    tc_fence_before();
    cta_end_barrier640();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace tri
