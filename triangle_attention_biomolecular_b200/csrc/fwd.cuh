// fwd.cuh -- triangle-attention forward for sm_100a.
//
// Computes, for one batch b, head h, query tile jt (128 queries) and TWO pair
// rows i0, i1 (one per softmax warpgroup):
//   S = Q K^T (tcgen05, BF16 -> FP32 in TMEM), y = scale*S + bias + mask,
//   online softmax over key tiles, O += P V (tcgen05, P from TMEM),
//   epilogue O32 = O / l, o = bf16(O32), resid = bf16(O32 - float(o)),
//   lse = m + log(l).
// The page "16张H100，训练步提速1.73倍：TurboPairFormer…" (biocloudservice.com),
// section "它优化了什么，而不是只'少存一点张量'", describes keeping the BF16
// output-rounding residual for an FP32 softmax-backward correction; the
// residual and the log-sum-exp are the state this kernel saves for the
// backward.
//
// B200 mapping:
//  * one CTA = 384 threads: warps 0-3 softmax for row i0, warps 4-7 softmax
//    for row i1, warp 8 TMA producer, warp 9 issues the PV products, warp 10
//    the S products (so an S never waits in one warp's issue order behind a
//    PV that waits for the other row's probabilities), warp 11 idle; the last
//    warpgroup hands most of its registers to the softmax warpgroups;
//  * both rows share every bias tile (the bias is the same for all rows i),
//    so each 32 KB bias tile crosses L2->SMEM once per two rows;
//  * TMEM (512 columns): per warpgroup w, S at 256w, P (BF16 pairs) at
//    256w+128, O at 256w+192;
//  * O is rescaled lazily: the exponent reference only moves when the row
//    maximum grows by more than 8 (base-2 units), which keeps P <= 256 and
//    makes the TMEM read-modify-write of O rare;
//  * the key tail (k >= N) and the user mask arrive as one FP32 row per key
//    tile, written by the producer warp (-inf past N); an all-zero row is
//    flagged so the add is skipped.
#pragma once

#include <type_traits>

#include "sm100.cuh"

namespace tri {

struct FwdParams {
    int B, N, H, nt, npairs;
    int R;  // rows i this launch covers (N, or a shard of the rows)
    float scale;
    const float* mask;
    int64_t ms0, ms1, ms2;
    __nv_bfloat16* o;
    int64_t os[5];
    __nv_bfloat16* r;
    int64_t rs[5];
    float* lse;
    uint64_t wait_limit_ns;
};

template <int D>
struct FwdLayout {
    static constexpr int NS = (D == 32) ? 3 : 2;  // pipeline stages
    static constexpr int ROWB = D * 2;            // bytes per Q/K/V row
    static constexpr int QKV_TILE = 128 * ROWB;   // one 128-row Q/K/V tile
    static constexpr int BIAS_TILE = 128 * 128 * 2;
    static constexpr int OFF_K0 = 0, OFF_V0 = QKV_TILE, OFF_K1 = 2 * QKV_TILE, OFF_V1 = 3 * QKV_TILE;
    static constexpr int OFF_BIAS = 4 * QKV_TILE;
    static constexpr int OFF_MASK = OFF_BIAS + BIAS_TILE;  // [2][128] fp32
    static constexpr int STAGE = OFF_MASK + 1024;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_STAGES = 2 * QKV_TILE;
    static constexpr int OFF_BAR = OFF_STAGES + NS * STAGE;
    // barrier indices
    static constexpr int B_Q = 0, B_FULL = 1, B_EMPTY = 1 + NS, B_SFULL = 1 + 2 * NS,
                         B_SFREE = B_SFULL + 2, B_PFULL = B_SFREE + 2, B_PVDONE = B_PFULL + 2,
                         B_EXPD = B_PVDONE + 2, B_QFREE = B_EXPD + 2, B_DRAIN = B_QFREE + 1, NBAR = B_DRAIN + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort flag, mask flags[NS][2]
    static constexpr int OFF_TRACE = (OFF_MISC + 16 + NS * 2 * 4 + 7) & ~7;  // phase timing (TRI_TRACE builds only)
    static constexpr int TRACE_BYTES = (OFF_TRACE + kTraceBytes <= 232448) ? kTraceBytes : 0;
    static constexpr int SMEM = OFF_TRACE + TRACE_BYTES;
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(QKV_TILE % 1024 == 0 && STAGE % 1024 == 0, "1 KB tile alignment");
};

__device__ __forceinline__ void reg_fence16(uint32_t (&r)[16]) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
                   "+r"(r[13]), "+r"(r[14]), "+r"(r[15]));
}

__device__ __forceinline__ void reg_fence32(uint32_t (&r)[32]) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
                   "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]),
                   "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]),
                   "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]),
                   "+r"(r[31]));
}

template <int D>
__global__ void __launch_bounds__(384, 1)
    tri_attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_bias,
                        const FwdParams p) {
    using L = FwdLayout<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sb = smem_addr(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto BAR = [&](int idx) -> uint32_t { return sb + L::OFF_BAR + idx * 8; };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
    volatile int* mask_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 16);

    // ---- work items (b, h, pair of rows, query tile), query tile fastest.  The grid is
    // persistent: CTA c takes items c, c + gridDim.x, ..., and every barrier phase runs
    // on counters that continue across items, so the producer fills the next item's Q
    // and first stages while the softmax warps finish the current one. ----
    struct Item {
        int jt, h, b, i0, i1;
        bool has1;
    };
    auto decode = [&](int item) {
        Item t;
        t.jt = item % p.nt;
        item /= p.nt;
        const int ip = item % p.npairs;
        item /= p.npairs;
        t.h = item % p.H;
        t.b = item / p.H;
        t.i0 = 2 * ip;
        t.i1 = min(2 * ip + 1, p.R - 1);
        t.has1 = (2 * ip + 1) < p.R;
        return t;
    };
    const int items = p.B * p.npairs * p.H * p.nt;
    const int nkt = p.nt;

    if (threadIdx.x == 0) {
        *abort_flag = device_error_pending() ? 1 : 0;
        if (sb & 1023u) {  // swizzled TMA tiles need 1 KB alignment
            atomicCAS(&g_error_word, 0u, ERR_TIMEOUT_BIT | KERNEL_FWD | 0xFFu);
            *abort_flag = 1;
        }
        mbar_init(BAR(L::B_Q), 1);
        for (int s = 0; s < L::NS; ++s) {
            mbar_init(BAR(L::B_FULL + s), 1);
            mbar_init(BAR(L::B_EMPTY + s), 1 + 8);  // MMA commit + 8 softmax warps
        }
        for (int w = 0; w < 2; ++w) {
            mbar_init(BAR(L::B_SFULL + w), 1);
            mbar_init(BAR(L::B_SFREE + w), 4);
            mbar_init(BAR(L::B_PFULL + w), 4);
            mbar_init(BAR(L::B_PVDONE + w), 1);
            mbar_init(BAR(L::B_EXPD + w), 4);
        }
        mbar_init(BAR(L::B_QFREE), 1);
        mbar_init(BAR(L::B_DRAIN), 2);  // both MMA-issuing warps
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
    const WaitCtx wc{p.wait_limit_ns, KERNEL_FWD, abort_flag};
    const bool aborted_early = *abort_flag != 0;

    if (warp == 8) {
        // =========================== TMA producer ===========================
        regs_shrink();
        int armed[L::NS];
#pragma unroll
        for (int s = 0; s < L::NS; ++s) armed[s] = 0;
        int nq = 0;  // Q loads issued
        const bool leader = elect_one();
        if (!aborted_early) {
            if (leader) {
                tma_prefetch_map(&tm_q);
                tma_prefetch_map(&tm_k);
                tma_prefetch_map(&tm_v);
                tma_prefetch_map(&tm_bias);
            }
            int gs = 0;  // stage fills so far
            bool ok = true;
            TRI_TRACE_DECL
            for (int item = blockIdx.x; ok && item < items; item += gridDim.x) {
                const Item t = decode(item);
                auto load_qkv = [&](uint32_t dst, const CUtensorMap* m, uint32_t bar, int i, int j0) {
                    tma_load_5d(dst, m, bar, 0, t.h, j0, i, t.b);
                };
                auto load_bias = [&](uint32_t dst, uint32_t bar, int k0, int j0) {
                    tma_load_4d(dst, &tm_bias, bar, k0, j0, t.h, t.b);
                };
                // key-mask rows (user mask, -inf past N) are fetched one stage ahead so
                // their latency overlaps the wait for a free stage
                float mnext[2][4];
                auto fetch_mask = [&](int kt) {
#pragma unroll
                    for (int w = 0; w < 2; ++w) {
                        const int i = w ? t.i1 : t.i0;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int k = kt * 128 + lane * 4 + e;
                            float x = -INFINITY;
                            if (k < p.N) x = p.mask ? __ldg(p.mask + t.b * p.ms0 + i * p.ms1 + k * p.ms2) : 0.f;
                            mnext[w][e] = x;
                        }
                    }
                };
                fetch_mask(0);
                // this item's Q tiles, once the previous item's S products have read the old ones
                if (nq > 0 && !mbar_wait_warp(BAR(L::B_QFREE), (nq - 1) & 1, wc, 13)) { ok = false; break; }
                if (leader) {
                    mbar_arrive_expect_tx(BAR(L::B_Q), 2 * L::QKV_TILE);
                    load_qkv(sb + L::OFF_Q, &tm_q, BAR(L::B_Q), t.i0, t.jt * 128);
                    load_qkv(sb + L::OFF_Q + L::QKV_TILE, &tm_q, BAR(L::B_Q), t.i1, t.jt * 128);
                }
                ++nq;
                for (int kt = 0; kt < nkt; ++kt, ++gs) {
                    const int s = gs % L::NS;
                    TRI_TP(1)
                    if (gs >= L::NS && !mbar_wait_warp(BAR(L::B_EMPTY + s), ((gs / L::NS) - 1) & 1, wc, 1)) {
                        ok = false;
                        break;
                    }
                    TRI_TP(0)
                    const uint32_t st = sb + L::OFF_STAGES + s * L::STAGE;
#pragma unroll
                    for (int w = 0; w < 2; ++w) {
                        bool nz = false;
#pragma unroll
                        for (int e = 0; e < 4; ++e) nz |= (mnext[w][e] != 0.f);
                        float4* dst = reinterpret_cast<float4*>(smem + (st - sb) + L::OFF_MASK + w * 512 + lane * 16);
                        *dst = make_float4(mnext[w][0], mnext[w][1], mnext[w][2], mnext[w][3]);
                        const unsigned any = __any_sync(0xFFFFFFFFu, nz);
                        if (lane == 0) mask_flag[s * 2 + w] = any ? 1 : 0;
                    }
                    __syncwarp();
                    if (leader) {
                        const uint32_t bar = BAR(L::B_FULL + s);
                        mbar_arrive_expect_tx(bar, 4 * L::QKV_TILE + L::BIAS_TILE);
                        load_qkv(st + L::OFF_K0, &tm_k, bar, t.i0, kt * 128);
                        load_qkv(st + L::OFF_V0, &tm_v, bar, t.i0, kt * 128);
                        load_qkv(st + L::OFF_K1, &tm_k, bar, t.i1, kt * 128);
                        load_qkv(st + L::OFF_V1, &tm_v, bar, t.i1, kt * 128);
                        load_bias(st + L::OFF_BIAS, bar, kt * 128, t.jt * 128);
                        load_bias(st + L::OFF_BIAS + L::BIAS_TILE / 2, bar, kt * 128 + 64, t.jt * 128);
                    }
                    armed[s]++;
                    if (kt + 1 < nkt) fetch_mask(kt + 1);
                }
            }
            TRI_TP(1)
            TRI_TRACE_FLUSH_AT(0)
        }
        // never leave with bulk copies still writing into this CTA's shared memory
        if (leader) {
            if (nq > 0) drain_wait(BAR(L::B_Q), (nq - 1) & 1, 100000000ull);
#pragma unroll
            for (int s = 0; s < L::NS; ++s)
                if (armed[s] > 0) drain_wait(BAR(L::B_FULL + s), (armed[s] - 1) & 1, 100000000ull);
        }
    } else if (warp == 9 || warp == 10) {
        // =========================== MMA issuers ============================
        regs_shrink();
        const bool leader = elect_one();
        if (!aborted_early) {
            constexpr uint32_t SW = (D == 32) ? SWZ_64B : SWZ_128B;
            constexpr uint32_t SBO = 8 * L::ROWB;
            constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, false, false);
            constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, false, true);
            // descriptors built once; per-stage / per-step variants are constant adds
            const uint64_t dq0 = smem_desc(sb + L::OFF_Q, 16, SBO, SW);
            const uint64_t dst0 = smem_desc(sb + L::OFF_STAGES, 16, SBO, SW);          // K-major rows
            const uint64_t dvt0 = smem_desc(sb + L::OFF_STAGES, L::QKV_TILE, SBO, SW);  // MN-major rows
            TRI_TRACE_DECL
            bool ok = true;
            int gs = 0, gt = 0, it = 0;  // stages consumed, tiles, items (all continue across items)
            if (warp == 10) {
                // ---- S = Q K^T for both rows of every key tile ----
                for (int item = blockIdx.x; ok && item < items; item += gridDim.x, ++it) {
                    if (!mbar_wait_warp(BAR(L::B_Q), it & 1, wc, 2)) { ok = false; break; }
                    TRI_TP(9)
                    for (int kt = 0; kt < nkt; ++kt, ++gs, ++gt) {
                        const int s = gs % L::NS;
                        TRI_TP(4)
                        if (!mbar_wait_warp(BAR(L::B_FULL + s), (gs / L::NS) & 1, wc, 3)) { ok = false; break; }
                        TRI_TP(0)
                        tc_fence_after();
#pragma unroll
                        for (int w = 0; w < 2; ++w) {
                            if (gt > 0) {
                                TRI_TP(4)
                                if (!mbar_wait_warp(BAR(L::B_SFREE + w), (gt - 1) & 1, wc, 4)) { ok = false; break; }
                                TRI_TP(1)
                                tc_fence_after();
                            }
                            const uint64_t qd = desc_add(dq0, w * L::QKV_TILE);
                            const uint64_t kd = desc_add(dst0, s * L::STAGE + (w ? L::OFF_K1 : L::OFF_K0));
                            if (leader) {
#pragma unroll
                                for (int kk = 0; kk < D / 16; ++kk)
                                    mma_ss(tmem + w * 256, desc_add(qd, kk * 32), desc_add(kd, kk * 32), IDESC_QK,
                                           kk > 0 ? 1u : 0u);
                                mma_commit(BAR(L::B_SFULL + w));
                            }
                            __syncwarp();
                        }
                        if (!ok) break;
                        if (kt == nkt - 1) {  // the item's last S products: Q is free once they finish
                            if (leader) mma_commit(BAR(L::B_QFREE));
                            __syncwarp();
                        }
                    }
                }
            } else {
                // ---- O += P V for both rows of every key tile; the stage (K, V, bias, mask) goes
                // back to the producer after them (its S products completed before the
                // probabilities they gave were written) ----
                for (int item = blockIdx.x; ok && item < items; item += gridDim.x, ++it) {
                    for (int kt = 0; kt < nkt; ++kt, ++gs, ++gt) {
                        const int s = gs % L::NS;
                        const uint64_t vbase = desc_add(dvt0, s * L::STAGE);
#pragma unroll
                        for (int w = 0; w < 2; ++w) {
                            TRI_TP(4)
                            if (!mbar_wait_warp(BAR(L::B_PFULL + w), gt & 1, wc, 5)) { ok = false; break; }
                            TRI_TP(2)
                            tc_fence_after();
                            const uint64_t vd = desc_add(vbase, w ? L::OFF_V1 : L::OFF_V0);
                            const uint32_t tS = tmem + w * 256;
                            if (leader) {
#pragma unroll
                                for (int kk = 0; kk < 8; ++kk)
                                    mma_ts(tS + 192, tS + 128 + kk * 8, desc_add(vd, kk * 16 * L::ROWB), IDESC_PV,
                                           (kt > 0 || kk > 0) ? 1u : 0u);
                                mma_commit(BAR(L::B_PVDONE + w));
                            }
                            __syncwarp();
                        }
                        if (!ok) break;
                        if (leader) mma_commit(BAR(L::B_EMPTY + s));
                        __syncwarp();
                    }
                }
            }
            TRI_TP(5)
            TRI_TRACE_FLUSH_AT(0)
            // every MMA the leader issued has completed before the CTA leaves
            if (leader) mma_commit(BAR(L::B_DRAIN));
            __syncwarp();
            drain_wait(BAR(L::B_DRAIN), 0, 100000000ull);
        }
        __syncwarp();
    } else if (warp >= 11) {
        regs_shrink();  // spare warp of the last warpgroup
    } else {
        regs_grow();
        if (!aborted_early) {
        // =========================== softmax warpgroups =====================
        const int w = warp >> 2;
        const int qd = warp & 3;
        const int row = qd * 32 + lane;
        const uint32_t tS = tmem + (static_cast<uint32_t>(qd * 32) << 16) + w * 256;
        const uint32_t tP = tS + 128, tO = tS + 192;
        const float scale = p.scale;
        constexpr float LOG2E = 1.4426950408889634f;
        constexpr float RESCALE_AT = 5.545177444479562f;  // 8 * ln 2
        bool ok = true;
        int gs = 0, gt = 0;  // stages and tiles consumed, continuing across items
        TRI_TRACE_DECL
        for (int item = blockIdx.x; ok && item < items; item += gridDim.x) {
        const Item t = decode(item);
        const int j = t.jt * 128 + row;
        const int i = w ? t.i1 : t.i0;
        const int b = t.b, h = t.h;
        float m_ref = -INFINITY, l = 0.f;
        for (int kt = 0; kt < nkt; ++kt, ++gs, ++gt) {
            const int s = gs % L::NS;
            if (!mbar_wait_warp(BAR(L::B_SFULL + w), gt & 1, wc, 6)) { ok = false; break; }
            if (kt == 0) { TRI_TP(9) } else { TRI_TP(0) }
            tc_fence_after();
            uint32_t r0[32], r1[32], r2[32], r3[32];
            tmem_ld32(tS + 0, r0);
            tmem_ld32(tS + 32, r1);
            tmem_ld32(tS + 64, r2);
            tmem_ld32(tS + 96, r3);
            tmem_wait_ld();
            reg_fence32(r0);
            reg_fence32(r1);
            reg_fence32(r2);
            reg_fence32(r3);
            TRI_TP(1)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(L::B_SFREE + w));
            if (!mbar_wait_warp(BAR(L::B_FULL + s), (gs / L::NS) & 1, wc, 7)) { ok = false; break; }
            TRI_TP(2)
            const uint32_t st = sb + L::OFF_STAGES + s * L::STAGE;
            float x[128];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                x[e] = __uint_as_float(r0[e]);
                x[32 + e] = __uint_as_float(r1[e]);
                x[64 + e] = __uint_as_float(r2[e]);
                x[96 + e] = __uint_as_float(r3[e]);
            }
            // y = scale * S + bias (+ mask), two lanes per instruction
            const uint32_t brow = st + L::OFF_BIAS + row * 128;
            const float2 sc2 = make_float2(scale, scale);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const uint4 bb = lds128(brow + (c >> 3) * (L::BIAS_TILE / 2) + (((c & 7) ^ (row & 7)) << 4));
                const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int x0 = c * 8 + 2 * e;
                    const float2 y = ffma2(make_float2(x[x0], x[x0 + 1]), sc2, bf16x2_to_f2(bw[e]));
                    x[x0] = y.x;
                    x[x0 + 1] = y.y;
                }
            }
            const bool tile_masked = mask_flag[s * 2 + w] != 0;
            if (tile_masked) {
                const uint32_t ma = st + L::OFF_MASK + w * 512;
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const float4 mv = lds128f(ma + c * 16);
                    const float2 y0 = fadd2(make_float2(x[4 * c], x[4 * c + 1]), make_float2(mv.x, mv.y));
                    const float2 y1 = fadd2(make_float2(x[4 * c + 2], x[4 * c + 3]), make_float2(mv.z, mv.w));
                    x[4 * c] = y0.x;
                    x[4 * c + 1] = y0.y;
                    x[4 * c + 2] = y1.x;
                    x[4 * c + 3] = y1.y;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(L::B_EMPTY + s));
            // row maximum: four independent chains of three-input maxima over x[4..123],
            // then the last four scores
            float ma0 = x[0], ma1 = x[1], ma2 = x[2], ma3 = x[3];
#pragma unroll
            for (int e = 4; e < 124; e += 8) {
                ma0 = fmax3(ma0, x[e], x[e + 1]);
                ma1 = fmax3(ma1, x[e + 2], x[e + 3]);
                ma2 = fmax3(ma2, x[e + 4], x[e + 5]);
                ma3 = fmax3(ma3, x[e + 6], x[e + 7]);
            }
            const float mt = fmaxf(fmaxf(fmaxf(ma0, x[124]), fmaxf(ma1, x[125])),
                                   fmaxf(fmaxf(ma2, x[126]), fmaxf(ma3, x[127])));
            TRI_TP(3)
            bool need = false;
            float alpha = 1.f;
            if (kt == 0) {
                m_ref = mt;
            } else if (mt > m_ref + RESCALE_AT) {
                need = true;
                alpha = ex2((m_ref - mt) * LOG2E);
                m_ref = mt;
                l *= alpha;
            }
            const float mb = fmaxf(m_ref, -3.0e38f) * LOG2E;
            // Ping-pong on the exponential unit: the two warpgroups take turns
            // (WG0 tile kt, WG1 tile kt, WG0 tile kt+1, ...), so one runs its
            // exponentials while the other loads, biases and reduces its next tile.
            if (w == 1 || gt > 0) {
                const int turn = w == 1 ? gt : gt - 1;
                if (!mbar_wait_warp(BAR(L::B_EXPD + (1 - w)), turn & 1, wc, 10)) { ok = false; break; }
            }
            TRI_TP(6)
            // probabilities into packed BF16 registers first; the previous PV may still be
            // reading the P columns
            const float2 l2e = make_float2(LOG2E, LOG2E), nmb = make_float2(-mb, -mb);
            float2 ls0 = make_float2(0.f, 0.f), ls1 = ls0, ls2 = ls0, ls3 = ls0;
            uint32_t pk[64];
            // in key tiles without a mask, one pair in four takes the FMA-pipe exponential
            auto exps = [&](auto mixed) {
                constexpr bool kMixed = decltype(mixed)::value;
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const float2 a2 = ffma2(make_float2(x[2 * c], x[2 * c + 1]), l2e, nmb);
                    const float2 pp = (kMixed && (c & 3) == 3) ? ex2_fma2(a2) : make_float2(ex2(a2.x), ex2(a2.y));
                    switch (c & 3) {
                        case 0: ls0 = fadd2(ls0, pp); break;
                        case 1: ls1 = fadd2(ls1, pp); break;
                        case 2: ls2 = fadd2(ls2, pp); break;
                        default: ls3 = fadd2(ls3, pp); break;
                    }
                    pk[c] = pack_bf16(pp.x, pp.y);
                }
            };
            if (tile_masked) exps(std::false_type{});
            else exps(std::true_type{});
            const float2 lsum = fadd2(fadd2(ls0, ls1), fadd2(ls2, ls3));
            const float ls = lsum.x + lsum.y;
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(L::B_EXPD + w));
            TRI_TP(5)
            if (kt > 0) {
                // PV of the previous tile has finished: the P columns are free and O is stable
                if (!mbar_wait_warp(BAR(L::B_PVDONE + w), (gt - 1) & 1, wc, 8)) { ok = false; break; }
                tc_fence_after();
            }
            TRI_TP(4)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t pq[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) pq[c] = pk[16 * q + c];
                tmem_st16(tP + 16 * q, pq);
            }
            l += ls;
            if (kt > 0 && __any_sync(0xFFFFFFFFu, need)) {
                // rare: the reference maximum moved, rescale this row of O before the next PV
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(tO + c0, o);
                    tmem_wait_ld();
                    reg_fence32(o);
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(tO + c0, o);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(L::B_PFULL + w));
            TRI_TP(7)
        }
        if (!ok) break;
        if (!mbar_wait_warp(BAR(L::B_PVDONE + w), (gt - 1) & 1, wc, 9)) { ok = false; break; }
        TRI_TP(10)
        {
            tc_fence_after();
            const bool store = (j < p.N) && (w == 0 || t.has1);
            const float inv_l = __frcp_rn(l);
            __nv_bfloat16* op = p.o + b * p.os[0] + i * p.os[1] + j * p.os[2] + h * p.os[3];
            __nv_bfloat16* rp = p.r + b * p.rs[0] + i * p.rs[1] + j * p.rs[2] + h * p.rs[3];
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t o[32];
                tmem_ld32(tO + c0, o);
                tmem_wait_ld();
                reg_fence32(o);
                if (store) {
                    // 32 columns -> 16 packed words each of o and resid; one 32-byte store per
                    // 16 columns where the row start allows it (a warp's rows are H*d*2 bytes
                    // apart, so 16-byte stores would fill half a sector each)
                    const bool v8 = ((reinterpret_cast<uintptr_t>(op + c0) | reinterpret_cast<uintptr_t>(rp + c0)) & 31u) == 0;
#pragma unroll
                    for (int c = 0; c < 4; c += 2) {
                        uint32_t ow[8], rw[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float a0 = __uint_as_float(o[8 * c + 2 * e]) * inv_l;
                            const float a1 = __uint_as_float(o[8 * c + 2 * e + 1]) * inv_l;
                            const uint32_t w16 = pack_bf16(a0, a1);
                            ow[e] = w16;
                            rw[e] = pack_bf16(a0 - bf16lo(w16), a1 - bf16hi(w16));
                        }
                        if (v8) {
                            st_global_v8(op + c0 + 8 * c, ow);
                            st_global_v8(rp + c0 + 8 * c, rw);
                        } else {
                            *reinterpret_cast<uint4*>(op + c0 + 8 * c) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                            *reinterpret_cast<uint4*>(op + c0 + 8 * c + 8) = make_uint4(ow[4], ow[5], ow[6], ow[7]);
                            *reinterpret_cast<uint4*>(rp + c0 + 8 * c) = make_uint4(rw[0], rw[1], rw[2], rw[3]);
                            *reinterpret_cast<uint4*>(rp + c0 + 8 * c + 8) = make_uint4(rw[4], rw[5], rw[6], rw[7]);
                        }
                    }
                }
            }
            if (store) {
                p.lse[((static_cast<int64_t>(b) * p.H + h) * p.R + i) * p.N + j] =
                    m_ref + lg2(l) * 0.6931471805599453f;
            }
        }
        TRI_TP(11)
        }  // items
        TRI_TP(8)
        TRI_TRACE_FLUSH_AT(0)
    }

    }

    tc_fence_before();
    cta_end_barrier();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace tri
