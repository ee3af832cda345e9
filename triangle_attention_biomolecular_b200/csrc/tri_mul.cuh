// tri_mul.cuh -- the contraction step of the triangle multiplicative update, sm_100a.
//
// The pages name the Triangle Multiplicative Update as the second operation
// TurboPairFormer optimises beside triangle attention ("16张H100，训练步提速
// 1.73倍：TurboPairFormer…", biocloudservice.com, opening paragraph), without a
// formula.  Its cubic step, read the AlphaFold way, contracts two projected
// pair tensors over the third residue k, channel by channel:
//   outgoing edges  x[b,c,i,j] = sum_k a[b,c,i,k] b[b,c,j,k]
//   incoming edges  x[b,c,i,j] = sum_k a[b,c,k,i] b[b,c,k,j]
// Forward and backward are six batched products of N x N matrices, which
// this file computes with one tcgen05 GEMM:
//   out[z][m][n] = sum_k A_z(m, k) B_z(n, k)      (z = one (batch, channel))
// where each operand is read either K-major (k contiguous in memory) or
// MN-major (m or n contiguous), so every transpose is absorbed by the TMA
// box and the shared-memory descriptor rather than by a copy.
//
// B200 mapping:
//  * a persistent CTA per SM, 192 threads: warps 0-3 epilogue (one TMEM lane
//    quarter each), warp 4 TMA producer, warp 5 MMA issuer; it walks 128 x 256
//    output tiles with the n tile fastest, so concurrent CTAs share operand
//    panels in L2;
//  * K advances 64 at a time through a four-stage TMA ring (A 16 KB + B 32 KB
//    per stage, 128-byte swizzle); four M128 N256 K16 MMAs per stage accumulate
//    into one of two 256-column TMEM accumulators, so the epilogue (TMEM ->
//    BF16 -> global) of one tile overlaps the MMAs of the next;
//  * residue counts that are not multiples of the tile are handled by the TMA
//    zero fill (the contraction over padded k adds zeros) and guarded stores.
#pragma once

#include "sm100.cuh"

namespace tri {

struct TriMulGemmParams {
    int N, C, Z;                // residues, channels, batch x channels (z = b * C + c)
    __nv_bfloat16* out;         // [B, C, N, N]
    int64_t os[4];              // element strides of (b, c, m, n)
    uint64_t wait_limit_ns;
};

struct TriMulLayout {
    static constexpr int BM = 128, BN = 256, BK = 64;
    static constexpr int NS = 4;
    static constexpr int A_TILE = BM * BK * 2;  // 16 KB
    static constexpr int B_TILE = BN * BK * 2;  // 32 KB
    static constexpr int STAGE = A_TILE + B_TILE;
    static constexpr int OFF_BAR = NS * STAGE;
    static constexpr int B_FULL = 0, B_EMPTY = NS, B_ACCF = 2 * NS, B_ACCE = 2 * NS + 2, B_DRAIN = 2 * NS + 4,
                         NBAR = 2 * NS + 5;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort flag
    static constexpr int SMEM = OFF_MISC + 16 + 1024;    // + slack for 1 KB alignment
    static constexpr int THREADS = 192;
    static constexpr uint32_t TMEM_COLS = 512;  // two 256-column accumulators
};

// A_MN / B_MN: the operand is stored with m (or n) contiguous; otherwise with k
// contiguous.  Tensor maps are 4-D (inner, outer, c, b).  K-major maps use a box of
// 64 k x rows; MN-major maps a box of 64 rows x 64 k, loaded once per 64 rows.
// Persistent: CTA c computes tiles c, c + gridDim.x, ... in (z, m, n) order with n
// fastest; the stage ring and the two accumulators run on counters that continue
// across tiles, so one tile's epilogue overlaps the next tile's loads and MMAs.
template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(192, 1)
    tri_mul_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                        const TriMulGemmParams p) {
    using L = TriMulLayout;
    extern __shared__ uint8_t smem_raw[];
    // 1 KB alignment for the swizzled tiles
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sb - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto BAR = [&](int idx) -> uint32_t { return sb + L::OFF_BAR + idx * 8; };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

    const int tm = (p.N + L::BM - 1) / L::BM, tn = (p.N + L::BN - 1) / L::BN;
    const int tiles = tm * tn * p.Z;
    const int nk = (p.N + L::BK - 1) / L::BK;
    struct Tile {
        int m0, n0, c, b;
    };
    auto decode = [&](int t) {
        Tile r;
        r.n0 = (t % tn) * L::BN;
        t /= tn;
        r.m0 = (t % tm) * L::BM;
        t /= tm;
        r.c = t % p.C;
        r.b = t / p.C;
        return r;
    };

    if (threadIdx.x == 0) {
        *abort_flag = device_error_pending() ? 1 : 0;
        for (int s = 0; s < L::NS; ++s) {
            mbar_init(BAR(L::B_FULL + s), 1);
            mbar_init(BAR(L::B_EMPTY + s), 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(BAR(L::B_ACCF + x), 1);  // MMA commit: accumulator x complete
            mbar_init(BAR(L::B_ACCE + x), 4);  // the four epilogue warps have read it
        }
        mbar_init(BAR(L::B_DRAIN), 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(const_cast<uint32_t*>(tmem_slot)), L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtx wc{p.wait_limit_ns, KERNEL_TRIMUL, abort_flag};
    const bool aborted_early = *abort_flag != 0;

    if (warp == 4) {
        // =========================== TMA producer ===========================
        const bool leader = elect_one();
        int armed[L::NS] = {};
        if (!aborted_early) {
            if (leader) {
                tma_prefetch_map(&tm_a);
                tma_prefetch_map(&tm_b);
            }
            int gs = 0;  // stage fills
            bool ok = true;
            for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
                const Tile T = decode(t);
                for (int kb = 0; kb < nk; ++kb, ++gs) {
                    const int s = gs % L::NS;
                    if (gs >= L::NS && !mbar_wait_warp(BAR(L::B_EMPTY + s), ((gs / L::NS) - 1) & 1, wc, 1)) {
                        ok = false;
                        break;
                    }
                    if (leader) {
                        const uint32_t bar = BAR(L::B_FULL + s);
                        const uint32_t da = sb + s * L::STAGE, db = da + L::A_TILE;
                        const int k0 = kb * L::BK;
                        mbar_arrive_expect_tx(bar, L::STAGE);
                        if constexpr (A_MN) {
#pragma unroll
                            for (int r = 0; r < L::BM / 64; ++r)
                                tma_load_4d(da + r * 8192, &tm_a, bar, T.m0 + 64 * r, k0, T.c, T.b);
                        } else {
                            tma_load_4d(da, &tm_a, bar, k0, T.m0, T.c, T.b);
                        }
                        if constexpr (B_MN) {
#pragma unroll
                            for (int r = 0; r < L::BN / 64; ++r)
                                tma_load_4d(db + r * 8192, &tm_b, bar, T.n0 + 64 * r, k0, T.c, T.b);
                        } else {
                            tma_load_4d(db, &tm_b, bar, k0, T.n0, T.c, T.b);
                        }
                    }
                    armed[s]++;
                }
            }
        }
        if (leader) {
#pragma unroll
            for (int s = 0; s < L::NS; ++s)
                if (armed[s] > 0) drain_wait(BAR(L::B_FULL + s), (armed[s] - 1) & 1, 100000000ull);
        }
    } else if (warp == 5) {
        // =========================== MMA issuer =============================
        const bool leader = elect_one();
        if (!aborted_early) {
            constexpr uint32_t IDESC = idesc_bf16_f32(L::BM, L::BN, A_MN, B_MN);
            // K-major, 128-byte swizzle: rows of 128 B, 8-row groups 1 KB apart; a K=16
            // step moves 32 B along the row.  MN-major: 64-element chunks 8 KB apart
            // (LBO), 8-k-row groups 1 KB apart (SBO); a K=16 step moves 2 KB.
            const uint64_t a0 = A_MN ? smem_desc(sb, 8192, 1024, SWZ_128B) : smem_desc(sb, 16, 1024, SWZ_128B);
            const uint64_t b0 =
                B_MN ? smem_desc(sb + L::A_TILE, 8192, 1024, SWZ_128B) : smem_desc(sb + L::A_TILE, 16, 1024, SWZ_128B);
            bool ok = true;
            int gs = 0, lt = 0;  // stages consumed, tiles of this CTA
            for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++lt) {
                const int x = lt & 1;
                // the epilogue has read what this accumulator held two tiles ago
                if (lt >= 2 && !mbar_wait_warp(BAR(L::B_ACCE + x), ((lt >> 1) - 1) & 1, wc, 4)) { ok = false; break; }
                tc_fence_after();
                for (int kb = 0; kb < nk; ++kb, ++gs) {
                    const int s = gs % L::NS;
                    if (!mbar_wait_warp(BAR(L::B_FULL + s), (gs / L::NS) & 1, wc, 2)) { ok = false; break; }
                    tc_fence_after();
                    if (leader) {
#pragma unroll
                        for (int kk = 0; kk < L::BK / 16; ++kk) {
                            const uint32_t ao = s * L::STAGE + (A_MN ? kk * 2048 : kk * 32);
                            const uint32_t bo = s * L::STAGE + (B_MN ? kk * 2048 : kk * 32);
                            mma_ss(tmem + x * 256, desc_add(a0, ao), desc_add(b0, bo), IDESC,
                                   (kb > 0 || kk > 0) ? 1u : 0u);
                        }
                        mma_commit(BAR(L::B_EMPTY + s));
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (leader) mma_commit(BAR(L::B_ACCF + x));
                __syncwarp();
            }
            // no MMA in flight when TMEM is freed (the commit tracks every MMA issued)
            if (leader) {
                mma_commit(BAR(L::B_DRAIN));
                drain_wait(BAR(L::B_DRAIN), 0, 100000000ull);
            }
            __syncwarp();
            (void)ok;
        }
    } else {
        // =========================== epilogue (warps 0-3) ====================
        if (!aborted_early) {
            const int row = warp * 32 + lane;
            int lt = 0;
            for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
                const int x = lt & 1;
                if (!mbar_wait_warp(BAR(L::B_ACCF + x), (lt >> 1) & 1, wc, 3)) break;
                tc_fence_after();
                const Tile T = decode(t);
                const int m = T.m0 + row;
                const uint32_t tl = tmem + (static_cast<uint32_t>(warp * 32) << 16) + x * 256;
                __nv_bfloat16* dst = p.out + T.b * p.os[0] + T.c * p.os[1] + static_cast<int64_t>(m) * p.os[2] + T.n0;
                const bool full_n = T.n0 + L::BN <= p.N;
#pragma unroll 1
                for (int c0 = 0; c0 < L::BN; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld32(tl + c0, v);
                    tmem_wait_ld();
                    if (c0 == L::BN - 32) {  // every column read: hand the accumulator back
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(BAR(L::B_ACCE + x));
                    }
                    if (m < p.N) {
                        if (full_n) {
#pragma unroll
                            for (int e = 0; e < 32; e += 8) {
                                uint4 q;
                                q.x = pack_bf16(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                                q.y = pack_bf16(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                                q.z = pack_bf16(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]));
                                q.w = pack_bf16(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7]));
                                *reinterpret_cast<uint4*>(dst + c0 + e) = q;
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (T.n0 + c0 + e < p.N) dst[c0 + e] = __float2bfloat16_rn(__uint_as_float(v[e]));
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

}  // namespace tri
