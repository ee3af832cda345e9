// bwd.cuh -- triangle-attention backward for sm_100a.
//
// Pages: "TurboPairFormer: более быстрое, стабильное и точное дообучение
// OpenFold3" (dev48.org), section "Как работает TurboPairFormer" (probability
// tiles recomputed in the backward; BF16 output-rounding residual used for
// the gradients; fixed accumulation order for bitwise-repeatable gradients),
// and "16张H100，训练步提速1.73倍：TurboPairFormer…" (biocloudservice.com),
// section "它优化了什么": the correction term is formed in FP32 from the saved
// residual; no floating-point atomics.
//
// Three reductions meet in this backward: dK/dV sum over queries j, dQ sums
// over keys k, and dBias sums over pair rows i (the bias is shared by every
// row).  A CTA cannot keep accumulators for all three on chip at N=768 (TMEM
// holds 128 x 512 FP32), so the work is split:
//
//  1. tri_attn_bwd_prep_kernel: D[b,h,i,j] = sum_c dout * (o + resid), FP32, and
//     the padded per-row vectors; tri_attn_bwd_bias_tiles_kernel: the pair bias
//     copied into the main kernel's read order (one 32 KB block per tile).
//  2. tri_attn_bwd_main_kernel (problem-stationary): one persistent CTA walks
//     whole problems (b,i,h): key tiles kt outer, query tiles jt inner.  Per
//     tile it recomputes S and dP with tcgen05, forms P and dS once, stages
//     them in SMEM (BF16, 128B-swizzled) and issues dV += P^T dO,
//     dK += dS^T Q, dQ_tile = dS K (S/dP and the gradient products from two
//     warps).  dK/dV finish in TMEM per key tile; dQ stays in TMEM for every
//     query tile when the columns allow (N <= 768 at d=32), else it
//     accumulates over key tiles in a per-CTA FP32 slot of the workspace, in
//     ascending kt order, by the same thread each time.
//  3. tri_attn_bwd_dbias_kernel (tile-stationary): one CTA per (b,h,jt,kt)
//     and row chunk walks i in ascending order, recomputes S, dP -> dS and
//     accumulates dBias in FP32 registers.  Chunks (only when there are
//     fewer tiles than SMs) are summed in ascending chunk order by
//     tri_attn_bwd_dbias_reduce_kernel.
// Every reduction therefore has one fixed order: results are bitwise
// repeatable and independent of the SM count.
#pragma once

#include <type_traits>

#include "../../include/tri_attn.h"
#include "sm100.cuh"
#include "fwd.cuh"

namespace tri {

constexpr int kDqSlots = 148;   // persistent CTAs of the main kernel (B200 SM count)
constexpr int kChunkTarget = 148;

struct BwdWorkspace {
    size_t off_D, off_L, off_M, off_F, off_dq, off_BT, off_part, total;
    int chunks;     // row chunks of the dBias kernel
    int grid_main;  // CTAs of the main kernel
    int Np;         // N rounded up to whole 128-wide tiles
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// R: rows i the launch covers (N for the whole problem, fewer for a row shard)
inline BwdWorkspace bwd_workspace_layout(int B, int R, int N, int H, int d) {
    BwdWorkspace w{};
    const size_t nt = (N + 127) / 128;
    const size_t tiles = static_cast<size_t>(B) * H * nt * nt;
    int chunks = 1;
    if (tiles < static_cast<size_t>(kChunkTarget)) {
        chunks = static_cast<int>(kChunkTarget / tiles);
        chunks = chunks < 1 ? 1 : chunks;
        const int max_chunks = (R + 7) / 8;  // at least 8 rows per chunk
        chunks = chunks > max_chunks ? max_chunks : chunks;
    }
    w.chunks = chunks;
    w.Np = static_cast<int>(nt * 128);
    const size_t problems = static_cast<size_t>(B) * R * H;
    w.grid_main = static_cast<int>(problems < static_cast<size_t>(kDqSlots) ? problems : kDqSlots);
    const size_t bhnp = static_cast<size_t>(B) * H * R * w.Np;
    const size_t bnp = static_cast<size_t>(B) * R * w.Np;
    w.off_D = 0;
    w.off_L = align256(bhnp * 4);
    w.off_M = w.off_L + align256(bhnp * 4);
    w.off_F = w.off_M + align256(bnp * 4);
    w.off_dq = w.off_F + align256(static_cast<size_t>(B) * R * 32 * 4);
    w.off_BT = w.off_dq + align256(static_cast<size_t>(kDqSlots) * N * d * 4);
    w.off_part = w.off_BT + align256(static_cast<size_t>(B) * H * w.Np * w.Np * 2);
    const size_t bhnn = static_cast<size_t>(B) * H * N * N;
    w.total = w.off_part + (chunks > 1 ? align256(static_cast<size_t>(chunks) * bhnn * 4) : 0);
    return w;
}

struct BwdParams {
    int B, N, H, nt, Np;
    int R;            // rows i this launch covers (N, or a shard of the rows)
    float scale;
    const float* Lv;  // [B,H,R,Np] -lse * log2(e); -inf past N
    const float* Dv;  // [B,H,R,Np] -D; 0 past N
    const float* Mv;  // [B,R,Np]   mask * log2(e); -inf past N
    const int* Fv;    // [B,R,32]   1 where a key tile needs the mask add
    const __nv_bfloat16* bias;  // [B,H,N,N] as given (the dBias pass reads it)
    int64_t bs0, bs1, bs2;
    const uint4* bias_tiles;    // [B,H,nt,nt][32 KB] the bias in main-kernel read order (pre-pass 1b)
    float* dq_slots;  // [kDqSlots][N][d] (used when dq_tmem == 0)
    int dq_tmem;      // 1: dQ for every query tile stays in TMEM across key tiles
    float* part;      // [chunks][B,H,N,N] (chunks > 1, or always when part_out)
    int chunks;
    int part_out;     // 1: dBias leaves as FP32 partial sums in part, never as BF16
    __nv_bfloat16 *dq, *dk, *dv, *dbias;
    int64_t dqs[5], dks[5], dvs[5], dbs[4];
    uint64_t wait_limit_ns;
};

// ===========================================================================
// 1. pre-pass: the per-row vectors both backward kernels stream, laid out so
//    that every 128-wide tile is one aligned 512-byte bulk copy:
//      ND = -rowsum(dout * (o + resid))  (FP32; the residual restores what BF16
//           rounding of the output dropped), 0 past N
//      NL = -lse * log2(e), -inf past N (so padded query rows get P = 0)
//      (both negated: the kernels add them)
//      M  = mask * log2(e) (0 without a mask), -inf past N (padded keys)
//      F  = per (b, i, key tile): 1 if that tile needs the mask add at all
// ===========================================================================
template <int D>
__global__ void __launch_bounds__(256) tri_attn_bwd_prep_kernel(
    const __nv_bfloat16* __restrict__ dout, int64_t s0, int64_t s1, int64_t s2, int64_t s3,
    const __nv_bfloat16* __restrict__ o, int64_t o0, int64_t o1, int64_t o2, int64_t o3,
    const __nv_bfloat16* __restrict__ r, int64_t r0, int64_t r1, int64_t r2, int64_t r3, int use_resid,
    const float* __restrict__ lse, const float* __restrict__ mask, int64_t m0, int64_t m1, int64_t m2,
    float* __restrict__ Dv, float* __restrict__ Lv, float* __restrict__ Mv, int* __restrict__ Fv, int B, int N,
    int R, int H, int Np, int nt) {
    constexpr float LOG2E = 1.4426950408889634f;
    const int lane = threadIdx.x & 31;
    const int64_t n1 = static_cast<int64_t>(B) * H * R * Np;
    const int64_t n2 = static_cast<int64_t>(B) * R * Np;
    const int64_t n3 = static_cast<int64_t>(B) * R * 32;
    // F first, one warp per (b, i, key tile): the warp reads the tile's 128 mask values in
    // one round (four per lane, coalesced along k) and votes, so no thread walks a tile
    // alone while the rest of the grid streams.
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); e < n3;
         e += nwarps) {
        const int kt = static_cast<int>(e & 31);
        const int64_t t = e >> 5;
        const int i = static_cast<int>(t % R);
        const int b = static_cast<int>(t / R);
        int f = 0;
        if (kt < nt) {
            if ((kt + 1) * 128 > N) {
                f = 1;  // padded keys need the -inf
            } else if (mask) {
                const float* mr = mask + b * m0 + i * m1 + static_cast<int64_t>(kt * 128 + lane) * m2;
                const float a0 = __ldg(mr), a1 = __ldg(mr + 32 * m2), a2 = __ldg(mr + 64 * m2),
                            a3 = __ldg(mr + 96 * m2);
                f = __any_sync(0xffffffffu, a0 != 0.f || a1 != 0.f || a2 != 0.f || a3 != 0.f) ? 1 : 0;
            }
        }
        if (lane == 0) Fv[e] = f;
    }
    // D, L (head fastest) and then M; the index decode runs in 32-bit arithmetic whenever
    // the item count allows (three 64-bit divisions per item cost more issue slots than
    // the item's loads)
    const bool small = n1 + n2 <= static_cast<int64_t>(0xffffffffu);
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < n1 + n2;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        if (idx < n1) {
            // head fastest: neighbouring threads read the heads of one pair row, which are
            // contiguous in memory, so a warp streams whole 256-byte rows
            int h, j, i, b;
            if (small) {
                uint32_t t = static_cast<uint32_t>(idx);
                h = static_cast<int>(t % static_cast<uint32_t>(H));
                t /= static_cast<uint32_t>(H);
                j = static_cast<int>(t % static_cast<uint32_t>(Np));
                t /= static_cast<uint32_t>(Np);
                i = static_cast<int>(t % static_cast<uint32_t>(R));
                b = static_cast<int>(t / static_cast<uint32_t>(R));
            } else {
                int64_t t = idx;
                h = static_cast<int>(t % H);
                t /= H;
                j = static_cast<int>(t % Np);
                t /= Np;
                i = static_cast<int>(t % R);
                b = static_cast<int>(t / R);
            }
            const int64_t out = ((static_cast<int64_t>(b) * H + h) * R + i) * Np + j;
            float dsum = 0.f, lv = -INFINITY;
            if (j < N) {
                const uint4* pd = reinterpret_cast<const uint4*>(dout + b * s0 + i * s1 + j * s2 + h * s3);
                const uint4* po = reinterpret_cast<const uint4*>(o + b * o0 + i * o1 + j * o2 + h * o3);
                const uint4* pr = reinterpret_cast<const uint4*>(r + b * r0 + i * r1 + j * r2 + h * r3);
#pragma unroll
                for (int c = 0; c < D / 8; ++c) {
                    const uint4 a = __ldg(pd + c), bo = __ldg(po + c);
                    uint4 br = make_uint4(0, 0, 0, 0);
                    if (use_resid) br = __ldg(pr + c);
                    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, ow[4] = {bo.x, bo.y, bo.z, bo.w},
                                   rw[4] = {br.x, br.y, br.z, br.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        dsum = fmaf(bf16lo(aw[e]), bf16lo(ow[e]) + bf16lo(rw[e]), dsum);
                        dsum = fmaf(bf16hi(aw[e]), bf16hi(ow[e]) + bf16hi(rw[e]), dsum);
                    }
                }
                lv = -(__ldg(lse + ((static_cast<int64_t>(b) * H + h) * R + i) * N + j) * LOG2E);
            }
            Dv[out] = -dsum;
            Lv[out] = lv;
        } else {
            const int64_t e = idx - n1;
            int k, i, b;
            if (small) {
                uint32_t t = static_cast<uint32_t>(e);
                k = static_cast<int>(t % static_cast<uint32_t>(Np));
                t /= static_cast<uint32_t>(Np);
                i = static_cast<int>(t % static_cast<uint32_t>(R));
                b = static_cast<int>(t / static_cast<uint32_t>(R));
            } else {
                k = static_cast<int>(e % Np);
                const int64_t t = e / Np;
                i = static_cast<int>(t % R);
                b = static_cast<int>(t / R);
            }
            float mv = -INFINITY;
            if (k < N) mv = mask ? __ldg(mask + b * m0 + i * m1 + k * m2) * LOG2E : 0.f;
            Mv[e] = mv;
        }
    }
}

// ===========================================================================
// 1b. pre-pass: the pair bias rearranged into the order in which the main
//     kernel's softmax threads read it.  A softmax thread owns one query row j
//     and 32 keys of every 128 x 128 tile, so in the stored [B,H,N,N] layout
//     the 32 lanes of a warp read 32 rows 2N bytes apart and every 16-byte
//     load touches 32 cache lines.  Here each tile (b, h, jt, kt) becomes one
//     32 KB block of 16-byte chunks, chunk index
//         ((w * 4 + qd) * 4 + c) * 32 + lane,
//     for row j = 128 jt + 32 qd + lane and keys k = 128 kt + 32 w + 8 c + 0..7,
//     so that the four loads of a warp per tile each cover 512 contiguous
//     bytes.  Values are copied bit for bit; zeros past N (padded rows get
//     P = 0 from the -inf lse, padded keys the -inf mask).
// ===========================================================================
__global__ void __launch_bounds__(256) tri_attn_bwd_bias_tiles_kernel(const __nv_bfloat16* __restrict__ bias,
                                                                      int64_t s0, int64_t s1, int64_t s2, int B,
                                                                      int H, int N, int nt, uint4* __restrict__ out) {
    const int Np = nt * 128, kcs = Np / 8;
    const int64_t total = static_cast<int64_t>(B) * H * Np * kcs;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        int64_t t = idx;
        const int k0 = static_cast<int>(t % kcs) * 8;  // neighbouring threads read one row: coalesced
        t /= kcs;
        const int j = static_cast<int>(t % Np);
        t /= Np;
        const int h = static_cast<int>(t % H);
        const int b = static_cast<int>(t / H);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (j < N && k0 < N) {
            const __nv_bfloat16* src = bias + b * s0 + h * s1 + static_cast<int64_t>(j) * s2 + k0;
            if (k0 + 8 <= N) {
                v = __ldg(reinterpret_cast<const uint4*>(src));
            } else {  // ragged key tail: element loads, zeros past N
                uint16_t e8[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) e8[u] = (k0 + u < N) ? __bfloat16_as_ushort(src[u]) : 0;
                v = make_uint4(e8[0] | (e8[1] << 16), e8[2] | (e8[3] << 16), e8[4] | (e8[5] << 16),
                               e8[6] | (static_cast<uint32_t>(e8[7]) << 16));
            }
        }
        const int row = j & 127, kk = k0 & 127;
        const int64_t tile = (static_cast<int64_t>(b * H + h) * nt + (j >> 7)) * nt + (k0 >> 7);
        out[(tile << 11) + ((((kk >> 5) * 4 + (row >> 5)) * 4 + ((kk & 31) >> 3)) << 5) + (row & 31)] = v;
    }
}

// ===========================================================================
// 2. main backward kernel: dq, dk, dv
// ===========================================================================
template <int D>
struct MainLayout {
    // warps 0-15: four softmax warpgroups, warpgroup w owns keys 32w..32w+31 of every
    // tile; warp 16 producer, warp 17 issues the gradient MMAs, warp 18 the S and dP
    // MMAs (so a tile's S/dP never waits in one warp's issue order behind the previous
    // tile's gradient MMAs), 19 spare
    static constexpr int THREADS = 640, SOFTMAX_WARPS = 16, W_PRODUCER = 16, W_MMA = 17, W_SMMA = 18;
    static constexpr int KVS = (D == 32) ? 2 : 1;  // K/V buffers
    static constexpr int NS = (D == 32) ? 3 : 2;   // per-tile stages (Q, dO, vectors)
    static constexpr int ROWB = D * 2;
    static constexpr int QKV_TILE = 128 * ROWB;
    static constexpr int PT_TILE = 128 * 128 * 2;  // P or dS, BF16, two 64-column SW128 halves
    // 1 KB aligned tiles
    static constexpr int OFF_KV = 0;                           // [KVS][K, V]
    static constexpr int OFF_T = OFF_KV + KVS * 2 * QKV_TILE;  // [NS][Q, dO]
    static constexpr int T_STAGE = 2 * QKV_TILE;
    static constexpr int OFF_PDS = OFF_T + NS * T_STAGE;       // [2 buffers][P, dS]
    static constexpr int PDS_BUF = 2 * PT_TILE;
    // vectors (bulk-copied from the pre-pass arrays)
    static constexpr int OFF_MASKV = OFF_PDS + 2 * PDS_BUF;  // [KVS][128] fp32 mask*log2(e)
    static constexpr int OFF_FLAGS = OFF_MASKV + KVS * 512;  // [KVS][32] int: key tile needs the mask add
    static constexpr int OFF_VEC = OFF_FLAGS + KVS * 128;    // [NS][lse*log2(e) 128, D 128] fp32
    static constexpr int OFF_BAR = OFF_VEC + NS * 1024;
    static constexpr int B_KVFULL = 0, B_KVEMPTY = KVS, B_TFULL = 2 * KVS, B_TEMPTY = 2 * KVS + NS,
                         B_SDPFULL = 2 * KVS + 2 * NS, B_SDPFREE = B_SDPFULL + 1, B_PDSFULL = B_SDPFULL + 2,
                         B_PDSFREE = B_SDPFULL + 4, B_DQFULL = B_SDPFULL + 6, B_DQFREE = B_SDPFULL + 7,
                         B_DKVFULL = B_SDPFULL + 8, B_DKVFREE = B_SDPFULL + 9, B_DRAIN = B_SDPFULL + 10,
                         NBAR = B_DRAIN + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort flag
    static constexpr int OFF_TRACE = (OFF_MISC + 16 + 7) & ~7;  // phase timing (TRI_TRACE builds only)
    static constexpr int TRACE_BYTES = (OFF_TRACE + kTraceBytes <= 232448) ? kTraceBytes : 0;
    static constexpr int SMEM = OFF_TRACE + TRACE_BYTES;
    static_assert(SMEM <= 232448, "shared memory budget");
    // TMEM columns; dQ is one D-wide block per query tile when they all fit
    // (256 + 2D + nt*D <= 512), else a single block drained every tile
    static constexpr int T_S = 0, T_DP = 128, T_DK = 256, T_DV = 256 + D, T_DQ = 256 + 2 * D;
};

template <int D>
__global__ void __launch_bounds__(640, 1)
    tri_attn_bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                             const BwdParams p) {
    using L = MainLayout<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sb = smem_addr(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto BAR = [&](int idx) -> uint32_t { return sb + L::OFF_BAR + idx * 8; };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

    const int nt = p.nt;
    const int problems = p.B * p.R * p.H;
    // problem index -> (b, h, i) with i fastest so concurrent CTAs share a head's bias
    auto decode = [&](int pr, int& b, int& h, int& i) {
        i = pr % p.R;
        const int t = pr / p.R;
        h = t % p.H;
        b = t / p.H;
    };

    if (threadIdx.x == 0) {
        *abort_flag = device_error_pending() ? 1 : 0;
        if (sb & 1023u) {
            atomicCAS(&g_error_word, 0u, ERR_TIMEOUT_BIT | KERNEL_BWD_MAIN | 0xFFu);
            *abort_flag = 1;
        }
        for (int s = 0; s < L::KVS; ++s) {
            mbar_init(BAR(L::B_KVFULL + s), 1);
            mbar_init(BAR(L::B_KVEMPTY + s), 1 + L::SOFTMAX_WARPS);
        }
        for (int s = 0; s < L::NS; ++s) {
            mbar_init(BAR(L::B_TFULL + s), 1);
            mbar_init(BAR(L::B_TEMPTY + s), 1 + L::SOFTMAX_WARPS);
        }
        mbar_init(BAR(L::B_SDPFULL), 1);
        mbar_init(BAR(L::B_SDPFREE), L::SOFTMAX_WARPS);
        for (int x = 0; x < 2; ++x) {
            mbar_init(BAR(L::B_PDSFULL + x), L::SOFTMAX_WARPS);
            mbar_init(BAR(L::B_PDSFREE + x), 1);
        }
        mbar_init(BAR(L::B_DQFULL), 1);
        mbar_init(BAR(L::B_DQFREE), L::SOFTMAX_WARPS);
        mbar_init(BAR(L::B_DKVFULL), 1);
        mbar_init(BAR(L::B_DKVFREE), L::SOFTMAX_WARPS);
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
    const WaitCtx wc{p.wait_limit_ns, KERNEL_BWD_MAIN, abort_flag};
    const bool aborted_early = *abort_flag != 0;
    constexpr float LOG2E = 1.4426950408889634f;

    if (warp == L::W_PRODUCER) {
        // =========================== producer ===============================
        regs_shrink640();
        int armed_kv[L::KVS], armed_t[L::NS];
#pragma unroll
        for (int s = 0; s < L::KVS; ++s) armed_kv[s] = 0;
#pragma unroll
        for (int s = 0; s < L::NS; ++s) armed_t[s] = 0;
        const bool leader = elect_one();
        if (!aborted_early) {
            if (leader) {
                tma_prefetch_map(&tm_q);
                tma_prefetch_map(&tm_k);
                tma_prefetch_map(&tm_v);
                tma_prefetch_map(&tm_do);
            }
            int gk = 0, g = 0;
            bool ok = true;
            for (int pr = blockIdx.x; ok && pr < problems; pr += gridDim.x) {
                int b, h, i;
                decode(pr, b, h, i);
                auto load_pair = [&](uint32_t dst, const CUtensorMap* m, uint32_t bar, int row0) {
                    tma_load_5d(dst, m, bar, 0, h, row0, i, b);
                };
                const float* mrow = p.Mv + (static_cast<int64_t>(b) * p.R + i) * p.Np;
                const int* frow = p.Fv + (static_cast<int64_t>(b) * p.R + i) * 32;
                const int64_t vrow = ((static_cast<int64_t>(b) * p.H + h) * p.R + i) * p.Np;
                for (int kt = 0; ok && kt < nt; ++kt) {
                    const int ks = gk % L::KVS;
                    if (gk >= L::KVS && !mbar_wait_warp(BAR(L::B_KVEMPTY + ks), ((gk / L::KVS) - 1) & 1, wc, 1)) {
                        ok = false;
                        break;
                    }
                    if (leader) {
                        const uint32_t bar = BAR(L::B_KVFULL + ks);
                        const uint32_t base = sb + L::OFF_KV + ks * 2 * L::QKV_TILE;
                        mbar_arrive_expect_tx(bar, 2 * L::QKV_TILE + 512 + 128);
                        load_pair(base, &tm_k, bar, kt * 128);
                        load_pair(base + L::QKV_TILE, &tm_v, bar, kt * 128);
                        bulk_load(sb + L::OFF_MASKV + ks * 512, mrow + kt * 128, 512, bar);
                        bulk_load(sb + L::OFF_FLAGS + ks * 128, frow, 128, bar);
                    }
                    armed_kv[ks]++;
                    ++gk;
                    for (int jt = 0; jt < nt; ++jt) {
                        const int ts = g % L::NS;
                        if (g >= L::NS && !mbar_wait_warp(BAR(L::B_TEMPTY + ts), ((g / L::NS) - 1) & 1, wc, 2)) {
                            ok = false;
                            break;
                        }
                        if (leader) {
                            const uint32_t bar = BAR(L::B_TFULL + ts);
                            const uint32_t base = sb + L::OFF_T + ts * L::T_STAGE;
                            mbar_arrive_expect_tx(bar, 2 * L::QKV_TILE + 1024);
                            load_pair(base, &tm_q, bar, jt * 128);
                            load_pair(base + L::QKV_TILE, &tm_do, bar, jt * 128);
                            bulk_load(sb + L::OFF_VEC + ts * 1024, p.Lv + vrow + jt * 128, 512, bar);
                            bulk_load(sb + L::OFF_VEC + ts * 1024 + 512, p.Dv + vrow + jt * 128, 512, bar);
                        }
                        armed_t[ts]++;
                        ++g;
                    }
                }
            }
        }
        if (leader) {
#pragma unroll
            for (int s = 0; s < L::KVS; ++s)
                if (armed_kv[s] > 0) drain_wait(BAR(L::B_KVFULL + s), (armed_kv[s] - 1) & 1, 100000000ull);
#pragma unroll
            for (int s = 0; s < L::NS; ++s)
                if (armed_t[s] > 0) drain_wait(BAR(L::B_TFULL + s), (armed_t[s] - 1) & 1, 100000000ull);
        }
    } else if (warp == L::W_MMA || warp == L::W_SMMA) {
        // =========================== MMA issuers ============================
        regs_shrink640();
        const bool leader = elect_one();
        if (!aborted_early) {
            constexpr uint32_t SW = (D == 32) ? SWZ_64B : SWZ_128B;
            constexpr uint32_t SBO = 8 * L::ROWB;
            constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false, false);  // Q K^T, dO V^T
            constexpr uint32_t IDESC_G = idesc_bf16_f32(128, D, true, true);      // P^T dO, dS^T Q
            constexpr uint32_t IDESC_Q = idesc_bf16_f32(128, D, false, true);     // dS K
            // descriptors built once; per-stage / per-step variants are constant adds
            const uint64_t d_tk = smem_desc(sb + L::OFF_T, 16, SBO, SW);            // Q / dO rows, K-major
            const uint64_t d_tmn = smem_desc(sb + L::OFF_T, L::QKV_TILE, SBO, SW);  // Q / dO rows, MN-major
            const uint64_t d_kvk = smem_desc(sb + L::OFF_KV, 16, SBO, SW);          // K / V rows, K-major
            const uint64_t d_kvmn = smem_desc(sb + L::OFF_KV, L::QKV_TILE, SBO, SW);
            const uint64_t d_pmn = smem_desc(sb + L::OFF_PDS, L::PT_TILE / 2, 1024, SWZ_128B);
            const uint64_t d_dsmn = smem_desc(sb + L::OFF_PDS + L::PT_TILE, L::PT_TILE / 2, 1024, SWZ_128B);
            const uint64_t d_dsk = smem_desc(sb + L::OFF_PDS + L::PT_TILE, 16, 1024, SWZ_128B);
            TRI_TRACE_DECL
            bool ok = true;
            if (warp == L::W_SMMA) {
                // ---- S = Q K^T and dP = dO V^T of every tile, as soon as the softmax warps have
                // taken the previous tile's columns ----
                int gk = 0, g = 0;
                for (int pr = blockIdx.x; ok && pr < problems; pr += gridDim.x) {
                    for (int kt = 0; ok && kt < nt; ++kt) {
                        const int ks = gk % L::KVS;
                        TRI_TP(7)
                        if (!mbar_wait_warp(BAR(L::B_KVFULL + ks), (gk / L::KVS) & 1, wc, 6)) { ok = false; break; }
                        TRI_TP(0)
                        const uint64_t kd = desc_add(d_kvk, ks * 2 * L::QKV_TILE);
                        const uint64_t vd = desc_add(kd, L::QKV_TILE);
                        for (int jt = 0; jt < nt; ++jt) {
                            const int ts = g % L::NS;
                            if (!mbar_wait_warp(BAR(L::B_TFULL + ts), (g / L::NS) & 1, wc, 7)) { ok = false; break; }
                            TRI_TP(1)
                            if (g > 0 && !mbar_wait_warp(BAR(L::B_SDPFREE), (g - 1) & 1, wc, 8)) { ok = false; break; }
                            TRI_TP(2)
                            tc_fence_after();
                            const uint64_t qd = desc_add(d_tk, ts * L::T_STAGE), dod = desc_add(qd, L::QKV_TILE);
                            if (leader) {
#pragma unroll
                                for (int kk = 0; kk < D / 16; ++kk) {
                                    mma_ss(tmem + L::T_S, desc_add(qd, kk * 32), desc_add(kd, kk * 32), IDESC_S,
                                           kk > 0 ? 1u : 0u);
                                    mma_ss(tmem + L::T_DP, desc_add(dod, kk * 32), desc_add(vd, kk * 32), IDESC_S,
                                           kk > 0 ? 1u : 0u);
                                }
                                mma_commit(BAR(L::B_SDPFULL));
                            }
                            __syncwarp();
                            TRI_TP(3)
                            ++g;
                        }
                        ++gk;
                    }
                }
            } else {
                // ---- dV += P^T dO, dK += dS^T Q, dQ (+)= dS K of every tile once its P and dS are
                // in SMEM.  Stages, K/V buffers and the P/dS buffer are released by this warp's
                // commits; they also cover the S/dP products of the same tile, which completed
                // before the softmax warps could store its P and dS ----
                int ep_count = 0;  // dQ epilogue tiles issued so far
                int gk = 0, g = 0;
                for (int pr = blockIdx.x; ok && pr < problems; pr += gridDim.x) {
                    for (int kt = 0; ok && kt < nt; ++kt) {
                        const int ks = gk % L::KVS;
                        for (int jt = 0; jt < nt; ++jt) {
                            const int ts = g % L::NS;
                            // a dQ epilogue tile: every tile (single block) or the last key tile of a query tile
                            const bool ep = !p.dq_tmem || kt == nt - 1;
                            TRI_TP(7)
                            const int pb = g & 1;  // P/dS buffer of this tile
                            if (!mbar_wait_warp(BAR(L::B_PDSFULL + pb), (g >> 1) & 1, wc, 3)) { ok = false; break; }
                            TRI_TP(4)
                            // the previous epilogue has read its dQ block (keeps DQ_FULL at most one phase
                            // ahead, and before a new problem overwrites the last query tile's block)
                            const bool reuse = p.dq_tmem && kt == 0 && jt == nt - 1;
                            if ((ep || reuse) && ep_count > 0 &&
                                !mbar_wait_warp(BAR(L::B_DQFREE), (ep_count - 1) & 1, wc, 4)) {
                                ok = false;
                                break;
                            }
                            TRI_TP(5)
                            if (jt == 0 && gk > 0 && !mbar_wait_warp(BAR(L::B_DKVFREE), (gk - 1) & 1, wc, 5)) {
                                ok = false;
                                break;
                            }
                            TRI_TP(6)
                            tc_fence_after();
                            const uint32_t toff = ts * L::T_STAGE;
                            const uint64_t bdo = desc_add(d_tmn, toff + L::QKV_TILE), bq = desc_add(d_tmn, toff);
                            const uint64_t bk = desc_add(d_kvmn, ks * 2 * L::QKV_TILE);
                            const uint32_t dq_col = p.dq_tmem ? L::T_DQ + jt * D : L::T_DQ;
                            const bool dq_acc = p.dq_tmem && kt > 0;
                            if (leader) {
#pragma unroll
                                for (int kk = 0; kk < 8; ++kk) {  // contraction over 128 queries
                                    const uint32_t acc = (jt > 0 || kk > 0) ? 1u : 0u;
                                    // A = P^T / dS^T: MN-major, 64-element chunks 16 KB apart, 8-row groups 1 KB apart
                                    mma_ss(tmem + L::T_DV, desc_add(d_pmn, pb * L::PDS_BUF + kk * 2048),
                                           desc_add(bdo, kk * 16 * L::ROWB), IDESC_G, acc);
                                    mma_ss(tmem + L::T_DK, desc_add(d_dsmn, pb * L::PDS_BUF + kk * 2048),
                                           desc_add(bq, kk * 16 * L::ROWB), IDESC_G, acc);
                                }
#pragma unroll
                                for (int kk = 0; kk < 8; ++kk)  // contraction over 128 keys; A = dS rows j, K-major halves 16 KB apart
                                    mma_ss(tmem + dq_col,
                                           desc_add(d_dsk, pb * L::PDS_BUF + (kk >> 2) * (L::PT_TILE / 2) + (kk & 3) * 32),
                                           desc_add(bk, kk * 16 * L::ROWB), IDESC_Q, (dq_acc || kk > 0) ? 1u : 0u);
                                mma_commit(BAR(L::B_PDSFREE + pb));
                                mma_commit(BAR(L::B_TEMPTY + ts));
                                if (ep) mma_commit(BAR(L::B_DQFULL));
                                if (jt == nt - 1) {
                                    mma_commit(BAR(L::B_DKVFULL));
                                    mma_commit(BAR(L::B_KVEMPTY + ks));
                                }
                            }
                            __syncwarp();
                            if (ep) ++ep_count;
                            ++g;
                        }
                        ++gk;
                    }
                }
            }
            TRI_TP(7)
            TRI_TRACE_FLUSH_AT(20000)
            if (leader) mma_commit(BAR(L::B_DRAIN));
            __syncwarp();
            drain_wait(BAR(L::B_DRAIN), 0, 100000000ull);
        }
        __syncwarp();
    } else if (warp >= L::SOFTMAX_WARPS) {
        regs_shrink640();  // spare warps of the control warpgroup
    } else {
        regs_grow640();
        if (!aborted_early) {
        // =========================== softmax + epilogue warps ===============
        const int w = warp >> 2;  // key quarter of every tile handled by this warpgroup
        const int qd = warp & 3;
        const int row = qd * 32 + lane;
        const uint32_t tl = tmem + (static_cast<uint32_t>(qd * 32) << 16);
        const float scale = p.scale;
        struct Done {
            int g, jt, kt, kcount, b, h, i;
            bool valid;
        } prev{0, 0, 0, 0, 0, 0, 0, false};
        bool ok = true;

        int ep_count = 0;  // dQ epilogues done
        auto epilogue = [&](const Done& t) -> bool {
            // ---- dQ: this warpgroup's D/4 columns of the tile's block ----
            if (!p.dq_tmem || t.kt == nt - 1) {
                if (!mbar_wait_warp(BAR(L::B_DQFULL), ep_count & 1, wc, 10)) return false;
                tc_fence_after();
                const uint32_t dq_col = p.dq_tmem ? L::T_DQ + t.jt * D : L::T_DQ;
                uint32_t dqr[D / 4];
                if constexpr (D == 32) {
                    uint32_t x[8];
                    tmem_ld8(tl + dq_col + w * 8, x);
                    tmem_wait_ld();
                    asm volatile("" : "+r"(x[0]), "+r"(x[1]), "+r"(x[2]), "+r"(x[3]), "+r"(x[4]), "+r"(x[5]),
                                 "+r"(x[6]), "+r"(x[7]));
#pragma unroll
                    for (int e = 0; e < 8; ++e) dqr[e] = x[e];
                } else {
                    uint32_t x[16];
                    tmem_ld16(tl + dq_col + w * 16, x);
                    tmem_wait_ld();
                    reg_fence16(x);
#pragma unroll
                    for (int e = 0; e < 16; ++e) dqr[e] = x[e];
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(L::B_DQFREE));
                ++ep_count;
                const int j = t.jt * 128 + row;
                if (j < p.N) {
                    float acc[D / 4];
#pragma unroll
                    for (int e = 0; e < D / 4; ++e) acc[e] = __uint_as_float(dqr[e]);
                    float* slot = p.dq_slots + (static_cast<int64_t>(blockIdx.x) * p.N + j) * D + w * (D / 4);
                    if (!p.dq_tmem && t.kt > 0) {
#pragma unroll
                        for (int e = 0; e < D / 4; e += 4) {
                            const float4 v = *reinterpret_cast<const float4*>(slot + e);
                            acc[e] += v.x;
                            acc[e + 1] += v.y;
                            acc[e + 2] += v.z;
                            acc[e + 3] += v.w;
                        }
                    }
                    if (!p.dq_tmem && t.kt < nt - 1) {
#pragma unroll
                        for (int e = 0; e < D / 4; e += 4)
                            *reinterpret_cast<float4*>(slot + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
                    } else {
                        __nv_bfloat16* dst = p.dq + t.b * p.dqs[0] + t.i * p.dqs[1] + j * p.dqs[2] + t.h * p.dqs[3] + w * (D / 4);
#pragma unroll
                        for (int e = 0; e < D / 4; e += 8) {
                            uint4 v;
                            v.x = pack_bf16(acc[e] * scale, acc[e + 1] * scale);
                            v.y = pack_bf16(acc[e + 2] * scale, acc[e + 3] * scale);
                            v.z = pack_bf16(acc[e + 4] * scale, acc[e + 5] * scale);
                            v.w = pack_bf16(acc[e + 6] * scale, acc[e + 7] * scale);
                            *reinterpret_cast<uint4*>(dst + e) = v;
                        }
                    }
                }
            }
            // ---- dK (warpgroups 0, 1) or dV (2, 3), D/2 columns each, of a finished key tile ----
            if (t.jt == nt - 1) {
                if (!mbar_wait_warp(BAR(L::B_DKVFULL), t.kcount & 1, wc, 11)) return false;
                tc_fence_after();
                const bool is_dk = w < 2;
                const int c_off = (w & 1) * (D / 2);
                uint32_t g16[D / 2];
                if constexpr (D == 32) {
                    uint32_t x[16];
                    tmem_ld16(tl + (is_dk ? L::T_DK : L::T_DV) + c_off, x);
                    tmem_wait_ld();
                    reg_fence16(x);
#pragma unroll
                    for (int e = 0; e < 16; ++e) g16[e] = x[e];
                } else {
                    uint32_t x[32];
                    tmem_ld32(tl + (is_dk ? L::T_DK : L::T_DV) + c_off, x);
                    tmem_wait_ld();
                    reg_fence32(x);
#pragma unroll
                    for (int e = 0; e < 32; ++e) g16[e] = x[e];
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(L::B_DKVFREE));
                const int k = t.kt * 128 + row;
                if (k < p.N) {
                    const float f = is_dk ? scale : 1.f;
                    __nv_bfloat16* dst = (is_dk
                        ? p.dk + t.b * p.dks[0] + t.i * p.dks[1] + k * p.dks[2] + t.h * p.dks[3]
                        : p.dv + t.b * p.dvs[0] + t.i * p.dvs[1] + k * p.dvs[2] + t.h * p.dvs[3]) + c_off;
                    uint32_t o[D / 4];  // the D/2 values as BF16 pairs
#pragma unroll
                    for (int e = 0; e < D / 2; e += 2)
                        o[e / 2] = pack_bf16(__uint_as_float(g16[e]) * f, __uint_as_float(g16[e + 1]) * f);
                    if ((reinterpret_cast<uintptr_t>(dst) & 31u) == 0) {
                        // 32-byte stores: half the store instructions, each still one row
#pragma unroll
                        for (int e = 0; e < D / 4; e += 8) st_global_v8(dst + 2 * e, o + e);
                    } else {
#pragma unroll
                        for (int e = 0; e < D / 4; e += 4)
                            *reinterpret_cast<uint4*>(dst + 2 * e) = make_uint4(o[e], o[e + 1], o[e + 2], o[e + 3]);
                    }
                }
            }
            return true;
        };

        int gk = 0, g = 0;
        TRI_TRACE_DECL
        for (int pr = blockIdx.x; ok && pr < problems; pr += gridDim.x) {
            int b, h, i;
            decode(pr, b, h, i);
            for (int kt = 0; ok && kt < nt; ++kt) {
                const int ks = gk % L::KVS;
                if (!mbar_wait_warp(BAR(L::B_KVFULL + ks), (gk / L::KVS) & 1, wc, 12)) { ok = false; break; }
                TRI_TP(9)
                const bool has_mask = reinterpret_cast<const int*>(smem + L::OFF_FLAGS + ks * 128)[kt] != 0;
                const uint32_t maskv = sb + L::OFF_MASKV + ks * 512 + w * 128;
                for (int jt = 0; jt < nt; ++jt) {
                    const int ts = g % L::NS;
                    // this thread's 32 bias values (row j, keys kt*128 + 32w ..) from the rearranged
                    // tiles of pre-pass 1b (L2-resident: shared by every row i; each load of the warp
                    // covers 512 contiguous bytes); issued before the waits below
                    uint32_t bw[16];
                    {
                        const uint4* bp = p.bias_tiles +
                                          ((static_cast<int64_t>((b * p.H + h) * nt + jt) * nt + kt) << 11) +
                                          ((w * 4 + qd) << 7) + lane;
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const uint4 v = __ldg(bp + c * 32);
                            bw[4 * c] = v.x;
                            bw[4 * c + 1] = v.y;
                            bw[4 * c + 2] = v.z;
                            bw[4 * c + 3] = v.w;
                        }
                    }
                    if (!mbar_wait_warp(BAR(L::B_SDPFULL), g & 1, wc, 13)) { ok = false; break; }
                    TRI_TP(0)
                    tc_fence_after();
                    if (!mbar_wait_warp(BAR(L::B_TFULL + ts), (g / L::NS) & 1, wc, 14)) { ok = false; break; }
                    TRI_TP(2)
                    const float* vec = reinterpret_cast<const float*>(smem + L::OFF_VEC + ts * 1024);
                    const float nlse2 = vec[row];  // -lse * log2(e)
                    const float nDj = vec[128 + row];  // -D
                    const float2 sc2 = make_float2(scale, scale), l2e = make_float2(LOG2E, LOG2E);
                    const float2 nl2 = make_float2(nlse2, nlse2), nD2 = make_float2(nDj, nDj);
                    // all 32 keys of S and dP first, so the S/dP columns are released to the MMA
                    // warp before any arithmetic
                    uint32_t sv[32], dv[32];
                    tmem_ld32(tl + L::T_S + w * 32, sv);
                    tmem_ld32(tl + L::T_DP + w * 32, dv);
                    tmem_wait_ld();
                    reg_fence32(sv);
                    reg_fence32(dv);
                    TRI_TP(1)
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(BAR(L::B_SDPFREE));
                    // the gradient MMAs of two tiles ago have finished reading this tile's P/dS
                    // buffer (the other one may still be read); each 8-key chunk of P and dS is
                    // stored as soon as it is formed, so the stores drain during the arithmetic
                    const int pb = g & 1;
                    if (g >= 2 && !mbar_wait_warp(BAR(L::B_PDSFREE + pb), ((g >> 1) - 1) & 1, wc, 15)) { ok = false; break; }
                    TRI_TP(3)
                    // this warpgroup's 32 keys = four 16-byte chunks of one 64-key SW128 half
                    const uint32_t prow = sb + L::OFF_PDS + pb * L::PDS_BUF + (w >> 1) * (L::PT_TILE / 2) + row * 128;
                    const uint32_t drow = prow + L::PT_TILE;
                    auto tile = [&](auto masked) {
                        constexpr bool kMasked = decltype(masked)::value;
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) {  // 8-key chunks of this warpgroup's 32 keys
                            float mk[8];
                            if constexpr (kMasked) {
                                const float4 m0 = lds128f(maskv + cc * 32), m1 = lds128f(maskv + cc * 32 + 16);
                                mk[0] = m0.x; mk[1] = m0.y; mk[2] = m0.z; mk[3] = m0.w;
                                mk[4] = m1.x; mk[5] = m1.y; mk[6] = m1.z; mk[7] = m1.w;
                            }
                            uint32_t pw[4], dw[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int xl = cc * 8 + 2 * e;
                                const float2 t = ffma2(make_float2(__uint_as_float(sv[xl]), __uint_as_float(sv[xl + 1])),
                                                       sc2, bf16x2_to_f2(bw[cc * 4 + e]));
                                float2 y = ffma2(t, l2e, nl2);
                                if constexpr (kMasked) y = fadd2(y, make_float2(mk[2 * e], mk[2 * e + 1]));
                                // in key tiles without a mask, one pair in four takes the FMA-pipe exponential
                                const float2 pp = (!kMasked && e == 3) ? ex2_fma2(y) : make_float2(ex2(y.x), ex2(y.y));
                                const float2 ds = fmul2(pp, fadd2(make_float2(__uint_as_float(dv[xl]),
                                                                              __uint_as_float(dv[xl + 1])), nD2));
                                pw[e] = pack_bf16(pp.x, pp.y);
                                dw[e] = pack_bf16(ds.x, ds.y);
                            }
                            const uint32_t off = ((((w & 1) * 4) + cc) ^ (row & 7)) << 4;
                            sts128(prow + off, make_uint4(pw[0], pw[1], pw[2], pw[3]));
                            sts128(drow + off, make_uint4(dw[0], dw[1], dw[2], dw[3]));
                        }
                    };
                    if (has_mask) tile(std::true_type{});
                    else tile(std::false_type{});
                    TRI_TP(4)
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(BAR(L::B_PDSFULL + pb));
                        mbar_arrive(BAR(L::B_TEMPTY + ts));
                        if (jt == nt - 1) mbar_arrive(BAR(L::B_KVEMPTY + ks));
                    }
                    TRI_TP(5)
                    if (prev.valid && !(ok = epilogue(prev))) break;
                    TRI_TP(6)
                    prev = Done{g, jt, kt, gk, b, h, i, true};
                    ++g;
                }
                ++gk;
            }
        }
        if (ok && prev.valid) epilogue(prev);
        TRI_TP(8)
        TRI_TRACE_FLUSH_AT(20000)
    }

    }

    tc_fence_before();
    cta_end_barrier640();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// 3. the dBias kernel is in dbias.cuh

// ascending-index sum of dBias partials (the chunks of one launch, or the chunks of
// every row shard in rank order) -> BF16
__global__ void __launch_bounds__(256) tri_attn_bwd_dbias_reduce_kernel(const float* __restrict__ part, int chunks,
                                                                        int B, int H, int N,
                                                                        __nv_bfloat16* __restrict__ dbias,
                                                                        int64_t s0, int64_t s1, int64_t s2) {
    if (device_error_pending()) return;
    const int64_t total = static_cast<int64_t>(B) * H * N * N;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float acc = part[idx];
        for (int c = 1; c < chunks; ++c) acc += part[static_cast<int64_t>(c) * total + idx];
        int64_t t = idx;
        const int k = static_cast<int>(t % N);
        t /= N;
        const int j = static_cast<int>(t % N);
        t /= N;
        const int h = static_cast<int>(t % H);
        const int b = static_cast<int>(t / H);
        dbias[b * s0 + h * s1 + static_cast<int64_t>(j) * s2 + k] = __float2bfloat16_rn(acc);
    }
}

// ===========================================================================
// host side
// ===========================================================================
bool bwd_set_attributes();
// R: rows i covered; parts: NULL, or where dBias goes as FP32 partial sums
tri_attn_status bwd_launch(const tri_attn_bwd_args* a, int R, float* parts, const BwdWorkspace& ws, float scale,
                           uint64_t wait_ns, cudaStream_t stream, void* const* markers);

}  // namespace tri
