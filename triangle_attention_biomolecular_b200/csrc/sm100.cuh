// sm100.cuh -- thin inline-PTX wrappers for the Blackwell (sm_100a) features the
// triangle-attention kernels use: mbarriers with bounded waits, TMA tensor
// loads, tcgen05 tensor-memory allocation, MMA, commit and TMEM load/store.
//
// Every spin-wait here is bounded by the GPU global timer.  A wait that runs
// out records a site code in the device error word, raises the CTA's abort
// flag and returns false; callers then leave their loops so that the kernel
// finishes instead of hanging.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

namespace tri {

// ---------------------------------------------------------------------------
// device error word (one per device; read by tri_attn_device_error)
// ---------------------------------------------------------------------------
__device__ uint32_t g_error_word;

// Optional phase timing (instrumentation only; compiled out unless TRI_TRACE is
// defined): lane 0 of each warp accumulates clock64() cycles per phase in shared
// memory (TRACE_BYTES at the kernel layout's OFF_TRACE, so that the timing takes
// no registers from the code it times; global memory where the layout has no room)
// and writes them at the end to a buffer of [blocks][32 warps][16 phases].
#ifdef TRI_TRACE
__device__ unsigned long long* g_trace;
constexpr int kTraceBytes = 24 * 16 * 8;
// accumulators of kernels whose layout has no room left for them (slower: global memory)
__device__ unsigned long long g_trace_spill[256 * 32 * 16];
#define TRI_TRACE_DECL                                                                                        \
    unsigned long long* tri_acc_ = (L::TRACE_BYTES > 0)                                                        \
        ? reinterpret_cast<unsigned long long*>(smem + L::OFF_TRACE) + (threadIdx.x >> 5) * 16                 \
        : g_trace_spill + ((blockIdx.x % 256) * 32 + (threadIdx.x >> 5)) * 16;                                 \
    if ((threadIdx.x & 31) == 0)                                                                            \
        for (int tri_q_ = 0; tri_q_ < 16; ++tri_q_) tri_acc_[tri_q_] = 0;                                  \
    unsigned long long tri_last_ = clock64();
#define TRI_TP(p)                                                  \
    {                                                              \
        const unsigned long long tri_t_ = clock64();               \
        if ((threadIdx.x & 31) == 0) tri_acc_[p] += tri_t_ - tri_last_; \
        tri_last_ = tri_t_;                                        \
    }
#define TRI_TRACE_FLUSH_AT(base)                                                                          \
    {                                                                                                     \
        if (g_trace && (threadIdx.x & 31) == 0)                                                           \
            for (int tri_q_ = 0; tri_q_ < 16; ++tri_q_)                                                   \
                g_trace[(static_cast<size_t>(blockIdx.x + (base)) * 32 + (threadIdx.x >> 5)) * 16 + tri_q_] =  \
                    tri_acc_[tri_q_];                                                                     \
    }
#else
constexpr int kTraceBytes = 0;
#define TRI_TRACE_DECL
#define TRI_TP(p)
#define TRI_TRACE_FLUSH_AT(base)
#endif

// site codes: high byte = kernel, low bits = wait site
enum : uint32_t {
    ERR_TIMEOUT_BIT = 0x80000000u,
    KERNEL_FWD = 1u << 16, KERNEL_BWD_MAIN = 2u << 16, KERNEL_BWD_DBIAS = 3u << 16, KERNEL_TRIMUL = 4u << 16,
    KERNEL_SELFTEST = 15u << 16,
};

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// True if an earlier wait (this launch or an earlier one not yet cleared by
// the host) expired; kernels then return at once without computing.
__device__ __forceinline__ bool device_error_pending() {
    return *reinterpret_cast<volatile uint32_t*>(&g_error_word) != 0u;
}

// Per-CTA wait context: the bound, the site tag and the CTA's abort flag.
struct WaitCtx {
    uint64_t limit_ns;
    uint32_t kernel;
    volatile int* abort_flag;  // shared memory
};

// Wait until the barrier phase with the given parity has completed.  Returns
// false (after recording the site) if the bound expires or another role of
// this CTA has already aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const WaitCtx& w,
                                          uint32_t site) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
#pragma unroll 1
        for (int r = 0; r < 32; ++r)
            if (mbar_try_wait(bar, parity)) return true;
        if (*w.abort_flag) return false;
        if (*reinterpret_cast<volatile uint32_t*>(&g_error_word) != 0u) {  // another CTA gave up
            *w.abort_flag = 1;
            return false;
        }
        if (global_timer_ns() - t0 > w.limit_ns) {
            atomicCAS(&g_error_word, 0u, ERR_TIMEOUT_BIT | w.kernel | site);
            *w.abort_flag = 1;
            return false;
        }
    }
}

// Bounded wait used only while draining on the way out: ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit_ns) break;
    }
}

// Whole-warp form: every lane waits and the result is made warp-uniform, so a
// bound that expires on some lanes only can never split the warp's control flow.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, const WaitCtx& w,
                                               uint32_t site) {
    const bool ok = mbar_wait(bar, parity, w, site);
    return __all_sync(0xFFFFFFFFu, ok) != 0;
}

// ---------------------------------------------------------------------------
// TMA (tensor maps are __grid_constant__ kernel parameters)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* m, uint32_t bar, int c0,
                                            int c1, int c2, int c3, int c4) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
        : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* m, uint32_t bar, int c0,
                                            int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
// 1-D bulk copy global -> shared (addresses 16-byte aligned, size a multiple of 16)
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}
// make generic-proxy writes to shared memory visible to the async proxy (tcgen05.mma operands)
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory
// ---------------------------------------------------------------------------
// Allocate `ncols` (power of two >= 32) TMEM columns; whole warp; base written to smem.
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// One lane of a converged warp (the lowest active one).  The MMA and TMA issuing
// roles keep the whole warp in their loops, so loop counters, barrier phases and
// descriptors stay warp-uniform, and issue only the asynchronous instructions from
// the elected lane: issuing from a lane-0-only branch measured up to 1.5x slower.
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "elect.sync _|P, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, P;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T-as-described, kind::f16 (bf16 in, fp32 acc)
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// A operand from TMEM
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on an mbarrier once every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// Instruction descriptor for kind::f16 with BF16 A/B and FP32 accumulation.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4)                                  // D format: f32
           | (1u << 7)                                // A: bf16
           | (1u << 10)                               // B: bf16
           | ((a_mn_major ? 1u : 0u) << 15)           // A major
           | ((b_mn_major ? 1u : 0u) << 16)           // B major
           | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);   // M / 16
}

// Shared-memory matrix descriptor (sm100 version bits = 1).
enum : uint32_t { SWZ_NONE = 0, SWZ_128B = 2, SWZ_64B = 4, SWZ_32B = 6 };
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t swizzle) {
    return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) |
           (static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) |
           (static_cast<uint64_t>(swizzle) << 61);
}

// A descriptor advanced by a byte offset (start-address field, 16-byte units; the
// field never carries because shared-memory addresses stay below 256 KB).
__device__ __forceinline__ uint64_t desc_add(uint64_t desc, uint32_t byte_offset) { return desc + (byte_offset >> 4); }

// TMEM loads/stores, shape 32x32b: each thread of the warp moves consecutive
// 32-bit columns of its own TMEM lane.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Register rebalancing between warpgroups.  Kernels launch 384 threads
// (168 registers each, 64512 total); the producer/MMA warpgroup gives up
// registers and the two softmax warpgroups take them:
// 128 * 88 + 256 * 208 = 64512, exactly the launch total.
constexpr int kRegsLaunch = 168, kRegsSmall = 88, kRegsLarge = 208;
static_assert(128 * kRegsSmall + 256 * kRegsLarge <= 384 * kRegsLaunch && kRegsSmall % 8 == 0 && kRegsLarge % 8 == 0,
              "register split must fit the launch total");
__device__ __forceinline__ void regs_shrink() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsSmall)); }
// The same for 640-thread kernels (four softmax warpgroups and one control
// warpgroup, 96 registers each at launch, 61440 total): 512 * 104 + 128 * 56 = 60416.
constexpr int kRegsLaunch640 = 96, kRegsSmall640 = 56, kRegsLarge640 = 104;
static_assert(128 * kRegsSmall640 + 512 * kRegsLarge640 <= 640 * kRegsLaunch640 && kRegsSmall640 % 8 == 0 &&
                  kRegsLarge640 % 8 == 0,
              "register split must fit the launch allocation");
__device__ __forceinline__ void regs_shrink640() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsSmall640));
}
__device__ __forceinline__ void regs_grow640() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsLarge640)); }
// A wider split of the same 640-thread launch for kernels whose control warps
// need few registers: 512 * 112 + 128 * 32 = 61440, the launch total.
constexpr int kRegsSmall640w = 32, kRegsLarge640w = 112;
static_assert(128 * kRegsSmall640w + 512 * kRegsLarge640w <= 640 * kRegsLaunch640, "register split must fit the launch");
__device__ __forceinline__ void regs_shrink640w() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsSmall640w));
}
__device__ __forceinline__ void regs_grow640w() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsLarge640w)); }
__device__ __forceinline__ void regs_grow() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsLarge)); }
// every role of the CTA meets here before tensor memory is released
__device__ __forceinline__ void cta_end_barrier() { asm volatile("bar.sync 1, 384;" ::: "memory"); }
__device__ __forceinline__ void cta_end_barrier640() { asm volatile("bar.sync 1, 640;" ::: "memory"); }

// ---------------------------------------------------------------------------
// arithmetic helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ex2(float x) {  // hardware 2^x (MUFU)
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// (lo, hi) -> bf16x2 with lo in the low half, round-to-nearest-even
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// packed FP32 pair arithmetic (one instruction for two lanes of work; IEEE
// round-to-nearest like the scalar forms, so results are identical)
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 fadd2_rm(float2 a, float2 b) {  // rounded toward minus infinity
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rm.ftz.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// 2^x for a pair of arguments on the FMA pipe, leaving the MUFU unit free: the
// kernels route a fixed share of their exponentials here so that both pipes work.
// Method (range reduction + polynomial): x = n + f with n = floor(x), taken from the
// low mantissa bits of x + 1.5*2^23 added with rounding toward minus infinity;
// 2^f on [0, 1) by the cubic c0 + c1 f + c2 f^2 + c3 f^3, whose coefficients were
// fitted for least maximum relative error by Lawson's iterated weighted least
// squares (7.5e-5 in exact arithmetic, 1.4e-4 with float32 evaluation); n is then
// added into the exponent field.  Arguments are clamped to >= -125, so anything
// below gives 2^-125 (about 2.4e-38) rather than 0: callers use it only where a
// masked key (which must give exactly 0) cannot occur.
constexpr float kEx2C0 = 0.9999251365661621f, kEx2C1 = 0.6958339810371399f, kEx2C2 = 0.22606706619262695f,
                kEx2C3 = 0.07802402973175049f;
__device__ __forceinline__ float2 ex2_fma2(float2 x) {
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
    x.x = fmaxf(x.x, -125.f);
    x.y = fmaxf(x.y, -125.f);
    const float2 t = fadd2_rm(x, make_float2(kMagic, kMagic));      // 1.5*2^23 + floor(x)
    const float2 n = fadd2(t, make_float2(-kMagic, -kMagic));       // floor(x), exact
    const float2 f = ffma2(n, make_float2(-1.f, -1.f), x);          // x - floor(x), exact
    float2 q = ffma2(make_float2(kEx2C3, kEx2C3), f, make_float2(kEx2C2, kEx2C2));
    q = ffma2(q, f, make_float2(kEx2C1, kEx2C1));
    q = ffma2(q, f, make_float2(kEx2C0, kEx2C0));
    // floor(x) sits in the low mantissa bits of t; shifting t left by 23 moves it into the
    // exponent field (the constant high bits shift out)
    return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}
// max of three
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
// the two BF16 halves of a packed word as an FP32 pair (low half first)
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) { return make_float2(bf16lo(w), bf16hi(w)); }

// one 32-byte global store of eight 32-bit words (address 32-byte aligned)
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t* w) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]), "r"(w[1]),
                 "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ float4 lds128f(uint32_t a) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

}  // namespace tri
