// Device helpers shared by the sink-attention kernels: inline PTX for mbarriers, TMA,
// tcgen05 (UMMA + tensor memory), cp.async and the warp-level mma.sync path, plus bounded
// waits. Everything here is written for sm_100a.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#define SA_DEV __device__ __forceinline__

namespace sinkattn {

// ---------------------------------------------------------------------------------------------
// Host: set-up that must happen once per CUDA context (kernel attributes, symbol addresses)
// ---------------------------------------------------------------------------------------------
// Process-unique id of the CUDA context current on this thread (cuCtxGetId), or 0 when none is
// current yet. A context created after a device reset gets a new id even if its handle value
// repeats, so set-up keyed on it is redone for the new context.
inline unsigned long long current_context_id()
{
    typedef CUresult (*GetCurrentFn)(CUcontext *);
    typedef CUresult (*GetIdFn)(CUcontext, unsigned long long *);
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Runs a set-up step once per CUDA context of each device, from any number of host threads.
// The step runs with the device current; if it fails, it is tried again on the next call.
class PerContextOnce {
  public:
    template <class F> cudaError_t run(F &&setup)
    {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess)
            return e;
        const bool cached = dev >= 0 && dev < kMaxDevices;
        std::lock_guard<std::mutex> lock(mu_);
        const unsigned long long id = current_context_id();
        if (cached && id != 0 && ctx_[dev] == id)
            return cudaSuccess;
        e = setup(dev);
        if (e == cudaSuccess && cached)
            ctx_[dev] = current_context_id(); // the step may have created the context
        return e;
    }

  private:
    static constexpr int kMaxDevices = 256;
    std::mutex mu_;
    unsigned long long ctx_[kMaxDevices] = {};
};

// Device-side error flag: bit 0 = a prefill wait gave up, bit 1 = a decode wait gave up.
// The library is built as one translation unit, so this is its only definition.
__device__ uint32_t g_device_error = 0;

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// A wait on an mbarrier that takes longer than this is treated as a fault: the kernel records
// it and leaves. Legitimate waits here last microseconds. The limit of the waits that give up
// is g_wait_limit_ns (set per device by sinkattn_set_wait_limit_ns; 0 gives up at the first wait
// whose first try fails); a CTA's final waits for its own copies and MMAs keep this one.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;
__constant__ uint64_t g_wait_limit_ns = kWaitLimitNs;

SA_DEV uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

SA_DEV uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------------------------
SA_DEV void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

SA_DEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

SA_DEV void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

SA_DEV void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

SA_DEV bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(smem_u32(bar)), "r"(parity)
                 : "memory");
    return ok != 0;
}

// Non-blocking test: has the phase with the given parity completed?
SA_DEV bool mbar_test(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(smem_u32(bar)), "r"(parity)
                 : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity to complete. Gives up (returns false) when
// *abort is set by another thread, or after g_wait_limit_ns, in which case it sets *abort and
// the device error bit `err_bit`. The limit is only read once the first try has failed, so a
// wait that finds its phase complete costs one instruction; a limit of 0 gives up at that point.
SA_DEV bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort, uint32_t err_bit)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t limit = g_wait_limit_ns;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (limit != 0) {
#pragma unroll 1
            for (int i = 0; i < 32; ++i)
                if (mbar_try_wait(bar, parity))
                    return true;
        }
        if (*abort)
            return false;
        if (globaltimer_ns() - t0 >= limit) {
            *abort = 1;
            atomicOr(&g_device_error, err_bit);
            return false;
        }
    }
}

// Waits for an operation this thread started (a copy or an MMA batch) before the CTA leaves:
// ignores the abort flag, still bounded by kWaitLimitNs.
SA_DEV bool mbar_wait_drain(uint64_t *bar, uint32_t parity)
{
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs)
            return false;
    }
    return true;
}

// ---------------------------------------------------------------------------------------------
// TMA (bulk tensor copies global -> shared, completion counted on an mbarrier)
// ---------------------------------------------------------------------------------------------
SA_DEV void tma_prefetch_desc(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

SA_DEV void tma_load_4d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1, int c2,
                        int c3)
{
    asm volatile("cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1),
                 "r"(c2), "r"(c3)
                 : "memory");
}

// Bulk tensor store shared -> global (tracked by bulk async-groups of the issuing thread).
// Elements outside the tensor are not written.
SA_DEV void tma_store_4d(const CUtensorMap *map, const void *src, int c0, int c1, int c2, int c3)
{
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}
SA_DEV void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until the shared-memory sources of all committed bulk stores have been read.
SA_DEV void bulk_wait_group_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Waits until all committed bulk stores have completed.
SA_DEV void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Barrier among `count` threads of the CTA (id 1..15; id 0 is __syncthreads).
SA_DEV void named_bar_sync(int id, int count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ---------------------------------------------------------------------------------------------
// tcgen05: tensor memory, UMMA, fences
// ---------------------------------------------------------------------------------------------
SA_DEV void tmem_alloc(uint32_t *dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

SA_DEV void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory"); }

SA_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

SA_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
SA_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
SA_DEV void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16 (bf16 inputs, fp32 accumulate).
SA_DEV void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                    uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
                 "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16. A (M x K, K-major) sits in tensor memory:
// row i in lane i, two consecutive bf16 K elements per 32-bit column.
SA_DEV void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                    uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
                 "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// Arrive once on `bar` when every tcgen05.mma issued so far by this thread has completed.
SA_DEV void umma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Instruction descriptor for kind::f16 with bf16 A/B, fp32 D, M x N, K-major A, and B K-major
// (b_mn_major = 0) or MN-major (1). Bit layout: [4,6) D format (1 = f32), [7,10) A format
// (1 = bf16), [10,13) B format, [15] A major, [16] B major, [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, int b_mn_major)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn_major << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor, 128-byte swizzle: [0,14) start >> 4, [16,30) leading byte
// offset >> 4, [32,46) stride byte offset >> 4, [46,48) = 1 (sm100 descriptor version),
// [61,64) = 2 (SWIZZLE_128B). The swizzle atom is 8 rows x 128 B and must be 1024-B aligned.
SA_DEV uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane (base lane + i),
// columns [col, col + 32).
SA_DEV void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                   "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]),
                   "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
                   "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
                   "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
}

SA_DEV void tmem_st32(uint32_t taddr, const uint32_t (&r)[32])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
                 "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                 "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
                 "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),
                 "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]),
                 "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
                 : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns.
SA_DEV void tmem_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                   "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
}

SA_DEV void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 8 consecutive 32-bit columns from registers.
SA_DEV void tmem_st8(uint32_t taddr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3,
                     uint32_t r4, uint32_t r5, uint32_t r6, uint32_t r7)
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(
                     taddr),
                 "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(r4), "r"(r5), "r"(r6), "r"(r7)
                 : "memory");
}

// tcgen05.ld of 16 columns followed by the wait; the registers are tied to the wait so no use
// of them is scheduled before it.
SA_DEV void tmem_ld16_sync(uint32_t taddr, uint32_t (&r)[16])
{
    tmem_ld16(taddr, r);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 16; i += 8)
        asm volatile("" : "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]),
                     "+r"(r[i + 4]), "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7])::"memory");
}
SA_DEV void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// tcgen05.ld of 4 x 32 columns, then one wait; the wait names the registers so no use of them
// can be scheduled before it.
SA_DEV void tmem_ld128(uint32_t taddr, uint32_t (&r)[128])
{
    uint32_t(&a)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[0]);
    uint32_t(&b)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[32]);
    uint32_t(&c)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[64]);
    uint32_t(&d)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[96]);
    tmem_ld32(taddr + 0, a);
    tmem_ld32(taddr + 32, b);
    tmem_ld32(taddr + 64, c);
    tmem_ld32(taddr + 96, d);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 128; i += 8)
        asm volatile("" : "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]),
                     "+r"(r[i + 4]), "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7])::"memory");
}

SA_DEV void tmem_ld32_sync(uint32_t taddr, uint32_t (&r)[32])
{
    tmem_ld32(taddr, r);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 32; i += 8)
        asm volatile("" : "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]),
                     "+r"(r[i + 4]), "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7])::"memory");
}

// A wait whose result is the same in every lane of the warp (required before warp-collective
// tcgen05.ld/st).
SA_DEV bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort)
{
    bool ok = mbar_wait(bar, parity, abort, 1u);
    return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------------------------------------
// scalar math
// ---------------------------------------------------------------------------------------------
// 2^x with the hardware approximation (ex2.approx, flush-to-zero); exact 0 for -inf.
SA_DEV float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

SA_DEV float fast_log2(float x)
{
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

SA_DEV uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// ---------------------------------------------------------------------------------------------
// Partial rotary embedding and value scale on 8-element bf16 pieces (the RoPE pass and the
// commit share these, so both give the same bits)
// ---------------------------------------------------------------------------------------------
// (cos, sin) of the angle m * w, w = theta^(-2i/rope_dim) given in fp64. The angle is formed in
// fp64 and reduced to [-pi, pi] by subtracting the nearest multiple of 2 pi, with 2 pi split into
// a leading and a trailing fp64 part (Cody and Waite's additive range reduction); only then is
// it rounded to fp32 (an error of at most 2^-24 pi, ~1.9e-7 rad) for the hardware sine and
// cosine, __sincosf, whose absolute error on [-pi, pi] is about 2^-21 (~4.8e-7): both far below
// the 2^-9 relative rounding of the bf16 result. At position 262143 the fp32 product alone would
// be off by ~0.016 rad.
SA_DEV float2 rope_cos_sin(int64_t m, double w)
{
    // 2 pi = k2PiHi + k2PiLo: k2PiHi is 2 pi rounded to fp64, k2PiLo what that rounding lost
    const double k2PiHi = 6.283185307179586232, k2PiLo = 2.4492935982947064e-16;
    const double kInv2Pi = 0.15915494309189533577;
    const double angle = (double)m * w;
    const double n2pi = rint(angle * kInv2Pi);
    const double red = fma(-n2pi, k2PiLo, fma(-n2pi, k2PiHi, angle));
    float s, c;
    __sincosf((float)red, &s, &c);
    return make_float2(c, s);
}

// Rotates 8 dimension pairs: a holds x_i (i = i0 .. i0 + 7 of the first rotary half), b the
// partners x_{i + rope_dim/2}; cs[j] = (cos, sin) of pair i0 + j. In fp32, each result rounded
// once to bf16 (nearest even):
//     y_i = x_i cos - x_{i+h} sin,   y_{i+h} = x_{i+h} cos + x_i sin.
SA_DEV void rope_rotate8(uint4 &a, uint4 &b, const float2 *cs)
{
    uint32_t *wa = reinterpret_cast<uint32_t *>(&a);
    uint32_t *wb = reinterpret_cast<uint32_t *>(&b);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 c0 = cs[2 * j], c1 = cs[2 * j + 1];
        const float x0 = __uint_as_float(wa[j] << 16), x1 = __uint_as_float(wa[j] & 0xffff0000u);
        const float y0 = __uint_as_float(wb[j] << 16), y1 = __uint_as_float(wb[j] & 0xffff0000u);
        wa[j] = pack_bf16x2(fmaf(x0, c0.x, -y0 * c0.y), fmaf(x1, c1.x, -y1 * c1.y));
        wb[j] = pack_bf16x2(fmaf(y0, c0.x, x0 * c0.y), fmaf(y1, c1.x, x1 * c1.y));
    }
}

// 8 bf16 values times s, each rounded once to bf16.
SA_DEV void scale8(uint4 &a, float s)
{
    uint32_t *w = reinterpret_cast<uint32_t *>(&a);
#pragma unroll
    for (int j = 0; j < 4; ++j)
        w[j] = pack_bf16x2(__uint_as_float(w[j] << 16) * s, __uint_as_float(w[j] & 0xffff0000u) * s);
}

// Sum of the two bf16 halves of a packed pair, as fp32 (bf16 -> fp32 is exact).
SA_DEV float sum_bf16x2(uint32_t v)
{
    return __uint_as_float(v << 16) + __uint_as_float(v & 0xffff0000u);
}

// ---------------------------------------------------------------------------------------------
// Warp-level tensor-core path (cp.async + ldmatrix + mma.sync), used by decode
// ---------------------------------------------------------------------------------------------
SA_DEV void cp_async16(void *smem_dst, const void *gsrc, bool valid)
{
    // src-size 0 zero-fills the 16 destination bytes without reading global memory
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)),
                 "l"(gsrc), "r"(valid ? 16 : 0)
                 : "memory");
}
SA_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> SA_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

SA_DEV void ldmatrix_x4(uint32_t saddr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(saddr));
}
SA_DEV void ldmatrix_x4_trans(uint32_t saddr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                              uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(saddr));
}

// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
SA_DEV void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                 "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

} // namespace sinkattn
