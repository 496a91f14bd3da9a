// ptx.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers with bounded
// waits, TMA and bulk copies, tcgen05 (TMEM allocation, loads/stores,
// scale-factor copies, block-scaled MXFP4 MMA) and E2M1 conversion.
#pragma once

#include <cstdint>

namespace mxattn {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// try_wait that lets the hardware suspend the thread for up to `hint_ns`
// while the phase is incomplete (it resumes as soon as the phase completes).
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return done != 0;
}

// Wait for the phase with the given parity to complete, giving up after
// `timeout_ns` of wall time or as soon as another role of the CTA raised
// `*abort_flag`.  On timeout it raises the flag and ORs `code` into the
// global status word.  Returns false when the wait gave up.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                  uint32_t* status, uint32_t code, uint64_t timeout_ns,
                                                  uint32_t hint_ns = 0) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (hint_ns ? mbar_try_wait_hint(bar, parity, hint_ns) : mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0u) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > timeout_ns) {
                *abort_flag = 1;
                atomicOr(status, code);
                return false;
            }
        }
    }
}

// ------------------------------------------------------------------ TMA / bulk copies

__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, uint64_t* bar, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(tmap), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Block-wide named barrier `id` over `nthreads` threads (the arrival point may
// differ between warps).
__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// True in exactly one lane of the converged warp (the same lane on every call
// from the same warp state); the warp's uniform loop state stays uniform.
__device__ __forceinline__ bool elect_one_sync() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

// ------------------------------------------------------------------ register reallocation

// Move registers between warpgroups (executed by every thread of a warpgroup).
template <uint32_t kRegs>
__device__ __forceinline__ void warpgroup_regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegs));
}
template <uint32_t kRegs>
__device__ __forceinline__ void warpgroup_regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegs));
}

// ------------------------------------------------------------------ tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Copy a 32-row x 16-byte scale-factor block from shared memory into TMEM
// (4 columns), replicated into all four 32-lane sub-partitions.
__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T with E2M1 operands and E8M0 block-32 scales (TMEM).
__device__ __forceinline__ void tc_mma_mxf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// The NVFP4 form: E2M1 operands with one E4M3 scale per 16 elements
// (block16); the four scale bytes of a row for one K = 64 step sit in one
// TMEM column, so the scale-factor ids are 0.
__device__ __forceinline__ void tc_mma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

#define MXATTN_R8(b) "=r"(v[b + 0]), "=r"(v[b + 1]), "=r"(v[b + 2]), "=r"(v[b + 3]), \
                     "=r"(v[b + 4]), "=r"(v[b + 5]), "=r"(v[b + 6]), "=r"(v[b + 7])
#define MXATTN_W8(b) "r"(v[b + 0]), "r"(v[b + 1]), "r"(v[b + 2]), "r"(v[b + 3]), \
                     "r"(v[b + 4]), "r"(v[b + 5]), "r"(v[b + 6]), "r"(v[b + 7])

// 32 consecutive fp32 columns of this thread's TMEM lane; waits for completion
// inside the same asm statement so the outputs are valid when it returns.
__device__ __forceinline__ void tmem_ld32_sync(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : MXATTN_R8(0), MXATTN_R8(8), MXATTN_R8(16), MXATTN_R8(24)
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}


__device__ __forceinline__ void tmem_ld64_sync(uint32_t taddr, uint32_t (&v)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
        "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
        "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : MXATTN_R8(0), MXATTN_R8(8), MXATTN_R8(16), MXATTN_R8(24), MXATTN_R8(32), MXATTN_R8(40),
          MXATTN_R8(48), MXATTN_R8(56)
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_st64(uint32_t taddr, const uint32_t (&v)[64]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, "
        "%33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, "
        "%49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, %64};" ::"r"(taddr),
        MXATTN_W8(0), MXATTN_W8(8), MXATTN_W8(16), MXATTN_W8(24), MXATTN_W8(32), MXATTN_W8(40), MXATTN_W8(48),
        MXATTN_W8(56)
        : "memory");
}

__device__ __forceinline__ void tmem_st1(uint32_t taddr, uint32_t v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t tmem_ld1_sync(uint32_t taddr) {
    uint32_t v;
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(v)
        : "r"(taddr)
        : "memory");
    return v;
}

#undef MXATTN_R8
#undef MXATTN_W8

// ------------------------------------------------------------------ descriptors

// Shared-memory matrix descriptor (tcgen05 "matrix descriptor"): start
// address, leading/stride byte offsets (16-byte units), version 1, layout.
enum : uint32_t { kLayoutNone = 0, kLayoutSw128 = 2, kLayoutSw64 = 4, kLayoutSw32 = 6 };

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t layout) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;  // descriptor version for sm_100
    d |= static_cast<uint64_t>(layout & 7u) << 61;
    return d;
}

// Instruction descriptor for kind::mxf4 (E2M1 x E2M1, E8M0 scales, K-major
// A and B, dense K = 64): M = 128, N given, scale-factor byte ids.
__host__ __device__ constexpr uint32_t mxf4_idesc(uint32_t n, uint32_t sfa_id, uint32_t sfb_id) {
    return (1u << 7)                  // A format E2M1
           | (1u << 10)               // B format E2M1
           | ((sfb_id & 3u) << 4)     // B scale-factor byte id
           | ((n >> 3) << 17)         // N / 8
           | (1u << 23)               // scale format E8M0
           | ((128u >> 4) << 24)      // M / 16
           | ((sfa_id & 3u) << 29);   // A scale-factor byte id
}


// Instruction descriptor of tcgen05.mma kind::mxf4nvf4 block16: M = 128, N = n,
// E2M1 A and B, E4M3 scale factors (format bit 0), scale-factor ids 0.
__host__ __device__ constexpr uint32_t nvf4_idesc(uint32_t n) {
    return (1u << 7)                  // A format E2M1
           | (1u << 10)               // B format E2M1
           | ((n >> 3) << 17)         // N / 8
           | ((128u >> 4) << 24);     // M / 16
}

__device__ __forceinline__ float lg2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// max(a, b, c) in one instruction (sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// (o0, o1) = (x0, x1) * k + (c, c) as one packed f32x2 FMA.
__device__ __forceinline__ void ffma2_bcast(float& o0, float& o1, float x0, float x1, float k, float c) {
    asm("{\n\t.reg .b64 a, b, c, d;\n\t"
        "mov.b64 a, {%2, %3};\n\t"
        "mov.b64 b, {%4, %4};\n\t"
        "mov.b64 c, {%5, %5};\n\t"
        "fma.rn.f32x2 d, a, b, c;\n\t"
        "mov.b64 {%0, %1}, d;\n\t}"
        : "=f"(o0), "=f"(o1)
        : "f"(x0), "f"(x1), "f"(k), "f"(c));
}


// (o0, o1) = (x0, x1) * k as one packed f32x2 multiply.
__device__ __forceinline__ void fmul2_bcast(uint32_t& o0, uint32_t& o1, uint32_t x0, uint32_t x1, float k) {
    asm("{\n\t.reg .b64 a, b, d;\n\t"
        "mov.b64 a, {%2, %3};\n\t"
        "mov.b64 b, {%4, %4};\n\t"
        "mul.rn.f32x2 d, a, b;\n\t"
        "mov.b64 {%0, %1}, d;\n\t}"
        : "=r"(o0), "=r"(o1)
        : "r"(x0), "r"(x1), "f"(k));
}

// 2^w for two values on the FMA pipe instead of the MUFU (Cody & Waite style
// range reduction: 2^w = 2^n * 2^f, n = round(w), f = w - n in [-1/2, 1/2]).
// 2^f is a degree-5 polynomial fitted for relative error on [-1/2, 1/2]
// (coefficients from csrc/exp2_poly_fit.py; max relative error 2.3e-7 in fp32),
// 2^n is added to the exponent field.  Inputs are clamped at -125 so the
// result stays a normal number (2^-125 where the exact value is smaller).
__device__ __forceinline__ void exp2_fma_x2(float w0, float w1, float& v0, float& v1) {
    w0 = fmaxf(w0, -125.f);
    w1 = fmaxf(w1, -125.f);
    uint32_t p0, p1, t0, t1;
    asm("{\n\t.reg .b64 w, t, n, f, p, c;\n\t"
        "mov.b64 w, {%4, %5};\n\t"
        "mov.b64 c, {%6, %6};\n\t"
        "add.rn.f32x2 t, w, c;\n\t"      // round(w) lands in the low mantissa bits of t
        "sub.rn.f32x2 n, t, c;\n\t"      // n = round(w)
        "sub.rn.f32x2 f, w, n;\n\t"      // f in [-1/2, 1/2]
        "mov.b64 p, {%12, %12};\n\t"
        "mov.b64 c, {%11, %11};\n\t"
        "fma.rn.f32x2 p, p, f, c;\n\t"
        "mov.b64 c, {%10, %10};\n\t"
        "fma.rn.f32x2 p, p, f, c;\n\t"
        "mov.b64 c, {%9, %9};\n\t"
        "fma.rn.f32x2 p, p, f, c;\n\t"
        "mov.b64 c, {%8, %8};\n\t"
        "fma.rn.f32x2 p, p, f, c;\n\t"
        "mov.b64 c, {%7, %7};\n\t"
        "fma.rn.f32x2 p, p, f, c;\n\t"
        "mov.b64 {%0, %1}, p;\n\t"
        "mov.b64 {%2, %3}, t;\n\t}"
        : "=r"(p0), "=r"(p1), "=r"(t0), "=r"(t1)
        : "f"(w0), "f"(w1), "f"(12582912.0f),  // 1.5 * 2^23
          "f"(0x1.000002p+0f), "f"(0x1.62e428p-1f), "f"(0x1.ebf91ap-3f), "f"(0x1.c6b782p-5f), "f"(0x1.3d0ba4p-7f),
          "f"(0x1.5bc922p-10f));
    v0 = __uint_as_float(p0 + (t0 << 23));
    v1 = __uint_as_float(p1 + (t1 << 23));
}

// A stand-in for 2^w whose E2M1 code (cvt.rn.satfinite.e2m1x2) equals the
// code of 2^w, for two values on the FMA pipe, with w = s * k + b given as
// u = sat(s * k8 + b8), k8 = k / 8, b8 = (b + 2) / 8: the saturating FMA maps
// w in [-2, 6] onto u in [0, 1] and clamps everything outside (w <= -2, every
// value whose code is 0, gives u = 0; -inf and NaN too).  The code of 2^w only
// depends on where w falls against the log2 of the seven E2M1 rounding points
// 0.25, 0.75, 1.25, 1.75, 2.5, 3.5 and 5, so p(u) is the degree-6 polynomial
// that takes the value t at u = (log2 t + 2) / 8 for each of them (p(0) = 0.25
// exactly, so the tie at 2^-2 rounds to 0 like the exact value) and increases
// on [0, 1] (p(1) = 59.4 > 5).  Coefficients from csrc/exp2_code_fit.py.  p
// lands on the same side of every rounding point as 2^w except within fp32
// rounding of the crossing (a few ulp of w + 2), as for ex2.approx.  Its value
// is NOT 2^w (7 % off above the last point): use it only where nothing but
// the code is kept.  Two scalar FMAs (f32x2 has no saturating form) and six
// packed ones per pair; no ALU instruction.
__device__ __forceinline__ void exp2_code_sat_x2(float s0, float s1, float k8, float b8, float& v0, float& v1) {
    float u0, u1;
    asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(u0) : "f"(s0), "f"(k8), "f"(b8));
    asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(u1) : "f"(s1), "f"(k8), "f"(b8));
    uint32_t p0, p1;
    asm("{\n\t.reg .b64 u, p, c;\n\t"
        "mov.b64 u, {%2, %3};\n\t"
        "mov.b64 p, {%4, %4};\n\t"
        "mov.b64 c, {%5, %5};\n\t"
        "fma.rn.f32x2 p, p, u, c;\n\t"
        "mov.b64 c, {%6, %6};\n\t"
        "fma.rn.f32x2 p, p, u, c;\n\t"
        "mov.b64 c, {%7, %7};\n\t"
        "fma.rn.f32x2 p, p, u, c;\n\t"
        "mov.b64 c, {%8, %8};\n\t"
        "fma.rn.f32x2 p, p, u, c;\n\t"
        "mov.b64 c, {%9, %9};\n\t"
        "fma.rn.f32x2 p, p, u, c;\n\t"
        "mov.b64 c, {%10, %10};\n\t"
        "fma.rn.f32x2 p, p, u, c;\n\t"
        "mov.b64 {%0, %1}, p;\n\t}"
        : "=r"(p0), "=r"(p1)
        : "f"(u0), "f"(u1),  // c6 .. c0
          "f"(0x1.0132fcp+6f), "f"(-0x1.b3010ap+5f), "f"(0x1.6e5d76p+5f), "f"(-0x1.9f6ee0p+1f), "f"(0x1.56cd60p+2f),
          "f"(0x1.4c45dep+0f), "f"(0x1.000000p-2f));
    v0 = __uint_as_float(p0);
    v1 = __uint_as_float(p1);
}

// ------------------------------------------------------------------ E2M1 / E8M0 helpers

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Eight fp32 values (already divided by the block scale) to eight E2M1 codes
// packed in a 32-bit word, element 0 in the lowest nibble; round to nearest
// even, saturate to +-6.
__device__ __forceinline__ uint32_t pack_e2m1x8(const float (&x)[8]) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(x[0]), "f"(x[1]), "f"(x[2]), "f"(x[3]), "f"(x[4]), "f"(x[5]), "f"(x[6]), "f"(x[7]));
    return out;
}

// E4M3 (OCP FP8, no infinities) byte of a non-negative fp32 value: round to
// nearest even, values at or above 448 saturate to 448 (0x7E).
__device__ __forceinline__ uint32_t e4m3_encode_sat(float v) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(0.f), "f"(v));
    return d & 0xFFu;
}

// E4M3 byte -> fp32 value (exact).
__device__ __forceinline__ float e4m3_decode(uint32_t b) {
    float f;
    asm("{\n\t.reg .b16 lo, hi;\n\t.reg .b32 h2;\n\t"
        "cvt.u16.u32 lo, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 h2, lo;\n\t"
        "mov.b32 {lo, hi}, h2;\n\t"
        "cvt.f32.f16 %0, lo;\n\t}"
        : "=f"(f)
        : "r"(b));
    return f;
}

// Block exponent e of an MXFP4 block of P, in the log domain, from d = bm - m
// (the block's largest score minus the running maximum, <= 0; -inf for a
// block that is all masked): x = d * kq is the log2 of the block's largest
// exponential.  Scale boundary Qmax < 8 (UOS: 7.25): e = ceil(x - log2 Qmax),
// the smallest e with 2^x <= Qmax * 2^e, formed as one rounding of
// d * kq - log2 Qmax; OCP (Qmax = 8 with the OCP convention): e = floor(x) - 2,
// with x rounded once, so x = 0 exactly for the block that holds the row
// maximum.  The integer part comes from an add of 1.5 * 2^23 rounded up (ceil)
// or down (floor), exact for |z| < 2^22; z is clamped first so e >= -127.
// Returns e as an integer-valued float and sets `byte` to the E8M0 code e + 127.
template <bool OCP>
__device__ __forceinline__ float p_block_exp(float d, float kq, float log2q, uint32_t& byte) {
    if constexpr (OCP) {
        const float x = fmaxf(d * kq, -125.f);
        const float t = __fadd_rd(x, 12582912.f);
        byte = __float_as_uint(t) - 0x4B3FFF83u;  // floor(x) - 2 + 127
        return t - 12582914.f;                    // floor(x) - 2
    } else {
        const float z = fmaxf(fmaf(d, kq, -log2q), -127.f);
        const float t = __fadd_ru(z, 12582912.f);
        byte = __float_as_uint(t) - 0x4B3FFF81u;  // ceil(z) + 127
        return t - 12582912.f;                    // ceil(z)
    }
}

// NVFP4 block of P from x = log2 of the block's largest exponential: the E4M3
// code of its scale, sb = E4M3(2^x * 448) (round to nearest even, saturating).
__device__ __forceinline__ uint32_t nv_p_block_scale(float x) {
    return e4m3_encode_sat(ex2_approx(x) * 448.f);
}

// log2(2688 / v) for a positive E4M3 scale value v (exact in fp32), as two
// parts whose sum carries one rounding of the fraction: with v = 2^(E - 127) * s,
// s in [1, 2), 2688 = 2^11 * 1.3125, so log2(2688 / v) = (138 - E) + (log2 1.3125
// - log2 s).  ei = 138 - E is an exact integer; fr lies in (-0.61, 0.40], so
// ei + fr (or (ei + 2) / 8 + fr / 8) rounds once at the size of the result.
// lg2 runs only on the significand.  v = 0 gives meaningless parts; callers
// select on the scale code.
__device__ __forceinline__ void nv_p_scale_log2_parts(float v, float& ei, float& fr) {
    const uint32_t bits = __float_as_uint(v);
    fr = 0.39231742277876f - lg2_approx(__uint_as_float((bits & 0x7FFFFFu) | 0x3F800000u));
    ei = static_cast<float>(138 - static_cast<int>(bits >> 23));
}

// Block exponent from the bfloat16 bit pattern of a block maximum (>= 0)
// under a scale boundary Qmax in (4, 8]: the smallest e with amax <= Qmax * 2^e
// is floor(log2 amax) - 2, plus one when the significand exceeds Qmax / 4,
// i.e. when the mantissa field exceeds floor((Qmax/4 - 1) * 2^7) (UOS: 0x68;
// OCP, floor(log2 amax) - 2: 0x7F, never exceeded).  Zero and subnormal
// maxima give -127.
__device__ __forceinline__ int block_exponent_bf16(uint32_t amax_bits, uint32_t mant_thresh) {
    const int E = static_cast<int>((amax_bits >> 7) & 0xFFu);
    if (E == 0) return -127;
    int e = E - 129 + (((amax_bits & 0x7Fu) > mant_thresh) ? 1 : 0);
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^-e as fp32 for e in [-127, 127] (2^-127 is the one subnormal case).
__device__ __forceinline__ float exp2_neg_int(int e) {
    return e >= 127 ? __uint_as_float(0x00400000u) : __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
}

}  // namespace mxattn
