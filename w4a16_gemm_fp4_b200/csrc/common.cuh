// common.cuh -- helpers shared by the sm_100a kernels of libfp4w4a16:
// format tables, the device status word, bf16 nibble dequantization, and
// thin inline-PTX wrappers for mbarrier, TMA and tcgen05 (tensor memory).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/fp4w4a16.h"

namespace fp4 {

// ------------------------------------------------------------ format table
// Magnitudes of codes 0..7 of one 4-bit ExMy format (the value formula of
// the LLM-FP4 summary page: p == 0 subnormal 2^(1-b) * 0.d, otherwise
// 2^(p-b) * 1.d, bias b = 2^(e-1)-1), their midpoints and Qmax.  Built on
// the host (capi.cu) and passed to kernels by value.
struct FmtTable {
    float mag[8];
    float mid[7];  // mid[i] = (mag[i] + mag[i+1]) / 2, exact in fp32
    float qmax;
};

struct FmtTables {
    FmtTable f[3];
    float cj[8];  // fl32(2^(-j/8)): real-valued exponent-bias candidates
    // Exact decision boundaries of the nearest-code tests (see code_threshold
    // in quantize.cu): test i of format f passes when fl32(|x|/s) lies above
    // hb[f][i], or exactly on it when bit i of tie_up[f] is set.
    double hb[3][7];
    uint32_t tie_up[3];
};

// Device status word bits (mirrors FP4_DEV_* of the public header).
constexpr int kStatusNonfinite = FP4_DEV_NONFINITE_INPUT;
constexpr int kStatusScaleOverflow = FP4_DEV_SCALE_OVERFLOW;
constexpr int kStatusTimeout = FP4_DEV_WAIT_TIMEOUT;
constexpr int kStatusLayout = FP4_DEV_LAYOUT;

__device__ __forceinline__ void raise_status(int* status, int bits) {
    if (status) atomicOr(status, bits);
}

// Nearest magnitude index of a = |q| (q = fl32(x / s)): count the
// midpoints below a; at an exact midpoint mid[i] (between i and i+1) the
// even index wins.  |q| >= Qmax is index 7 (a > mid[6]).
__device__ __forceinline__ int nearest_index(float a, const FmtTable& t) {
    int idx = 0;
#pragma unroll
    for (int i = 0; i < 7; ++i) {
        // strictly above the midpoint -> at least i+1; equal -> i+1 only if
        // i+1 is even (i odd)
        idx += (a > t.mid[i]) || ((a == t.mid[i]) && (i & 1));
    }
    return idx;
}

// ---------------------------------------------------- bf16 nibble dequant
// A 16-entry code -> bf16 table held in four registers as split byte
// planes: lo0/hi0 = low/high bytes of the bf16 values of magnitude indices
// 0..3, lo1/hi1 = indices 4..7.  The sign is applied separately, because
// bf16(-v) differs from bf16(v) only in bit 15.
struct Bf16Lut {
    uint32_t lo0, lo1, hi0, hi1;
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// LUT of bf16(mag[i] * s) (s = 1 gives the exact magnitudes).
__device__ __forceinline__ Bf16Lut make_lut(const float* mag, float s) {
    uint32_t b01 = pack_bf16x2(__fmul_rn(mag[0], s), __fmul_rn(mag[1], s));
    uint32_t b23 = pack_bf16x2(__fmul_rn(mag[2], s), __fmul_rn(mag[3], s));
    uint32_t b45 = pack_bf16x2(__fmul_rn(mag[4], s), __fmul_rn(mag[5], s));
    uint32_t b67 = pack_bf16x2(__fmul_rn(mag[6], s), __fmul_rn(mag[7], s));
    Bf16Lut l;
    l.lo0 = prmt(b01, b23, 0x6420);
    l.hi0 = prmt(b01, b23, 0x7531);
    l.lo1 = prmt(b45, b67, 0x6420);
    l.hi1 = prmt(b45, b67, 0x7531);
    return l;
}

// Dequantize one 32-bit word of packed codes (nibble i = element i, low
// nibble first) into four bf16x2 words p[j] = (elem 2j, elem 2j+1), low
// half = lower k.  15 integer ops for 8 elements:
//  - the magnitude index (code & 7) selects a byte of each byte plane;
//  - prmt in sign-replicate mode (selector bit 3) turns each code's sign bit
//    into a 0x00/0xFF byte, and bit 7 of it is OR-ed into the high byte.
__device__ __forceinline__ void dequant8(uint32_t w, const Bf16Lut& l, uint32_t p[4]) {
    const uint32_t m = w & 0x77777777u;
    const uint32_t w4 = w << 4;
    const uint32_t mh = m >> 16;
    {
        uint32_t lo = prmt(l.lo0, l.lo1, m);
        uint32_t hi = prmt(l.hi0, l.hi1, m);
        uint32_t sg = prmt(w, w4, 0x9D8Cu);  // sign bytes of elements 0..3
        hi |= sg & 0x80808080u;
        p[0] = prmt(lo, hi, 0x5140u);
        p[1] = prmt(lo, hi, 0x7362u);
    }
    {
        uint32_t lo = prmt(l.lo0, l.lo1, mh);
        uint32_t hi = prmt(l.hi0, l.hi1, mh);
        uint32_t sg = prmt(w, w4, 0xBFAEu);  // sign bytes of elements 4..7
        hi |= sg & 0x80808080u;
        p[2] = prmt(lo, hi, 0x5140u);
        p[3] = prmt(lo, hi, 0x7362u);
    }
}

// Exact code values by bit placement, 8 codes of one 32-bit word at a time,
// for a format with MANT mantissa bits (E1M2: 2, E2M1: 1, E3M0: 0) and bias
// b = 2^(2-MANT) - 1.  The 3 magnitude bits of a code are placed so that the
// format's exponent field lands on the lowest bf16 exponent bits: the bf16
// value is then v * 2^(b-127) for every code, subnormal ones included (both
// formats put a zero exponent field in the subnormal binade), and one bf16
// multiply by 2^(127-b) gives v exactly.  A single integer multiply places
// magnitude and sign of two codes 16 bits apart at once (the shifted copies
// never overlap, so there are no carries); the result pairs are
// p[i] = (code i, code i+4), low half first.  9 ALU + 8 FMA-pipe ops.
template <int MANT>
__device__ __forceinline__ void dequant8_exact(uint32_t w, uint32_t p[4]) {
    constexpr int SHIFT = 7 - MANT;
    constexpr uint32_t MUL0 = (1u << SHIFT) + (1u << 12);
    constexpr uint32_t MUL1 = MUL0 >> 4;
    constexpr uint32_t MASK = (0x8000u | (7u << SHIFT)) * 0x10001u;
    constexpr int BIAS = (1 << (2 - MANT)) - 1;
    constexpr uint32_t SC = (uint32_t)((254 - BIAS) << 7) * 0x10001u;  // bf16x2 of 2^(127-b)
    const uint32_t w8 = w >> 8;
    const uint32_t q0 = ((w & 0x000F000Fu) * MUL0) & MASK;
    const uint32_t q1 = ((w & 0x00F000F0u) * MUL1) & MASK;
    const uint32_t q2 = ((w8 & 0x000F000Fu) * MUL0) & MASK;
    const uint32_t q3 = ((w8 & 0x00F000F0u) * MUL1) & MASK;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(p[0]) : "r"(q0), "r"(SC));
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(p[1]) : "r"(q1), "r"(SC));
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(p[2]) : "r"(q2), "r"(SC));
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(p[3]) : "r"(q3), "r"(SC));
}

// Per-half maxima of the finite magnitudes of a bf16x2 word folded into mx2
// (bf16 bit patterns order like the magnitudes; inf and NaN are skipped).
__device__ __forceinline__ uint32_t finite_mag_max2(uint32_t mx2, uint32_t w) {
    const uint32_t a = w & 0x7fff7fffu;  // magnitudes; >= 0x7f80 is inf or NaN
    return __vmaxu2(mx2, a & __vcmpltu2(a, 0x7f807f80u));
}

// Eight bf16 values times a power of two sc -> eight f16 (round to nearest).
__device__ __forceinline__ uint4 bf16x8_to_f16x8(const uint4 v, float sc) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t h[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float lo = __uint_as_float(w[j] << 16) * sc, hi = __uint_as_float(w[j] & 0xffff0000u) * sc;
        asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(h[j]) : "f"(hi), "f"(lo));
    }
    return make_uint4(h[0], h[1], h[2], h[3]);
}

// Output activation of the GEMM epilogue, applied to the finished fp32 value
// y = rho * sum before the bf16 rounding (HiFloat4 page, section 5, fused
// operators: the activation that follows the linear layer runs in the GEMM's
// epilogue).  0: none; 1: SiLU y * sigmoid(y); 2: GeLU y * Phi(y), the erf
// form.
// 3: SiLU-gated pairs (SwiGLU with interleaved weights): rows 2i and 2i+1
// of the weight matrix are the gate and up rows of output column i, and the
// output holds N/2 columns y = silu(y[2i]) * y[2i+1] (silu_gate below).
enum { kActNone = 0, kActSilu = 1, kActGelu = 2, kActSiluGate = 3 };
__device__ __forceinline__ float silu_gate(float g, float u) { return g / (1.f + expf(-g)) * u; }
__device__ __forceinline__ float apply_act(float y, int act) {
    if (act == kActSilu) return y / (1.f + expf(-y));
    if (act == kActGelu) return 0.5f * y * (1.f + erff(y * 0.70710678118654752f));
    return y;
}

// bf16 bit pattern of v, round to nearest even.
__device__ __forceinline__ uint16_t bf16_bits(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }

__device__ __forceinline__ float load_scale(const void* scales, int sdt, size_t idx) {
    if (sdt == FP4_SCALE_F16) return __half2float(__ldg(reinterpret_cast<const __half*>(scales) + idx));
    return __ldg(reinterpret_cast<const float*>(scales) + idx);
}

// ------------------------------------------------------------- PTX: misc
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(pred));
    return pred;
}

// --------------------------------------------------------- PTX: mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.release.cta.shared::cta.b64 st, [%0];\n\t}" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Arrive after shared-memory loads have returned their data.  `dep` must be
// computed from the loaded values and is stored to the calling thread's own
// scratch word `slot` before the arrive: that store cannot issue before the
// loads complete, and the arrive (release) is ordered after it, so the stage
// cannot be released, and overwritten by the next copy, while its loads are
// still in flight.  A plain arrive right after the loads was seen to let that
// happen.
__device__ __forceinline__ void mbar_arrive_after(uint64_t* bar, uint32_t dep, uint32_t* slot) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(smem_u32(slot)), "r"(dep) : "memory");
    mbar_arrive(bar);
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.release.cta.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
            smem_u32(bar)),
        "r"(bytes)
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking test of the phase with the given parity.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait: returns false (and the caller must give up) after
// `timeout_ns` of global time.  Every wait in the library goes through here.
// try_wait with a suspend-time hint: the thread sleeps in hardware until the
// phase completes or about `hint_ns` pass, instead of spinning (polling warps
// would take issue slots from the warps doing the work).
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}
// Bounded wait that sleeps between checks (see mbar_try_wait_hint).
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
        if (globaltimer_ns() - t0 > timeout_ns) return false;
    }
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > timeout_ns) return false;
    }
}

// -------------------------------------------------------------- PTX: TMA
// 2D tiled bulk tensor load global -> shared, completion on an mbarrier.
// No multicast.  c0 = innermost coordinate (elements), c1 = row.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

// Shared-memory accesses by 32-bit shared-window address (explicit ld/st
// .shared, whatever the compiler can infer about a pointer's space).  Not
// volatile: ordering comes from the mbarrier waits and arrives around them.
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ float lds_f32(uint32_t a) {
    float v;
    asm("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ float lds_f16_as_f32(uint32_t a) {
    unsigned short h;
    asm("ld.shared.u16 %0, [%1];" : "=h"(h) : "r"(a) : "memory");
    return __half2float(__ushort_as_half(h));
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
__device__ __forceinline__ void sts_f32(uint32_t a, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}

// cp.async of 4 bytes from global to shared (both 4-byte aligned); only the
// first `src_bytes` (0 or 4) are read, the rest is zero-filled.
__device__ __forceinline__ void cp_async4_zfill(uint32_t dst, const void* src, int src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

// Arrival on an mbarrier when all of this thread's earlier cp.async copies
// have landed; counts as one of the phase's expected arrivals.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// 3D tiled TMA load global -> shared, completion on an mbarrier.  No multicast.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// barrier among `count` threads (a multiple of 32) of the CTA, id 1..15
__device__ __forceinline__ void named_barrier_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// 1D bulk copy global -> shared (16-byte aligned addresses and size),
// completion on an mbarrier.  No multicast.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// Eight E2M1 codes (one 32-bit word, code 2j in the low nibble of byte j)
// -> four f16x2 words by the hardware convert, one instruction per byte:
// q_j = (v(code 2j) low half, v(code 2j+1) high half), exact values.
__device__ __forceinline__ void e2m1_to_f16x8(uint32_t w, uint32_t& q0, uint32_t& q1, uint32_t& q2, uint32_t& q3) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(q0), "=r"(q1), "=r"(q2), "=r"(q3)
        : "r"(w));
}

// Bulk prefetch of a global range into L2 (16-byte aligned address and size).
// L2 is the point of coherence, so a line fetched early still reflects any
// later write: the consumer's real reads, issued after the dependency wait,
// see the producer's data.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------ PTX: programmatic dependent launch
// A kernel launched with programmatic stream serialization may start while
// the previous kernel in the stream is still running: everything before
// pdl_wait() (barrier setup, tensor-memory allocation, descriptor prefetch)
// overlaps it; pdl_wait() returns once that kernel has completed and its
// memory is visible, so every read of an input comes after it.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------- PTX: clusters / DSMEM
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// address of the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_dsmem(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}

__device__ __forceinline__ float4 ld_dsmem_f32x4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

// ---------------------------------------------------------- PTX: tcgen05
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

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 inputs, fp32
// accumulate).  Issued by one thread.
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on an mbarrier once all previously issued tcgen05.mma of this
// thread have completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 32 lanes x 32 bit, 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t r[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::f16, cta_group::1.  A is
// 128 lanes (rows) x 16 k, two 16-bit values per 32-bit column (lower k in
// the low half), at columns a_tmem .. a_tmem + 7.  Issued by one thread.
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 lanes x 32 bit, 32 consecutive columns per thread (register i ->
// column taddr + i of the thread's lane).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t r[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// the calling thread's tensor-memory stores have completed
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 bit, 32 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t r[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// L2 prefetch of one box of a 3-D tiled tensor map.
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap* map, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}

// L2 prefetch of one box of a tiled tensor map (no shared memory, no
// completion mechanism).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int c0, int c1) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1)
                 : "memory");
}

// Shared-memory matrix descriptor, K-major operand with the 128-byte
// swizzle: rows of 128 B, 8-row atoms of 1024 B stacked at a stride of
// 1024 B (SBO), base 1024-byte aligned, descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;            // leading byte offset (unused here)
    d |= (uint64_t)(1024u >> 4) << 32;  // stride byte offset
    d |= (uint64_t)1u << 46;            // version
    d |= (uint64_t)2u << 61;            // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor: kind::f16, A = B = bf16 (K-major), D = fp32,
// shape M x N.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
    return (1u << 4)                       // D format fp32; A and B format f16 (0)
           | ((uint32_t)(N >> 3) << 17)    // N / 8
           | ((uint32_t)(M >> 4) << 24);   // M / 16
}

__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
    return (1u << 4)                       // D format fp32
           | (1u << 7)                     // A format bf16
           | (1u << 10)                    // B format bf16
           | ((uint32_t)(N >> 3) << 17)    // N / 8
           | ((uint32_t)(M >> 4) << 24);   // M / 16
}

}  // namespace fp4
