// gemm_rowblk.cu -- W4A16 GEMM, group 128, M <= 16 tokens, row-block form:
//   Y[m, n] = bf16( rho * sum_g s[n, g] * sum_{k in g} X[m, k] * v(code[n, k]) )
// (LLM-FP4 summary page, efficient matrix multiplication: the 4-bit products
// are formed on the exact code values and each group scale multiplies a
// partial sum.)
//
// Each CTA owns whole 16-row blocks (all of K), so no tile is ever split
// between CTAs and nothing is reduced across them; this makes it the kernel
// of choice when the activations fit shared memory once per CTA.
#include "common.cuh"

namespace fp4 {

struct RbParams {
    const uint16_t* X;
    const uint8_t* packed;
    const void* scales;
    int sdt;
    int M, N, K;
    const float* x_scale;
    uint16_t* Y;
    int act;
};

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

__device__ __forceinline__ void mma_bf16_16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// Group-128 path.  One 128-wide chunk is one group: each chunk accumulates
// the exact code values separately (the mma sums x * v in fp32) and is then
// scaled once by s in fp32, so no weight is rounded.
//
// Memory.  A block is 16 adjacent weight rows x all of K: one contiguous
// piece of the packed matrix, whose 16 rows of group scales are contiguous
// too.  CTAs are persistent and walk the blocks blockIdx.x + i * gridDim.x
// through nbuf shared-memory buffers (2 where they fit): one thread issues
// the next blocks' copies while the warps compute the current one.  Each
// block takes exactly two bulk copies (its codes and its scale rows): a
// bulk copy costs the issuing thread on the order of a hundred cycles, so
// per-row copies would make issue, not HBM, the limit.  Every DRAM request
// is one long contiguous run.  Before its dependency wait (the weights do
// not come from the previous kernel) thread 0 starts all of the CTA's blocks
// towards L2, so the weight stream overlaps the previous kernel's tail.
//
// Activations.  They are staged once per CTA in shared memory, already in
// the operand form of the mma and ordered so that the four lanes sharing a
// token read 64 contiguous bytes; where M * K is too large for that they are
// read from L2 per chunk instead.  Tokens form NT tiles of 8 mma columns
// (NT = 2 for 9 <= M <= 16): each chunk's codes are dequantized once and
// feed every tile's mma.  The warps split K into chunks and reduce their
// fp32 sums in shared memory in warp order (deterministic).
//
// Dequantization:
//  - E2M1: the hardware e2m1x2 -> f16x2 convert, one instruction per two
//    codes; the mma runs in f16 with fp32 accumulation and the activations
//    are converted bf16 -> f32 -> f16 (exact for |x| in the fp16 normal
//    range);
//  - E1M2 / E3M0: exact bf16 by bit placement (dequant8_exact) with the
//    activation pairs rebuilt as (k, k+4) pairs by prmt.
__device__ __forceinline__ void mma_f16_16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bf16x2 -> f16x2 (exact inside the fp16 normal range)
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t x) {
    const float lo = __uint_as_float(x << 16), hi = __uint_as_float(x & 0xffff0000u);
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// 8 bf16 activations (k0..k7 of one 16-byte vector) -> the four B-operand
// registers of that vector: f16 natural pairs for the E2M1 path, bf16
// (k, k+4) pairs matching dequant8_exact for the others.
template <bool kCvt>
__device__ __forceinline__ uint4 x_operand(const uint4 x) {
    if (kCvt)
        return make_uint4(bf16x2_to_f16x2(x.x), bf16x2_to_f16x2(x.y), bf16x2_to_f16x2(x.z), bf16x2_to_f16x2(x.w));
    return make_uint4(prmt(x.x, x.z, 0x5410u), prmt(x.x, x.z, 0x7632u), prmt(x.y, x.w, 0x5410u),
                      prmt(x.y, x.w, 0x7632u));
}

__device__ __forceinline__ uint4 rb_lds(const void* p) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

__device__ __forceinline__ void rb_sts(void* p, const uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(smem_u32(p)), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w));
}

constexpr int kDecMaxK = 24576;  // one buffer of 16 code rows and scale rows must fit shared memory
constexpr int kDecSmemMax = 226 * 1024;
constexpr int kDecMaxBuf = 6;  // block buffers per CTA

// Code rows are dense (one bulk copy per block); activation rows sit at a
// pitch of 64 modulo 128 bytes so that the 8 lanes of a quarter-warp hit 8
// different bank groups.
__host__ __device__ constexpr int dec_pitch(int K) { return K / 2; }
// codes of 16 rows at the padded pitch + their scale rows (room for fp32)
__host__ __device__ constexpr int dec_buf_bytes(int K) { return 16 * dec_pitch(K) + 16 * (K / 128) * 4; }
__host__ __device__ constexpr int dec_xpitch(int K) { return 2 * K + 64; }
// NT = token tiles of 8 (1 for M <= 8, 2 for M <= 16): the reduction buffer
// holds NT partial tiles per warp, double-buffered
__host__ __device__ constexpr int dec_smem_bytes(int K, int M, int nw, int nbuf, bool xs) {
    return nbuf * dec_buf_bytes(K) + (xs ? M * dec_xpitch(K) : 0) + 2 * nw * 32 * 4 * 4 * (M > 8 ? 2 : 1) + 128;
}

template <int MANT, int SDT, int NW, int NT>
__global__ void __launch_bounds__(NW * 32, 16 / NW)
    gemm_rowblk_kernel(RbParams p, int nbuf, int sc_bulk, int* status, unsigned long long timeout_ns) {
    constexpr bool kCvt = MANT == 1;  // E2M1: hardware convert + f16 mma
    constexpr int kEs = SDT == FP4_SCALE_F16 ? 2 : 4;
    extern __shared__ uint8_t dsmem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem_raw) + 127) & ~uintptr_t(127));
    __shared__ __align__(8) uint64_t bar[kDecMaxBuf];  // per buffer: codes and scale rows landed
    __shared__ volatile int abort_flag;
    __shared__ uint32_t row_max[16];  // per token row: largest finite bf16 magnitude (bits)
    __shared__ float row_sc[16], row_f[16];  // its power-of-two scale and the inverse
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int K = p.K, G = K >> 7;
    const int P = dec_pitch(K), SB = dec_buf_bytes(K), XP = dec_xpitch(K);
    uint8_t* xs = base + nbuf * SB;
    float* red = reinterpret_cast<float*>(xs + p.M * XP);  // [2][NT][NW][32][4]
    const int sc_bytes = 16 * G * kEs;  // scale rows of a full block: a multiple of 32 bytes
    const int nblk = (p.N + 15) / 16;
    const int iters = blockIdx.x < nblk ? (nblk - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

    if (threadIdx.x == 0) {
        for (int b = 0; b < nbuf; ++b) mbar_init(&bar[b], 1);
        fence_mbar_init();
        abort_flag = 0;
    }
    if (threadIdx.x < 16) row_max[threadIdx.x] = 0;
    if (threadIdx.x == 0) {
        // start every block of this CTA towards L2 before the dependency wait:
        // the weight stream overlaps the tail of the previous kernel
        for (int it = 0; it < iters; ++it) {
            const int n0 = ((int)blockIdx.x + it * (int)gridDim.x) * 16;
            const int nrows = p.N - n0 < 16 ? p.N - n0 : 16;
            bulk_prefetch_l2(p.packed + (size_t)n0 * (K / 2), (uint32_t)nrows * (uint32_t)(K / 2));
            if (sc_bulk && nrows == 16)
                bulk_prefetch_l2(static_cast<const uint8_t*>(p.scales) + (size_t)n0 * G * kEs, (uint32_t)sc_bytes);
        }
    }
    __syncthreads();

    int issued = 0;  // blocks whose copies were issued (thread 0 only)
    auto issue = [&](int it) {  // bulk copies of block `it` of this CTA into buffer it % nbuf
        const int n0 = ((int)blockIdx.x + it * (int)gridDim.x) * 16;
        const int nrows = p.N - n0 < 16 ? p.N - n0 : 16;
        const int b = it % nbuf;
        uint8_t* buf = base + b * SB;
        // a ragged last block, or an unaligned scale pointer, reads its scales from global memory
        const bool sc = sc_bulk && nrows == 16;
        const uint32_t code_bytes = (uint32_t)nrows * (uint32_t)(K / 2);
        mbar_arrive_expect_tx(&bar[b], code_bytes + (sc ? (uint32_t)sc_bytes : 0u));
        bulk_load(buf, p.packed + (size_t)n0 * (K / 2), code_bytes, &bar[b]);
        if (sc)
            bulk_load(buf + 16 * P, static_cast<const uint8_t*>(p.scales) + (size_t)n0 * G * kEs,
                      (uint32_t)sc_bytes, &bar[b]);
        issued = it + 1;
    };
    // The first buffers' copies go out before the dependency wait as well:
    // codes and scales are inputs that no kernel still running may write
    // (the previous kernel in the stream triggers this launch early only
    // when it is one of these GEMMs), and the buffers are free at entry.
    if (threadIdx.x == 0)
        for (int it = 0; it < nbuf && it < iters; ++it) issue(it);
    pdl_wait();  // the activations, rho and the output may involve the previous kernel
    pdl_launch_dependents();

    {
        // The activations, once per CTA, in operand form at row pitch XP:
        // vector 4t + q of chunk c (lane t's q-th) sits at 16 * (4q + t).
        // E2M1 (f16 MMAs): first the raw bf16 rows and each row's largest
        // finite magnitude, then in place f16 scaled by the power of two that
        // brings that maximum into [2^14, 2^15) (exact for every element
        // within 2^31 of it; the factor is undone in fp32 in the epilogue).
        // Other formats: bf16 re-paired to (k, k+4) order in one pass.
        const int vpr = K >> 3, total = p.M * vpr;
        const uint4* src = reinterpret_cast<const uint4*>(p.X);
        constexpr int kB = 8;  // loads in flight per thread
        int cur = -1;
        uint32_t cmax = 0;
        for (int i0 = threadIdx.x; i0 < total; i0 += kB * NW * 32) {
            uint4 v[kB];
#pragma unroll
            for (int u = 0; u < kB; ++u) {
                const int i = i0 + u * NW * 32;
                if (i < total) v[u] = __ldg(src + i);
            }
#pragma unroll
            for (int u = 0; u < kB; ++u) {
                const int i = i0 + u * NW * 32;
                if (i < total) {
                    const int m = i / vpr, w = i - m * vpr;
                    const int pos = (w & ~15) * 16 + 16 * (4 * (w & 3) + ((w >> 2) & 3));
                    if (kCvt) {
                        rb_sts(xs + m * XP + pos, v[u]);
                        if (m != cur) {
                            if (cur >= 0) atomicMax(&row_max[cur], cmax);
                            cur = m;
                            cmax = 0;
                        }
                        const uint32_t mx2 = finite_mag_max2(
                            finite_mag_max2(finite_mag_max2(finite_mag_max2(0u, v[u].x), v[u].y), v[u].z), v[u].w);
                        cmax = max(cmax, max(mx2 & 0xffffu, mx2 >> 16));
                    } else {
                        rb_sts(xs + m * XP + pos, x_operand<false>(v[u]));
                    }
                }
            }
        }
        if (kCvt) {
            if (cur >= 0) atomicMax(&row_max[cur], cmax);
            __syncthreads();
            if (threadIdx.x < p.M) {
                const uint32_t mx = row_max[threadIdx.x];
                const int E = (int)(mx >> 7);  // biased exponent of the row maximum
                int sh = mx == 0 ? 0 : 141 - (E < 1 ? 1 : E);
                if (sh > 126) sh = 126;
                row_sc[threadIdx.x] = __int_as_float((127 + sh) << 23);
                row_f[threadIdx.x] = __int_as_float((127 - sh) << 23);
            }
            __syncthreads();
            for (int i = threadIdx.x; i < total; i += NW * 32) {
                const int m = i / vpr, w = i - m * vpr;
                uint8_t* d = xs + m * XP + (w & ~15) * 16 + 16 * (4 * (w & 3) + ((w >> 2) & 3));
                rb_sts(d, bf16x8_to_f16x8(rb_lds(d), row_sc[m]));
            }
        }
        __syncthreads();
    }

    const int c_begin = warp * G / NW, c_end = (warp + 1) * G / NW;
    // token 8 tt + g of tile tt's 8 mma columns (columns >= M use token 0 and
    // are never stored)
    const uint8_t* xrow[NT];
#pragma unroll
    for (int tt = 0; tt < NT; ++tt) {
        const int gx = 8 * tt + g < p.M ? 8 * tt + g : 0;
        xrow[tt] = xs + gx * XP + 16 * t;
    }
    const float rho = p.x_scale ? *p.x_scale : 1.f;

    for (int it = 0; it < iters; ++it) {
        const int n0 = ((int)blockIdx.x + it * (int)gridDim.x) * 16;
        const int b = it % nbuf;
        const uint8_t* wsm = base + b * SB;
        const uint8_t* ssm = wsm + 16 * P;
        const uint32_t ph = (uint32_t)(it / nbuf) & 1u;
        const bool sc_smem = sc_bulk && p.N - n0 >= 16;
        auto scale_at = [&](int rl, int c) -> float {  // block row rl, group c
            if (sc_smem) {
                if (SDT == FP4_SCALE_F16)
                    return __half2float(*reinterpret_cast<const __half*>(ssm + 2 * (rl * G + c)));
                return *reinterpret_cast<const float*>(ssm + 4 * (rl * G + c));
            }
            const size_t row = n0 + rl < p.N ? n0 + rl : n0;
            if (SDT == FP4_SCALE_F16)
                return __half2float(__ldg(reinterpret_cast<const __half*>(p.scales) + row * G + c));
            return __ldg(reinterpret_cast<const float*>(p.scales) + row * G + c);
        };
        // decided per warp (vote) before any warp-collective MMA
        bool ok = abort_flag == 0;
        if (c_begin < c_end) ok = __all_sync(0xffffffffu, ok && mbar_wait(&bar[b], ph, timeout_ns));
        if (!ok) abort_flag = 1;

        float acc[NT][4];
#pragma unroll
        for (int tt = 0; tt < NT; ++tt) acc[tt][0] = acc[tt][1] = acc[tt][2] = acc[tt][3] = 0.f;
        for (int c = c_begin; c < c_end && ok; ++c) {
            uint4 xv[NT][4];
#pragma unroll
            for (int tt = 0; tt < NT; ++tt) {
#pragma unroll
                for (int q = 0; q < 4; ++q) xv[tt][q] = rb_lds(xrow[tt] + 256 * c + 64 * q);
            }
            const float sa = scale_at(g, c), sb = scale_at(g + 8, c);
            // this lane's 16 bytes of rows g and g+8 for chunk c: bytes 64c + 16t
            const uint4 wa = rb_lds(wsm + g * P + 64 * c + 16 * t);
            const uint4 wb = rb_lds(wsm + (g + 8) * P + 64 * c + 16 * t);
            float part[NT][4];
#pragma unroll
            for (int tt = 0; tt < NT; ++tt) part[tt][0] = part[tt][1] = part[tt][2] = part[tt][3] = 0.f;
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
                uint32_t qa[4], qb[4];
                if (kCvt) {
                    e2m1_to_f16x8(word_of(wa, wi), qa[0], qa[1], qa[2], qa[3]);
                    e2m1_to_f16x8(word_of(wb, wi), qb[0], qb[1], qb[2], qb[3]);
                } else {
                    dequant8_exact<MANT>(word_of(wa, wi), qa);
                    dequant8_exact<MANT>(word_of(wb, wi), qb);
                }
                // the dequantized A fragment serves every token tile
#pragma unroll
                for (int tt = 0; tt < NT; ++tt) {
                    const uint32_t xb0 = word_of(xv[tt][wi], 0), xb1 = word_of(xv[tt][wi], 1);
                    const uint32_t xb2 = word_of(xv[tt][wi], 2), xb3 = word_of(xv[tt][wi], 3);
                    if (kCvt) {
                        mma_f16_16816(part[tt], qa[0], qb[0], qa[1], qb[1], xb0, xb1);
                        mma_f16_16816(part[tt], qa[2], qb[2], qa[3], qb[3], xb2, xb3);
                    } else {
                        mma_bf16_16816(part[tt], qa[0], qb[0], qa[1], qb[1], xb0, xb1);
                        mma_bf16_16816(part[tt], qa[2], qb[2], qa[3], qb[3], xb2, xb3);
                    }
                }
            }
#pragma unroll
            for (int tt = 0; tt < NT; ++tt) {
                acc[tt][0] = fmaf(sa, part[tt][0], acc[tt][0]);
                acc[tt][1] = fmaf(sa, part[tt][1], acc[tt][1]);
                acc[tt][2] = fmaf(sb, part[tt][2], acc[tt][2]);
                acc[tt][3] = fmaf(sb, part[tt][3], acc[tt][3]);
            }
        }

        // cross-warp reduction in warp order (double-buffered region)
        float* rd = red + (it & 1) * (NT * NW * 32 * 4);
#pragma unroll
        for (int tt = 0; tt < NT; ++tt)
#pragma unroll
            for (int j = 0; j < 4; ++j) rd[((tt * NW + warp) * 32 + lane) * 4 + j] = acc[tt][j];
        __syncthreads();  // every warp is done with this block's buffer and partials
        if (threadIdx.x == 0 && it + nbuf < iters && abort_flag == 0) issue(it + nbuf);
        if (threadIdx.x < 128 * NT) {
            const int tt = threadIdx.x >> 7, e = threadIdx.x & 127, l = e >> 2, j = e & 3;
            float sum = 0.f;
#pragma unroll
            for (int w = 0; w < NW; ++w) sum += rd[((tt * NW + w) * 32 + l) * 4 + j];
            const int n = n0 + (l >> 2) + 8 * (j >> 1), m = 8 * tt + 2 * (l & 3) + (j & 1);
            const float v = rho * (kCvt ? row_f[m] * sum : sum);
            if (p.act == kActSiluGate) {
                // row n ^ 1 (the other half of the gate/up pair) sits in lane ^ 16
                const float w = __shfl_xor_sync(0xffffffffu, v, 16);
                if (m < p.M && n + 1 < p.N && (n & 1) == 0) p.Y[(size_t)m * (p.N >> 1) + (n >> 1)] = bf16_bits(silu_gate(v, w));
            } else if (m < p.M && n < p.N) {
                p.Y[(size_t)m * p.N + n] = bf16_bits(apply_act(v, p.act));
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && abort_flag) {
        raise_status(status, kStatusTimeout);
        // copies still in flight (at most the last nbuf issued blocks: none
        // is issued after an abort) must land before the CTA exits
        for (int it = issued - nbuf < 0 ? 0 : issued - nbuf; it < issued; ++it)
            mbar_wait(&bar[it % nbuf], (uint32_t)(it / nbuf) & 1u, timeout_ns);
    }
}

// Shared-memory plan: two CTAs of 8 warps per SM where they fit, else one
// CTA of 16 warps; two block buffers before one.  The activations are
// always staged (measured: covering every block of a CTA with a buffer,
// e.g. one 16-warp CTA per SM with 5 buffers for 688 blocks, was slower than
// two 8-warp CTAs with two buffers each, whose per-block barriers and
// reductions overlap).  No plan: the shape goes to the streaming kernel.
struct RbPlan {
    int nw, nbuf;
    int smem;
};

static RbPlan rb_plan(int M, int K) {
    if (K > kDecMaxK || M > 16) return {0, 0, 0};
    for (int nbuf = 2; nbuf >= 1; --nbuf) {
        const int s8 = dec_smem_bytes(K, M, 8, nbuf, true);
        if (2 * (s8 + 1024 + 128) <= 228 * 1024) return {8, nbuf, s8};
        const int s16 = dec_smem_bytes(K, M, 16, nbuf, true);
        if (s16 <= kDecSmemMax) return {16, nbuf, s16};
    }
    return {0, 0, 0};
}

template <int MANT, int SDT, int NW, int NT>
static cudaError_t launch_rb_t(const RbParams& p, const RbPlan& plan, int* status, unsigned long long to,
                               cudaStream_t st) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64) return cudaErrorInvalidDevice;
    auto kern = gemm_rowblk_kernel<MANT, SDT, NW, NT>;
    static bool attr_set[64] = {};
    if (!attr_set[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmemMax);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    int per_sm = 0, sms = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NW * 32, plan.smem);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    const int nblk = (p.N + 15) / 16;
    int grid = per_sm * sms;
    if (grid > nblk) grid = nblk;
    // scale rows travel with the codes when the scale pointer allows bulk copies
    const int sc_bulk = (reinterpret_cast<uintptr_t>(p.scales) & 15) == 0 ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(NW * 32, 1, 1);
    cfg.dynamicSmemBytes = (size_t)plan.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p, plan.nbuf, sc_bulk, status, to);
}

template <int MANT, int SDT>
static cudaError_t launch_rb_nw(const RbParams& p, int* status, unsigned long long to, cudaStream_t st) {
    const RbPlan plan = rb_plan(p.M, p.K);
    if (plan.nw == 0) return cudaErrorInvalidValue;
    if (p.M > 8)
        return plan.nw == 8 ? launch_rb_t<MANT, SDT, 8, 2>(p, plan, status, to, st)
                            : launch_rb_t<MANT, SDT, 16, 2>(p, plan, status, to, st);
    return plan.nw == 8 ? launch_rb_t<MANT, SDT, 8, 1>(p, plan, status, to, st)
                        : launch_rb_t<MANT, SDT, 16, 1>(p, plan, status, to, st);
}

// Whether the row-block kernel takes this shape (M <= 16, staged activations).
bool rowblk_fits(int M, int K) { return rb_plan(M, K).nw != 0; }

// Whether the automatic engine should run it: always up to 8 tokens; from 9
// to 16 only with two block buffers (measured: otherwise the tensor engine
// is faster).
bool rowblk_preferred(int M, int K) {
    const RbPlan plan = rb_plan(M, K);
    return plan.nw != 0 && (M <= 8 || plan.nbuf == 2);
}

cudaError_t launch_gemm_rowblk(const uint16_t* X, const uint8_t* packed, const void* scales, int sdt, int fmt,
                               int M, int N, int K, const float* x_scale, uint16_t* Y, int act, int* status,
                               unsigned long long timeout_ns, cudaStream_t st) {
    if (K % 128 != 0 || M <= 0 || N <= 0) return cudaErrorInvalidValue;
    RbParams p{X, packed, scales, sdt, M, N, K, x_scale, Y, act};
    const bool f16 = sdt == FP4_SCALE_F16;
    if (fmt == FP4_E1M2)
        return f16 ? launch_rb_nw<2, FP4_SCALE_F16>(p, status, timeout_ns, st)
                   : launch_rb_nw<2, FP4_SCALE_F32>(p, status, timeout_ns, st);
    if (fmt == FP4_E2M1)
        return f16 ? launch_rb_nw<1, FP4_SCALE_F16>(p, status, timeout_ns, st)
                   : launch_rb_nw<1, FP4_SCALE_F32>(p, status, timeout_ns, st);
    return f16 ? launch_rb_nw<0, FP4_SCALE_F16>(p, status, timeout_ns, st)
               : launch_rb_nw<0, FP4_SCALE_F32>(p, status, timeout_ns, st);
}

}  // namespace fp4
