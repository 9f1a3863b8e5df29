// gemm_w4a4.cu -- the W4A4 product with both operands in E2M1, on the
// 5th-generation tensor cores with no dequantization step.
//
//   Y[m,n] = bf16( act( s_a * sum_g s[n,g] * sum_{k in g} v(a[m,k]) * v(w[n,k]) ) )
//
// (LLM-FP4 summary page "首个支持4-bit浮点量化的LLM来了": efficient matrix
// multiplication, the scale factors taken out of the low-bit product; the
// activations quantized with the pre-shifted exponent bias.)
//
// The packed codes of both operands go from global memory to shared memory
// by TMA with the 16 x U4 / 16-byte-aligned element type: every 16 codes
// (8 bytes) land in a 16-byte slot, the layout `tcgen05.mma kind::f8f6f4`
// reads for 4-bit operands, so a 128-k stage is a K-major tile of 128-byte
// rows under the 128-byte swizzle, exactly like an 8-bit operand.  One
// thread issues four K = 32 MMAs per stage (E2M1 x E2M1, fp32 accumulate)
// into the stage's own TMEM accumulator.  Every product of two E2M1 values
// is a multiple of 1/4 below 36, so a group's 128-term sum is exact in
// fp32; fold warps then add s[n,g] * acc to fp32 totals, as in the W4A16
// tensor engine, and the epilogue multiplies by s_a.
//
// Tiles of 128 weight rows x 256 tokens (N = 256 MMAs read half the
// shared-memory operand bytes per flop of a 128-token tile, whose operand
// reads matched the MMA rate) with four copy stages and two 256-column
// accumulators; 128-token tiles for M <= 128 with six stages and four.
// The accumulators fill all 512 TMEM columns.
//
// Warp roles (2 + NF warps, one CTA per SM):
//   warp 0   TMA producer: the first ring-full of weight codes before the
//            dependency wait, activation codes after it;
//   warp 1   TMEM allocator and MMA issuer;
//   warps 2+ fold warps: 4 TMEM lane quadrants x BT/64 column blocks.
// Every wait is bounded (FP4_DEV_WAIT_TIMEOUT); no TMA multicast.
#include "common.cuh"

namespace fp4 {

bool encode_2d_u4(CUtensorMap* map, const void* base, uint64_t elems, uint64_t rows, uint32_t box_rows);

struct W4Params {
    const void* scales;
    int sdt;
    int M, N, K;
    const float* a_scale;
    uint16_t* Y;
    int act;
    int* status;
    unsigned long long timeout_ns;
};

template <int BT>
struct W4Cfg {
    static constexpr int BW = 128;               // weight rows per tile (MMA M)
    static constexpr int KB = 128;               // k per stage = one group
    static constexpr int ABYTES = BW * KB;       // weight codes in shared memory (one byte per code)
    static constexpr int BBYTES = BT * KB;       // activation codes in shared memory
    static constexpr int TX = (BW + BT) * KB / 2;  // bytes the two copies deliver (packed codes)
    static constexpr int SST = BT == 256 ? 4 : 6;  // shared-memory stages (copies in flight)
    static constexpr int ACC = 512 / BT;         // TMEM accumulators (all 512 columns)
    static constexpr int FCOLS = 64;             // accumulator columns per fold thread
    static constexpr int LDB = BT == 256 ? 16 : 64;  // TMEM columns loaded per wait (register budget)
    static constexpr int NF = 4 * (BT / FCOLS);  // fold warps
    static constexpr int FW0 = 2;
    static constexpr int THREADS = (FW0 + NF) * 32;
    static constexpr int TMEM_COLS = ACC * BT;
    static constexpr int NBAR = 2 * SST + 2 * ACC;
    static constexpr int SMEM = SST * (ABYTES + BBYTES) + 1024 + NBAR * 8 + 16;
    static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM allocation is a power of two");
    static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

// Instruction descriptor: kind::f8f6f4, A = B = E2M1 (format 5), K-major,
// D = fp32, shape M x N.
__host__ __device__ constexpr uint32_t idesc_e2m1_f32(int M, int N) {
    return (1u << 4)                      // D format fp32
           | (5u << 7)                    // A format E2M1
           | (5u << 10)                   // B format E2M1
           | ((uint32_t)(N >> 3) << 17)   // N / 8
           | ((uint32_t)(M >> 4) << 24);  // M / 16
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f8f6f4, K = 32.
__device__ __forceinline__ void tc_mma_f8f6f4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

template <int BT>
__global__ void __launch_bounds__(W4Cfg<BT>::THREADS, 1)
    gemm_w4a4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW, W4Params p) {
    using C = W4Cfg<BT>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ws = smem;                      // SST x ABYTES: weight codes
    uint8_t* xs = ws + C::SST * C::ABYTES;   // SST x BBYTES: activation codes
    uint64_t* bars = reinterpret_cast<uint64_t*>(xs + C::SST * C::BBYTES);
    uint64_t* full = bars;                   // [SST] both tiles of the stage landed
    uint64_t* sfree = full + C::SST;         // [SST] the stage's MMAs have read it
    uint64_t* kdone = sfree + C::SST;        // [ACC] the accumulator's MMAs completed
    uint64_t* gempty = kdone + C::ACC;       // [ACC] accumulator folded
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gempty + C::ACC);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * C::BW, m0 = blockIdx.y * BT;
    const int nkb = p.K / C::KB;
    const uint64_t to = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::SST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&sfree[s], 1);
        }
        for (int a = 0; a < C::ACC; ++a) {
            mbar_init(&kdone[a], 1);
            mbar_init(&gempty[a], C::NF);
        }
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmW);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // weight codes are not written by a kernel still running (see the
    // stream-order rule of the interface), so the first ring-full of them
    // goes out before the dependency wait
    const int pre = nkb < C::SST ? nkb : C::SST;
    if (warp == 0 && elect_one()) {
        for (int j = 0; j < pre; ++j) {
            mbar_arrive_expect_tx(&full[j], C::TX);
            tma_load_2d(ws + j * C::ABYTES, &tmW, j * C::KB, n0, &full[j]);
        }
    }
    __syncwarp();
    pdl_wait();  // the activation codes, s_a and the output involve the previous kernel
    pdl_launch_dependents();

    if (warp == 0) {
        // -------------------------------------------------------- producer
        if (elect_one()) {
            for (int j = 0; j < pre; ++j) tma_load_2d(xs + j * C::BBYTES, &tmA, j * C::KB, m0, &full[j]);
            int issued = pre;
            for (int i = pre; i < nkb; ++i) {
                const int s = i % C::SST;
                // the stage's previous MMAs have read it
                if (!mbar_wait(&sfree[s], (uint32_t)((i / C::SST) - 1) & 1u, to)) {
                    raise_status(p.status, kStatusTimeout);
                    break;
                }
                mbar_arrive_expect_tx(&full[s], C::TX);
                tma_load_2d(ws + s * C::ABYTES, &tmW, i * C::KB, n0, &full[s]);
                tma_load_2d(xs + s * C::BBYTES, &tmA, i * C::KB, m0, &full[s]);
                issued = i + 1;
            }
            // no copy may still be in flight when the CTA leaves
            for (int i = issued - C::SST < 0 ? 0 : issued - C::SST; i < issued; ++i)
                if (!mbar_wait(&full[i % C::SST], (uint32_t)(i / C::SST) & 1u, to)) {
                    raise_status(p.status, kStatusTimeout);
                    break;
                }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ----------------------------------------------------- MMA issuer
        if (elect_one()) {
            const uint32_t idesc = idesc_e2m1_f32(C::BW, BT);
            const uint64_t wdesc0 = sw128_desc(smem_u32(ws)), xdesc0 = sw128_desc(smem_u32(xs));
            constexpr uint32_t kWStep = C::ABYTES >> 4, kXStep = C::BBYTES >> 4;
            int committed = 0;
            for (int i = 0; i < nkb; ++i) {
                const int s = i % C::SST, a = i % C::ACC;
                if (!mbar_wait(&full[s], (uint32_t)(i / C::SST) & 1u, to) ||
                    !mbar_wait(&gempty[a], ((uint32_t)(i / C::ACC) & 1u) ^ 1u, to)) {
                    raise_status(p.status, kStatusTimeout);
                    break;
                }
                tc_fence_after();
                const uint64_t wd = wdesc0 + (uint64_t)(s * kWStep);
                const uint64_t xd = xdesc0 + (uint64_t)(s * kXStep);
                const uint32_t d = tmem + (uint32_t)(a * BT);
                // K = 32 codes = 32 bytes of each 128-byte row per MMA
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc_mma_f8f6f4(d, wd + (uint64_t)(2 * kk), xd + (uint64_t)(2 * kk), idesc, kk ? 1u : 0u);
                tc_commit(&sfree[s]);
                tc_commit(&kdone[a]);
                ++committed;
            }
            // TMEM is freed below: the last commit must have landed
            if (committed > 0) {
                const int last = committed - 1;
                if (!mbar_wait(&kdone[last % C::ACC], (uint32_t)(last / C::ACC) & 1u, to))
                    raise_status(p.status, kStatusTimeout);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------- fold + epilogue
        const int fw = warp - C::FW0;
        const int q = warp & 3;                // TMEM lane quadrant of this warp
        const int cb = (fw >> 2) * C::FCOLS;   // first accumulator column of this thread
        const int r = q * 32 + lane;           // weight row within the tile == TMEM lane
        const int n = n0 + r;
        const bool nvalid = n < p.N;
        const float sa = *p.a_scale;
        float tot[C::FCOLS];
#pragma unroll
        for (int j = 0; j < C::FCOLS; ++j) tot[j] = 0.f;
        const uint32_t tlane = tmem + ((uint32_t)(q * 32) << 16);
        bool ok = true;
        float s_next = (nvalid && nkb > 0) ? load_scale(p.scales, p.sdt, (size_t)n * nkb) : 0.f;
        for (int i = 0; i < nkb; ++i) {
            const int s = i % C::ACC;
            const float sc = s_next;
            if (i + 1 < nkb) s_next = nvalid ? load_scale(p.scales, p.sdt, (size_t)n * nkb + i + 1) : 0.f;
            // the warp decides together: the TMEM loads are warp-collective
            if (!__all_sync(0xffffffffu, mbar_wait(&kdone[s], (uint32_t)(i / C::ACC) & 1u, to))) {
                raise_status(p.status, kStatusTimeout);
                ok = false;
                break;
            }
            tc_fence_after();
            // LDB columns in flight per wait
#pragma unroll
            for (int c0 = 0; c0 < C::FCOLS; c0 += C::LDB) {
                uint32_t v[C::LDB];
#pragma unroll
                for (int c = 0; c < C::LDB; c += 16) tmem_ld16(tlane + (uint32_t)(s * BT + cb + c0 + c), v + c);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < C::LDB; ++j) tot[c0 + j] = fmaf(sc, __uint_as_float(v[j]), tot[c0 + j]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&gempty[s]);
        }
        if (ok && p.act == kActSiluGate) {
            // row n ^ 1, the other half of the gate/up pair, is lane ^ 1
#pragma unroll
            for (int j = 0; j < C::FCOLS; ++j) {
                const int m = m0 + cb + j;
                const float v = sa * tot[j];
                const float w = __shfl_xor_sync(0xffffffffu, v, 1);
                if (m < p.M && (n & 1) == 0 && n + 1 < p.N)
                    p.Y[(size_t)m * (p.N >> 1) + (n >> 1)] = bf16_bits(silu_gate(v, w));
            }
        } else if (ok && nvalid) {
#pragma unroll
            for (int j = 0; j < C::FCOLS; ++j) {
                const int m = m0 + cb + j;
                if (m < p.M) p.Y[(size_t)m * p.N + n] = bf16_bits(apply_act(sa * tot[j], p.act));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ----------------------------------------------------------- host launch

// Whether the native path applies: E2M1 x E2M1 at group 128, K a multiple
// of 128 (the 4-bit copy's row length rule), both code arrays 32-byte
// aligned (its base-address rule).
bool w4a4_native_fits(int afmt, int fmt, int M, int N, int K, int group, const void* apacked,
                      const void* packed) {
    (void)N;
    return afmt == FP4_E2M1 && fmt == FP4_E2M1 && group == 128 && K % 128 == 0 && M > 64 &&
           (reinterpret_cast<uintptr_t>(apacked) & 31) == 0 && (reinterpret_cast<uintptr_t>(packed) & 31) == 0;
}

template <int BT>
static cudaError_t launch_w4a4_bt(const uint8_t* apacked, const float* a_scale, const uint8_t* packed,
                                  const void* scales, int sdt, int M, int N, int K, uint16_t* Y, int act, int* status,
                                  unsigned long long timeout_ns, cudaStream_t st) {
    using C = W4Cfg<BT>;
    CUtensorMap ma, mw;
    if (!encode_2d_u4(&ma, apacked, (uint64_t)K, (uint64_t)M, BT)) return cudaErrorInvalidValue;
    if (!encode_2d_u4(&mw, packed, (uint64_t)K, (uint64_t)N, C::BW)) return cudaErrorInvalidValue;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        e = cudaFuncSetAttribute(gemm_w4a4_kernel<BT>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    W4Params p;
    p.scales = scales;
    p.sdt = sdt;
    p.M = M;
    p.N = N;
    p.K = K;
    p.a_scale = a_scale;
    p.Y = Y;
    p.act = act;
    p.status = status;
    p.timeout_ns = timeout_ns;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((N + C::BW - 1) / C::BW, (M + BT - 1) / BT, 1);
    cfg.blockDim = dim3(C::THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, gemm_w4a4_kernel<BT>, ma, mw, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// 256-token tiles (N = 256 MMAs: half the shared-memory operand reads per
// flop of the 128-token tile) once M fills them; 128 below.
cudaError_t launch_gemm_w4a4(const uint8_t* apacked, const float* a_scale, const uint8_t* packed, const void* scales,
                             int sdt, int M, int N, int K, uint16_t* Y, int act, int* status,
                             unsigned long long timeout_ns, cudaStream_t st) {
    if (M > 128)
        return launch_w4a4_bt<256>(apacked, a_scale, packed, scales, sdt, M, N, K, Y, act, status, timeout_ns, st);
    return launch_w4a4_bt<128>(apacked, a_scale, packed, scales, sdt, M, N, K, Y, act, status, timeout_ns, st);
}

}  // namespace fp4
