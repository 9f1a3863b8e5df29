// gemm_decode.cu -- W4A16 GEMM for skinny activations (M <= 8) on sm_100a.
//
// Y[m,n] = bf16( rho * sum_k X[m,k] * v(code[n,k]) * s[n, k/g] )
// (LLM-FP4 summary page "首个支持4-bit浮点量化的LLM来了", efficient matrix
// multiplication: the per-group scales stay outside the 4-bit products.)
//
// Decode is bound by streaming the packed weights from HBM (0.5 B per
// weight plus the scales).  Design:
//  - a CTA owns 16*R weight rows and all of K; its 8 warps split K in
//    128-element chunks and reduce their fp32 partial sums in shared memory
//    (fixed order, no workspace, deterministic);
//  - each lane issues 16-byte coalesced loads of packed codes (32 codes);
//    chunk c+1 is loaded while chunk c is computed;
//  - codes become bf16 in registers through a 16-entry byte-plane LUT held
//    in four registers (prmt), ~2 integer ops per weight;
//  - the products run on the tensor cores as mma.m16n8k16 (bf16 in, fp32
//    accumulate) with the weights as the 16-row A operand and the <= 8
//    activation rows as the 8-column B operand.  The k order inside a chunk
//    is permuted identically for A and B so that every lane's A fragment
//    comes straight out of its own 16-byte load;
//  - group 128: the LUT holds the exact code values, each chunk (= one
//    group) accumulates separately and is scaled once in fp32;
//    group 32/64: the LUT holds bf16(v * s) of the lane's own group.
#include "common.cuh"

namespace fp4 {

struct DecodeParams {
    const uint16_t* X;
    const uint8_t* packed;
    const void* scales;
    int sdt;
    FmtTable t;
    int M, N, K, group;
    const float* x_scale;
    uint16_t* Y;
};

__device__ __forceinline__ void mma_bf16_16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int R>
struct ChunkRegs {
    uint4 wa[R], wb[R];  // packed codes of rows g and g+8 of each 16-row tile
    uint4 x[4];          // 32 bf16 activations of token g
    float sa[R], sb[R];  // group scales of those rows
};

template <int R>
__device__ __forceinline__ void load_chunk(const DecodeParams& p, int n0, int c, int g, int t, ChunkRegs<R>& cr) {
    const int kt = c * 128 + 32 * t;
    const bool kv = kt < p.K;
    const int G = p.K / p.group;
    const size_t rowbytes = (size_t)p.K >> 1;
    if (kv && g < p.M) {
        const uint4* xp = reinterpret_cast<const uint4*>(p.X + (size_t)g * p.K + kt);
#pragma unroll
        for (int i = 0; i < 4; ++i) cr.x[i] = __ldg(xp + i);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) cr.x[i] = make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int na = n0 + 16 * r + g, nb = na + 8;
        const bool va = kv && na < p.N, vb = kv && nb < p.N;
        cr.wa[r] = va ? __ldg(reinterpret_cast<const uint4*>(p.packed + (size_t)na * rowbytes + (kt >> 1)))
                      : make_uint4(0, 0, 0, 0);
        cr.wb[r] = vb ? __ldg(reinterpret_cast<const uint4*>(p.packed + (size_t)nb * rowbytes + (kt >> 1)))
                      : make_uint4(0, 0, 0, 0);
        const int gi = kt / p.group;
        cr.sa[r] = va ? load_scale(p.scales, p.sdt, (size_t)na * G + gi) : 0.f;
        cr.sb[r] = vb ? load_scale(p.scales, p.sdt, (size_t)nb * G + gi) : 0.f;
    }
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

template <int R, bool kScaleInLut>
__global__ void __launch_bounds__(256) gemm_decode_kernel(DecodeParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int n0 = blockIdx.x * 16 * R;
    const int nchunks = (p.K + 127) >> 7;
    const int c_begin = warp * nchunks / 8, c_end = (warp + 1) * nchunks / 8;

    const Bf16Lut lut1 = make_lut(p.t.mag, 1.f);
    float acc[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0.f;

    ChunkRegs<R> cur, nxt;
    if (c_begin < c_end) load_chunk<R>(p, n0, c_begin, g, t, cur);
    for (int c = c_begin; c < c_end; ++c) {
        if (c + 1 < c_end) load_chunk<R>(p, n0, c + 1, g, t, nxt);
        uint32_t xw[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            xw[4 * i + 0] = cur.x[i].x;
            xw[4 * i + 1] = cur.x[i].y;
            xw[4 * i + 2] = cur.x[i].z;
            xw[4 * i + 3] = cur.x[i].w;
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float part[4] = {0.f, 0.f, 0.f, 0.f};
            float* dst = kScaleInLut ? acc[r] : part;
            Bf16Lut la = lut1, lb = lut1;
            if (kScaleInLut) {
                la = make_lut(p.t.mag, cur.sa[r]);
                lb = make_lut(p.t.mag, cur.sb[r]);
            }
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
                uint32_t pa[4], pb[4];
                dequant8(word_of(cur.wa[r], wi), la, pa);
                dequant8(word_of(cur.wb[r], wi), lb, pb);
                mma_bf16_16816(dst, pa[0], pb[0], pa[1], pb[1], xw[4 * wi + 0], xw[4 * wi + 1]);
                mma_bf16_16816(dst, pa[2], pb[2], pa[3], pb[3], xw[4 * wi + 2], xw[4 * wi + 3]);
            }
            if (!kScaleInLut) {
                acc[r][0] = fmaf(cur.sa[r], part[0], acc[r][0]);
                acc[r][1] = fmaf(cur.sa[r], part[1], acc[r][1]);
                acc[r][2] = fmaf(cur.sb[r], part[2], acc[r][2]);
                acc[r][3] = fmaf(cur.sb[r], part[3], acc[r][3]);
            }
        }
        cur = nxt;
    }

    // cross-warp reduction in warp order, then the epilogue
    __shared__ float red[8][R][32][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int j = 0; j < 4; ++j) red[warp][r][lane][j] = acc[r][j];
    __syncthreads();
    const float rho = p.x_scale ? *p.x_scale : 1.f;
    for (int e = threadIdx.x; e < R * 128; e += 256) {
        const int r = e >> 7, l = (e >> 2) & 31, j = e & 3;
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) s += red[w][r][l][j];
        const int n = n0 + 16 * r + (l >> 2) + 8 * (j >> 1);
        const int m = 2 * (l & 3) + (j & 1);
        if (m < p.M && n < p.N) {
            __nv_bfloat16 y = __float2bfloat16_rn(rho * s);
            p.Y[(size_t)m * p.N + n] = *reinterpret_cast<uint16_t*>(&y);
        }
    }
}

// ---------------------------------------------------------------------------
// Group-128 path.  One 128-wide chunk is one group: each chunk accumulates
// the exact code values separately (the mma sums x * v in fp32) and is then
// scaled once by s in fp32, so no weight is rounded.
//
// Memory: each warp owns a ring of kStages shared-memory stages filled by
// TMA (its elected lane issues the copies): per chunk the R x 16 x 64-byte
// packed-code tile and the activation tile (M rows x 128 k as two 128-byte
// swizzled boxes).  A warp keeps kStages chunks in flight without holding
// them in registers, which is what streaming HBM needs.
//
// Dequantization (the instruction count per weight decides decode speed):
//  - E2M1: the hardware e2m1x2 -> f16x2 convert, one instruction per two
//    codes; the mma runs in f16 with fp32 accumulation, so the activations
//    are converted bf16 -> f32 -> f16 in registers (exact for |x| in the fp16
//    normal range, shared by the R row tiles of the warp);
//  - E1M2 / E3M0: exact bf16 by bit placement (dequant8_exact) with the
//    activation pairs rebuilt as (k, k+4) pairs by prmt.
constexpr int kWarpsPerCta = 8;

template <int R>
struct DecodeRing {
    static constexpr int STAGES = R == 1 ? 4 : 3;
    static constexpr int XBYTES = 2048;          // two 1 KB swizzled activation halves
    static constexpr int WBYTES = R * 1024;      // R x 16 rows x 64 bytes of codes
    static constexpr int STAGE = XBYTES + WBYTES;
    static constexpr int SMEM = kWarpsPerCta * STAGES * STAGE + 1024 + kWarpsPerCta * STAGES * 8;
};

__device__ __forceinline__ void mma_f16_16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 8 E2M1 codes (one word, low nibble first) -> 4 f16x2 natural pairs
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

// bf16x2 -> f16x2 (exact inside the fp16 normal range)
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t x) {
    const float lo = __uint_as_float(x << 16), hi = __uint_as_float(x & 0xffff0000u);
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

template <int R, int MANT, int SDT>
__global__ void __launch_bounds__(256, 2)
    gemm_decode_g128_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                            DecodeParams p, int* status, unsigned long long timeout_ns) {
    using RG = DecodeRing<R>;
    constexpr bool kCvt = MANT == 1;  // E2M1: hardware convert + f16 mma
    extern __shared__ uint8_t dsmem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    uint8_t* ring = smem + warp * RG::STAGES * RG::STAGE;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kWarpsPerCta * RG::STAGES * RG::STAGE) + warp * RG::STAGES;

    const int n0 = blockIdx.x * 16 * R;
    const int nchunks = (p.K + 127) >> 7;
    const int c_begin = warp * nchunks / kWarpsPerCta, c_end = (warp + 1) * nchunks / kWarpsPerCta;
    const int mrows = p.M < 8 ? p.M : 8;
    const uint32_t tx_bytes = (uint32_t)RG::WBYTES + 2u * 128u * (uint32_t)mrows;

    // activation rows >= M are never loaded: zero them once so that the
    // unused mma columns stay finite
    for (int i = lane; i < RG::STAGES * (RG::XBYTES / 4); i += 32) {
        const int st = i / (RG::XBYTES / 4), rem = i % (RG::XBYTES / 4);
        reinterpret_cast<uint32_t*>(ring + st * RG::STAGE)[rem] = 0u;
    }
    if (lane == 0) {
        for (int s = 0; s < RG::STAGES; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
    fence_proxy_async_smem();
    __syncwarp();
    pdl_wait();  // inputs may come from the previous kernel in the stream
    pdl_launch_dependents();

    if (lane == 0) {
        for (int c = c_begin; c < c_end && c < c_begin + RG::STAGES; ++c) {
            const int s = c - c_begin;
            uint8_t* st = ring + s * RG::STAGE;
            mbar_arrive_expect_tx(&full[s], tx_bytes);
            tma_load_2d(st, &tmX, c * 128, 0, &full[s]);
            tma_load_2d(st + 1024, &tmX, c * 128 + 64, 0, &full[s]);
            tma_load_2d(st + RG::XBYTES, &tmW, c * 64, n0, &full[s]);
        }
    }

    // scales of rows g and g+8 of each tile (rows past N read row 0; never stored)
    const int G = p.K >> 7;
    int rows[2 * R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int na = n0 + 16 * r + g, nb = na + 8;
        rows[2 * r] = na < p.N ? na : 0;
        rows[2 * r + 1] = nb < p.N ? nb : 0;
    }
    auto scale_at = [&](int row, int c) -> float {
        if (SDT == FP4_SCALE_F16)
            return __half2float(__ldg(reinterpret_cast<const __half*>(p.scales) + (size_t)row * G + c));
        return __ldg(reinterpret_cast<const float*>(p.scales) + (size_t)row * G + c);
    };
    float sc[2 * R];
#pragma unroll
    for (int i = 0; i < 2 * R; ++i) sc[i] = c_begin < c_end ? scale_at(rows[i], c_begin) : 0.f;

    float acc[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0.f;
    bool ok = true;
    for (int c = c_begin; c < c_end; ++c) {
        const int s = (c - c_begin) % RG::STAGES;
        const uint32_t ph = (uint32_t)((c - c_begin) / RG::STAGES) & 1u;
        float sn[2 * R];
#pragma unroll
        for (int i = 0; i < 2 * R; ++i) sn[i] = c + 1 < c_end ? scale_at(rows[i], c + 1) : 0.f;
        if (!mbar_wait(&full[s], ph, timeout_ns)) {
            ok = false;
            break;
        }
        const uint8_t* st = ring + s * RG::STAGE;
        // activations of token g, k = 32t .. 32t+31: half t/2, 16-byte chunks
        // (t&1)*4 + i stored at chunk ^ (g & 7) (128-byte swizzle)
        const uint8_t* xrow = st + (t >> 1) * 1024 + g * 128;
        uint32_t xb[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 x = *reinterpret_cast<const uint4*>(xrow + ((((t & 1) * 4 + i) ^ (g & 7)) << 4));
            if (kCvt) {
                xb[4 * i + 0] = bf16x2_to_f16x2(x.x);
                xb[4 * i + 1] = bf16x2_to_f16x2(x.y);
                xb[4 * i + 2] = bf16x2_to_f16x2(x.z);
                xb[4 * i + 3] = bf16x2_to_f16x2(x.w);
            } else {
                xb[4 * i + 0] = prmt(x.x, x.z, 0x5410u);  // (k0, k4)
                xb[4 * i + 1] = prmt(x.x, x.z, 0x7632u);  // (k1, k5)
                xb[4 * i + 2] = prmt(x.y, x.w, 0x5410u);  // (k2, k6)
                xb[4 * i + 3] = prmt(x.y, x.w, 0x7632u);  // (k3, k7)
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const uint8_t* wt = st + RG::XBYTES + r * 1024;
            const uint4 wa = *reinterpret_cast<const uint4*>(wt + g * 64 + 16 * t);
            const uint4 wb = *reinterpret_cast<const uint4*>(wt + (g + 8) * 64 + 16 * t);
            float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
                uint32_t qa[4], qb[4];
                if (kCvt) {
                    e2m1_to_f16x8(word_of(wa, wi), qa[0], qa[1], qa[2], qa[3]);
                    e2m1_to_f16x8(word_of(wb, wi), qb[0], qb[1], qb[2], qb[3]);
                    mma_f16_16816(part, qa[0], qb[0], qa[1], qb[1], xb[4 * wi + 0], xb[4 * wi + 1]);
                    mma_f16_16816(part, qa[2], qb[2], qa[3], qb[3], xb[4 * wi + 2], xb[4 * wi + 3]);
                } else {
                    dequant8_exact<MANT>(word_of(wa, wi), qa);
                    dequant8_exact<MANT>(word_of(wb, wi), qb);
                    mma_bf16_16816(part, qa[0], qb[0], qa[1], qb[1], xb[4 * wi + 0], xb[4 * wi + 1]);
                    mma_bf16_16816(part, qa[2], qb[2], qa[3], qb[3], xb[4 * wi + 2], xb[4 * wi + 3]);
                }
            }
            acc[r][0] = fmaf(sc[2 * r], part[0], acc[r][0]);
            acc[r][1] = fmaf(sc[2 * r], part[1], acc[r][1]);
            acc[r][2] = fmaf(sc[2 * r + 1], part[2], acc[r][2]);
            acc[r][3] = fmaf(sc[2 * r + 1], part[3], acc[r][3]);
        }
#pragma unroll
        for (int i = 0; i < 2 * R; ++i) sc[i] = sn[i];
        __syncwarp();  // every lane has consumed the stage
        if (lane == 0 && c + RG::STAGES < c_end) {
            const int cn = c + RG::STAGES;
            uint8_t* stn = ring + s * RG::STAGE;
            mbar_arrive_expect_tx(&full[s], tx_bytes);
            tma_load_2d(stn, &tmX, cn * 128, 0, &full[s]);
            tma_load_2d(stn + 1024, &tmX, cn * 128 + 64, 0, &full[s]);
            tma_load_2d(stn + RG::XBYTES, &tmW, cn * 64, n0, &full[s]);
        }
    }
    if (!ok && lane == 0) {
        raise_status(status, kStatusTimeout);
        // copies still in flight must land before the CTA exits
        for (int c = c_end - RG::STAGES > c_begin ? c_end - RG::STAGES : c_begin; c < c_end; ++c) {
            const int s = (c - c_begin) % RG::STAGES;
            mbar_wait(&full[s], (uint32_t)((c - c_begin) / RG::STAGES) & 1u, timeout_ns);
        }
    }

    // cross-warp reduction in warp order (reusing the ring), then the epilogue
    __syncthreads();
    float* red = reinterpret_cast<float*>(smem);  // [8 warps][R][32][4]
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int j = 0; j < 4; ++j) red[((warp * R + r) * 32 + lane) * 4 + j] = acc[r][j];
    __syncthreads();
    const float rho = p.x_scale ? *p.x_scale : 1.f;
    for (int e = threadIdx.x; e < R * 128; e += 256) {
        const int r = e >> 7, l = (e >> 2) & 31, j = e & 3;
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kWarpsPerCta; ++w) sum += red[((w * R + r) * 32 + l) * 4 + j];
        const int n = n0 + 16 * r + (l >> 2) + 8 * (j >> 1);
        const int m = 2 * (l & 3) + (j & 1);
        if (m < p.M && n < p.N) {
            __nv_bfloat16 y = __float2bfloat16_rn(rho * sum);
            p.Y[(size_t)m * p.N + n] = *reinterpret_cast<uint16_t*>(&y);
        }
    }
}

// Rows per CTA = 16 * R; two row tiles share each activation conversion,
// one keeps enough CTAs for narrow matrices.
int decode_rows_per_cta(int N) { return N >= 8192 ? 2 : 1; }

bool encode_2d(CUtensorMap* map, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t inner,
               uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw);

template <int R, int MANT, int SDT>
static cudaError_t launch_g128_t(const CUtensorMap& mw, const CUtensorMap& mx, const DecodeParams& p, int* status,
                                 unsigned long long to, cudaStream_t st) {
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(gemm_decode_g128_kernel<R, MANT, SDT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, DecodeRing<R>::SMEM);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((p.N + 16 * R - 1) / (16 * R), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.dynamicSmemBytes = DecodeRing<R>::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemm_decode_g128_kernel<R, MANT, SDT>, mw, mx, p, status, to);
}

template <int R>
static cudaError_t launch_g128_r(const DecodeParams& p, int fmt, int* status, unsigned long long to,
                                 cudaStream_t st) {
    CUtensorMap mw, mx;
    const int mrows = p.M < 8 ? p.M : 8;
    if (!encode_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.packed, (uint64_t)p.K / 2, (uint64_t)p.N, 64,
                   (uint32_t)(16 * R), CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    if (!encode_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.X, (uint64_t)p.K, (uint64_t)p.M, 64, (uint32_t)mrows,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const bool f16 = p.sdt == FP4_SCALE_F16;
    if (fmt == FP4_E1M2)
        return f16 ? launch_g128_t<R, 2, FP4_SCALE_F16>(mw, mx, p, status, to, st)
                   : launch_g128_t<R, 2, FP4_SCALE_F32>(mw, mx, p, status, to, st);
    if (fmt == FP4_E2M1)
        return f16 ? launch_g128_t<R, 1, FP4_SCALE_F16>(mw, mx, p, status, to, st)
                   : launch_g128_t<R, 1, FP4_SCALE_F32>(mw, mx, p, status, to, st);
    return f16 ? launch_g128_t<R, 0, FP4_SCALE_F16>(mw, mx, p, status, to, st)
               : launch_g128_t<R, 0, FP4_SCALE_F32>(mw, mx, p, status, to, st);
}

cudaError_t launch_gemm_decode(const uint16_t* X, const uint8_t* packed, const void* scales, int sdt,
                               const FmtTable& t, int fmt, int M, int N, int K, int group, const float* x_scale,
                               uint16_t* Y, int* status, unsigned long long timeout_ns, cudaStream_t st) {
    DecodeParams p{X, packed, scales, sdt, t, M, N, K, group, x_scale, Y};
    if (group == 128)
        return decode_rows_per_cta(N) == 1 ? launch_g128_r<1>(p, fmt, status, timeout_ns, st)
                                           : launch_g128_r<2>(p, fmt, status, timeout_ns, st);
    const int R = decode_rows_per_cta(N);
    const int blocks = (N + 16 * R - 1) / (16 * R);
    if (R == 1)
        gemm_decode_kernel<1, true><<<blocks, 256, 0, st>>>(p);
    else
        gemm_decode_kernel<2, true><<<blocks, 256, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace fp4
