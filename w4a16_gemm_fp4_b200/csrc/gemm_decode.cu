// gemm_decode.cu -- W4A16 GEMM for skinny activations on sm_100a at groups
// of 32 and 64 (M <= 8): the per-lane-LUT kernel.  Group 128 runs on the
// tensor-memory engine of gemm_ts.cu at every M <= 64.
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
    int act;
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
            __nv_bfloat16 y = __float2bfloat16_rn(apply_act(rho * s, p.act));
            p.Y[(size_t)m * p.N + n] = *reinterpret_cast<uint16_t*>(&y);
        }
    }
}

// Rows per CTA of the group-32/64 kernel (16 * R).
int decode_rows_per_cta(int N) { return N >= 8192 ? 2 : 1; }

// Largest M the per-lane-LUT kernel takes: one 8-token MMA tile.
int decode_max_m_lut() { return 8; }

cudaError_t launch_gemm_decode(const uint16_t* X, const uint8_t* packed, const void* scales, int sdt,
                               const FmtTable& t, int M, int N, int K, int group, const float* x_scale, uint16_t* Y,
                               int act, cudaStream_t st) {
    DecodeParams p{X, packed, scales, sdt, t, M, N, K, group, x_scale, Y, act};
    if (M > decode_max_m_lut()) return cudaErrorInvalidValue;
    const int R = decode_rows_per_cta(N);
    const int blocks = (N + 16 * R - 1) / (16 * R);
    if (R == 1)
        gemm_decode_kernel<1, true><<<blocks, 256, 0, st>>>(p);
    else
        gemm_decode_kernel<2, true><<<blocks, 256, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace fp4
