// quantize.cu -- FP4 (ExMy) weight quantization on sm_100a.
//
// Implements scale-and-clip, compare-and-quantize and the format / range
// search of the LLM-FP4 summary page ("首个支持4-bit浮点量化的LLM来了",
// sections on scale-and-clip, eq. (2)-(4), compare-and-quantize, eq. (5),
// and the search over exponent/mantissa split and quantization range), the
// fold of the pre-shifted exponent bias into the weights (same page), and
// the 2-codes-per-byte packing of the "为什么我们需要4-bit浮点量化" tutorial,
// section 2.2.
//
// Data layout: W is walked as a flat array of N*K fp32 (rows contiguous,
// K % group == 0, so groups never straddle rows).  One warp handles a unit
// of 128 consecutive elements (4 per lane, one 16-byte load per lane), i.e.
// 128/group groups; the group absmax is a shuffle reduction over group/4
// lanes.  The pass is HBM-bound: 4 B read + 0.5 B + (2|4)/group B written
// per weight.
//
// Arithmetic that decides a code is IEEE binary32 with round-to-nearest
// (__fmul_rn / __fdiv_rn, never contracted), so codes and scales are
// bit-identical to the CPU oracle.
#include <cstring>

#include "common.cuh"

namespace fp4 {

constexpr int kQuantThreads = 256;
constexpr int kSearchBlocksMax = 1184;  // fixed (shape-only) grid cap => deterministic SSE order
constexpr int kUnroll = 4;             // units (128 weights) per warp iteration in the packing pass

struct QuantParams {
    const float* W;
    const int8_t* shift;  // [K] or null
    long long total;      // N*K
    int K;
    int group;
    int sdt;
    uint8_t* packed;
    void* scales;
    int* status;
};

__device__ __forceinline__ float pow2i(int e) {  // 2^e for e in [-126, 127], exact
    return __int_as_float((127 + e) << 23);
}

// Load the 4 elements of this lane (folded by 2^shift).  Returns false for
// lanes past the end of the tensor.
__device__ __forceinline__ bool load4(const QuantParams& p, long long base, float w[4]) {
    long long off = base + 4 * (threadIdx.x & 31);
    if (off >= p.total) {
        w[0] = w[1] = w[2] = w[3] = 0.f;
        return false;
    }
    float4 v = __ldg(reinterpret_cast<const float4*>(p.W + off));
    w[0] = v.x;
    w[1] = v.y;
    w[2] = v.z;
    w[3] = v.w;
    if (p.shift) {
        int k0 = (int)(off % p.K);
        char4 s = __ldg(reinterpret_cast<const char4*>(p.shift + k0));
        w[0] = __fmul_rn(w[0], pow2i(s.x));
        w[1] = __fmul_rn(w[1], pow2i(s.y));
        w[2] = __fmul_rn(w[2], pow2i(s.z));
        w[3] = __fmul_rn(w[3], pow2i(s.w));
    }
    return true;
}

// Max over the group/4 lanes that hold one group.
__device__ __forceinline__ float group_absmax(float a, int lanes_per_group) {
    for (int o = 1; o < lanes_per_group; o <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    return a;
}

// Stored scale (fp32, or fp16 round-to-nearest-even widened back) for
// group absmax A, bias factor cj and format maximum qmax.
__device__ __forceinline__ float stored_scale(float A, float cj, float qmax, int sdt, bool* overflow,
                                              uint32_t* raw) {
    float s32 = __fdiv_rn(__fmul_rn(A, cj), qmax);
    if (sdt == FP4_SCALE_F16) {
        __half h = __float2half_rn(s32);
        *raw = __half_as_ushort(h);
        float s = __half2float(h);
        *overflow = isinf(s);
        return s;
    }
    *raw = __float_as_uint(s32);
    *overflow = !isfinite(s32);
    return s32;
}

__device__ __forceinline__ int code_of(float w, float s, const FmtTable& t, float* v_signed) {
    int idx = 0;
    if (s != 0.f) idx = nearest_index(fabsf(__fdiv_rn(w, s)), t);
    const bool neg = signbit(w);
    const float v = t.mag[idx];
    *v_signed = neg ? -v : v;
    return (neg ? 8 : 0) | idx;
}

// Smallest magnitude |x| (fp32) whose quotient fl32(|x|/s) passes a
// nearest-code test with rounding boundary hb (see FmtTables::hb): the test
// is monotone in |x|, and it passes exactly when |x| > hb*s, or |x| == hb*s
// and the tie rounds up.  hb*s is exact in fp64 (25 + 24 significant bits),
// so the threshold equals what the IEEE division followed by the midpoint
// compare decides, with no division per weight.  A zero or non-finite
// scale maps every quotient to index 0 (NaN threshold: no |x| passes).
__device__ __forceinline__ float code_threshold(double hb, bool tie_up, float s) {
    if (!(s > 0.f) || isinf(s)) return __int_as_float(0x7fc00000);
    const double H = hb * (double)s;
    float T = __double2float_ru(H);  // smallest float >= H
    if ((double)T == H && !tie_up) T = __int_as_float(__float_as_int(T) + 1);
    return T;
}

// Fused pass: group absmax -> scale -> codes -> pack, for a fixed
// candidate (format, j) taken from kernel arguments or, when `choice` is
// non-null, from device memory (written by the search).  Optionally
// accumulates SSE per block into ws_sse[block] (fp64).
__global__ void __launch_bounds__(kQuantThreads, 4) quantize_kernel(QuantParams p, FmtTables tabs, int fmt, int j,
                                                                 const int32_t* choice, int32_t* choice_out,
                                                                 double* ws_sse) {
    if (choice) {
        fmt = choice[0];
        j = choice[1];
    }
    const FmtTable& t = tabs.f[fmt];
    const float cj = tabs.cj[j];
    const int lane = threadIdx.x & 31;
    const int lpg = p.group >> 2;  // lanes per group
    const long long units = (p.total + 127) / 128;
    const long long wid = (long long)blockIdx.x * (kQuantThreads / 32) + (threadIdx.x >> 5);
    const long long nw = (long long)gridDim.x * (kQuantThreads / 32);
    if (choice_out && blockIdx.x == 0 && threadIdx.x == 0) {
        choice_out[0] = fmt;
        choice_out[1] = j;
    }
    double sse = 0.0;
    bool bad = false, ovf = false;
    // kUnroll consecutive units per warp iteration: their loads are all in
    // flight before the first one is used
    for (long long u0 = wid * kUnroll; u0 < units; u0 += nw * kUnroll) {
        float w[kUnroll][4];
        bool valid[kUnroll];
#pragma unroll
        for (int q = 0; q < kUnroll; ++q) valid[q] = load4(p, (u0 + q) * 128, w[q]);
#pragma unroll
        for (int q = 0; q < kUnroll; ++q) {
            const long long base = (u0 + q) * 128;
            float a = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                bad |= valid[q] && !isfinite(w[q][i]);
                a = fmaxf(a, fabsf(w[q][i]));
            }
            const float A = group_absmax(a, lpg);
            bool o;
            uint32_t raw;
            const float s = stored_scale(A, cj, t.qmax, p.sdt, &o, &raw);
            // the unit's 7 x (128 / group) thresholds: lane L < 7 * groups
            // computes test L % 7 of group L / 7, then every lane gathers
            // the 7 of its own group
            const int gl = lane / 7, ti = lane - 7 * gl;
            const bool tl = gl < (128 / p.group);
            const float sg = __shfl_sync(0xffffffffu, s, (tl ? gl : 0) * lpg);
            const float myT = tl ? code_threshold(tabs.hb[fmt][ti], (tabs.tie_up[fmt] >> ti) & 1u, sg) : 0.f;
            const int g0 = (lane / lpg) * 7;
            float T[7];
#pragma unroll
            for (int i = 0; i < 7; ++i) T[i] = __shfl_sync(0xffffffffu, myT, g0 + i);
            if (!valid[q]) continue;
            ovf |= o;
            uint32_t codes = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float ax = fabsf(w[q][i]);
                int idx = 0;
#pragma unroll
                for (int k = 0; k < 7; ++k) idx += ax >= T[k] ? 1 : 0;
                const bool neg = signbit(w[q][i]);
                codes |= (uint32_t)((neg ? 8 : 0) | idx) << (4 * i);
                if (ws_sse) {
                    const float v = neg ? -t.mag[idx] : t.mag[idx];
                    const double d = (double)w[q][i] - (double)v * (double)s;
                    sse = fma(d, d, sse);
                }
            }
            const long long off = base + 4 * lane;
            *reinterpret_cast<uint16_t*>(p.packed + off / 2) = (uint16_t)codes;
            if ((lane & (lpg - 1)) == 0) {
                const long long gi = off / p.group;
                if (p.sdt == FP4_SCALE_F16)
                    reinterpret_cast<uint16_t*>(p.scales)[gi] = (uint16_t)raw;
                else
                    reinterpret_cast<uint32_t*>(p.scales)[gi] = raw;
            }
        }
    }
    if (bad) raise_status(p.status, kStatusNonfinite);
    if (ovf) raise_status(p.status, kStatusScaleOverflow);
    if (ws_sse) {
        // fixed-order block reduction: warp shuffles, then warps in order
        __shared__ double red[kQuantThreads / 32];
        for (int o = 16; o > 0; o >>= 1) sse += __shfl_xor_sync(0xffffffffu, sse, o);
        if (lane == 0) red[threadIdx.x >> 5] = sse;
        __syncthreads();
        if (threadIdx.x == 0) {
            double acc = 0.0;
            for (int i = 0; i < kQuantThreads / 32; ++i) acc += red[i];
            ws_sse[blockIdx.x] = acc;
        }
    }
}

// Search pass: for every candidate (f, j) in the set, SSE of quantizing
// the whole tensor with it; per-block fp64 partials into ws[block][24].
// Every element is loaded once and evaluated for all candidates from
// registers (the pass is ALU-bound: one IEEE division per element and
// candidate).
__global__ void __launch_bounds__(kQuantThreads) search_kernel(QuantParams p, FmtTables tabs, int f0, int f1,
                                                               int jn, double* ws) {
    const int lane = threadIdx.x & 31;
    const int lpg = p.group >> 2;
    const long long units = (p.total + 127) / 128;
    const long long wid = (long long)blockIdx.x * (kQuantThreads / 32) + (threadIdx.x >> 5);
    const long long nw = (long long)gridDim.x * (kQuantThreads / 32);
    double sse[24];
#pragma unroll
    for (int c = 0; c < 24; ++c) sse[c] = 0.0;
    bool bad = false;
    for (long long u = wid; u < units; u += nw) {
        float w[4];
        const bool valid = load4(p, u * 128, w);
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            bad |= valid && !isfinite(w[i]);
            a = fmaxf(a, fabsf(w[i]));
        }
        const float A = group_absmax(a, lpg);
        if (!valid) continue;
#pragma unroll
        for (int f = 0; f < 3; ++f) {
            if (f < f0 || f > f1) continue;
            const FmtTable& t = tabs.f[f];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (j >= jn) continue;
                bool o;
                uint32_t raw;
                const float s = stored_scale(A, tabs.cj[j], t.qmax, p.sdt, &o, &raw);
                double acc = 0.0;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float v;
                    code_of(w[i], s, t, &v);
                    const double d = (double)w[i] - (double)v * (double)s;
                    acc = fma(d, d, acc);
                }
                sse[f * 8 + j] += acc;
            }
        }
    }
    if (bad) raise_status(p.status, kStatusNonfinite);
    __shared__ double red[kQuantThreads / 32][24];
#pragma unroll
    for (int c = 0; c < 24; ++c) {
        double v = sse[c];
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[threadIdx.x >> 5][c] = v;
    }
    __syncthreads();
    if (threadIdx.x < 24) {
        double acc = 0.0;
        for (int i = 0; i < kQuantThreads / 32; ++i) acc += red[i][threadIdx.x];
        ws[(size_t)blockIdx.x * 24 + threadIdx.x] = acc;
    }
}

// Sum the per-block partials in block order, pick the first strict minimum
// in (format, j) order, write choice and sse (NaN for candidates outside
// the searched set).  One block.
__global__ void search_finalize_kernel(const double* ws, int nblocks, int f0, int f1, int jn, int32_t* choice,
                                       double* sse_out) {
    __shared__ double tot[24];
    const int c = threadIdx.x;
    if (c < 24) {
        double acc = 0.0;
        for (int b = 0; b < nblocks; ++b) acc += ws[(size_t)b * 24 + c];
        tot[c] = acc;
    }
    __syncthreads();
    if (c == 0) {
        int bf = f0, bj = 0;
        double best = INFINITY;
        for (int f = f0; f <= f1; ++f)
            for (int j = 0; j < jn; ++j)
                if (tot[f * 8 + j] < best) {
                    best = tot[f * 8 + j];
                    bf = f;
                    bj = j;
                }
        if (choice) {
            choice[0] = bf;
            choice[1] = bj;
        }
        if (sse_out) {
            for (int f = 0; f < 3; ++f)
                for (int j = 0; j < 8; ++j) {
                    const bool in = f >= f0 && f <= f1 && j < jn;
                    sse_out[f * 8 + j] = in ? tot[f * 8 + j] : __longlong_as_double(0x7ff8000000000000LL);
                }
        }
    }
}

// SSE of a single fixed candidate (no search): per-block partials written
// by quantize_kernel, summed in block order.
__global__ void sse_single_finalize_kernel(const double* ws, int nblocks, int fmt, int j, double* sse_out) {
    if (threadIdx.x != 0) return;
    double acc = 0.0;
    for (int b = 0; b < nblocks; ++b) acc += ws[b];
    for (int c = 0; c < 24; ++c) sse_out[c] = __longlong_as_double(0x7ff8000000000000LL);
    sse_out[fmt * 8 + j] = acc;
}

// ------------------------------------------------------ scale granularity
// The absmax behind a scale is taken over a block: g elements of a row
// (group, as in quantize_kernel), a whole row (output channel) or
// rows_per_block consecutive rows (one attention head); the block's scale
// goes into every group slot it covers, so the GEMM reads the usual
// [N][K/group] layout.  Channel and head blocks need K % 128 == 0: a
// 128-element unit then lies in one row, hence in one block.  With a bias
// search each block takes the index j with the smallest SSE over its own
// elements (first strict minimum); the format stays the tensor's.

struct BlkParams {
    QuantParams q;
    int gran;             // FP4_GRAN_*
    int rows_per_block;   // channel: 1, head: N / heads
    const float* blockA;  // [blocks] absmax of W' per channel / head block
    const int8_t* jsel;   // [blocks] bias index per channel / head block, or null
    int8_t* jmap;         // [blocks] out: bias index per group block, or null
    int j;                // fixed bias index, or -1: per-group search
};

__device__ __forceinline__ float warp_max(float a) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    return a;
}

// Butterfly sum over the whole warp: every lane ends with the same bits
// (each step adds a pair in both orders, and IEEE addition commutes).
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Channel / head blocks: absmax of W' per block (float bits of a
// non-negative value order like unsigned integers: atomicMax on the bits).
__global__ void __launch_bounds__(kQuantThreads) block_absmax_kernel(QuantParams p, int rows_per_block,
                                                                     unsigned* blockA) {
    const int lane = threadIdx.x & 31;
    const long long units = p.total / 128;
    const long long wid = (long long)blockIdx.x * (kQuantThreads / 32) + (threadIdx.x >> 5);
    const long long nw = (long long)gridDim.x * (kQuantThreads / 32);
    bool bad = false;
    for (long long u = wid; u < units; u += nw) {
        float w[4];
        load4(p, u * 128, w);
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            bad |= !isfinite(w[i]);
            a = fmaxf(a, fabsf(w[i]));
        }
        a = warp_max(a);
        if (lane == 0) atomicMax(&blockA[(int)((u * 128) / p.K) / rows_per_block], __float_as_uint(a));
    }
    if (bad) raise_status(p.status, kStatusNonfinite);
}

// Channel / head blocks with a bias search: the 8 candidates' SSE of every
// 128-element unit, usse[unit][j] (summed per block in unit order below,
// so the choice does not depend on timing).
__global__ void __launch_bounds__(kQuantThreads) block_sse_kernel(QuantParams p, FmtTables tabs, int fmt,
                                                                  int rows_per_block, const float* blockA,
                                                                  double* usse) {
    const FmtTable& t = tabs.f[fmt];
    const int lane = threadIdx.x & 31;
    const long long units = p.total / 128;
    const long long wid = (long long)blockIdx.x * (kQuantThreads / 32) + (threadIdx.x >> 5);
    const long long nw = (long long)gridDim.x * (kQuantThreads / 32);
    for (long long u = wid; u < units; u += nw) {
        float w[4];
        load4(p, u * 128, w);
        const float A = blockA[(int)((u * 128) / p.K) / rows_per_block];
#pragma unroll 1
        for (int jj = 0; jj < 8; ++jj) {
            bool o;
            uint32_t raw;
            const float s = stored_scale(A, tabs.cj[jj], t.qmax, p.sdt, &o, &raw);
            double acc = 0.0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float v;
                code_of(w[i], s, t, &v);
                const double d = (double)w[i] - (double)v * (double)s;
                acc = fma(d, d, acc);
            }
            acc = warp_sum(acc);
            if (lane == jj) usse[u * 8 + jj] = acc;
        }
    }
}

// One warp per channel / head block: its units' SSE summed in a fixed
// order, then the first strict minimum over j.
__global__ void block_choose_kernel(const double* usse, long long units_per_block, int nblocks, int8_t* jsel) {
    const int lane = threadIdx.x & 31;
    const int b = (int)(((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    if (b >= nblocks) return;  // whole warps leave together
    double e[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) e[jj] = 0.0;
    for (long long v = lane; v < units_per_block; v += 32) {
        const double* row = usse + ((long long)b * units_per_block + v) * 8;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) e[jj] += row[jj];
    }
    int best = 0;
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
        e[jj] = warp_sum(e[jj]);
        if (e[jj] < e[best]) best = jj;
    }
    if (lane == 0) jsel[b] = (int8_t)best;
}

// Codes and scales for every granularity: the group absmax or the block's
// precomputed one, a fixed, chosen or (group blocks) searched bias index,
// then scale-and-clip, compare-and-quantize and packing as in
// quantize_kernel.
__global__ void __launch_bounds__(kQuantThreads) quantize_blocks_kernel(BlkParams bp, FmtTables tabs, int fmt) {
    const QuantParams& p = bp.q;
    const FmtTable& t = tabs.f[fmt];
    const int lane = threadIdx.x & 31;
    const int lpg = p.group >> 2;
    const long long units = (p.total + 127) / 128;
    const long long wid = (long long)blockIdx.x * (kQuantThreads / 32) + (threadIdx.x >> 5);
    const long long nw = (long long)gridDim.x * (kQuantThreads / 32);
    bool bad = false, ovf = false;
    for (long long u = wid; u < units; u += nw) {
        float w[4];
        const bool valid = load4(p, u * 128, w);
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            bad |= valid && !isfinite(w[i]);
            a = fmaxf(a, fabsf(w[i]));
        }
        const float Ag = group_absmax(a, lpg);
        const long long off = u * 128 + 4 * lane;
        long long blk;
        float A;
        if (bp.gran == FP4_GRAN_GROUP) {
            blk = off / p.group;
            A = Ag;
        } else {
            blk = valid ? (off / p.K) / bp.rows_per_block : 0;
            A = valid ? bp.blockA[blk] : 0.f;
        }
        int j = bp.j;
        if (j < 0 && bp.jsel) {
            j = valid ? bp.jsel[blk] : 0;
        } else if (j < 0) {
            // per-group search: the group's SSE for every candidate (a sum
            // over its lanes, identical bits in all of them)
            double best = 0.0;
            j = 0;
#pragma unroll 1
            for (int jj = 0; jj < 8; ++jj) {
                bool o;
                uint32_t raw;
                const float s = stored_scale(A, tabs.cj[jj], t.qmax, p.sdt, &o, &raw);
                double acc = 0.0;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float v;
                    code_of(w[i], s, t, &v);
                    const double d = (double)w[i] - (double)v * (double)s;
                    acc = fma(d, d, acc);
                }
                for (int o2 = 1; o2 < lpg; o2 <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o2);
                if (jj == 0 || acc < best) {
                    best = acc;
                    j = jj;
                }
            }
        }
        if (!valid) continue;
        bool o;
        uint32_t raw;
        const float s = stored_scale(A, tabs.cj[j], t.qmax, p.sdt, &o, &raw);
        ovf |= o;
        uint32_t codes = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float v;
            codes |= (uint32_t)code_of(w[i], s, t, &v) << (4 * i);
        }
        *reinterpret_cast<uint16_t*>(p.packed + off / 2) = (uint16_t)codes;
        if ((lane & (lpg - 1)) == 0) {
            const long long gi = off / p.group;
            if (p.sdt == FP4_SCALE_F16)
                reinterpret_cast<uint16_t*>(p.scales)[gi] = (uint16_t)raw;
            else
                reinterpret_cast<uint32_t*>(p.scales)[gi] = raw;
            if (bp.jmap && bp.gran == FP4_GRAN_GROUP) bp.jmap[blk] = (int8_t)j;
        }
    }
    if (bad) raise_status(p.status, kStatusNonfinite);
    if (ovf) raise_status(p.status, kStatusScaleOverflow);
}

// ------------------------------------------------------ 4-bit activations
// Codes of X' = X * 2^-shift[k] against one per-tensor scale
// s_a = fl32(fl32(rho * c_j) / Qmax) (the per-channel power of two of the
// pre-shifted exponent bias lives in the weights).  Eight elements per
// thread: one 16-byte load of X, one 4-byte store of codes.  The nearest-
// code decisions use the exact thresholds of code_threshold (no division
// per element).  HBM-bound: 2 B read + 0.5 B written per element.
__global__ void __launch_bounds__(256) act_quantize_kernel(const uint4* __restrict__ X, long long nvec, int K,
                                                           const int8_t* __restrict__ shift,
                                                           const float* __restrict__ rho, FmtTables tabs, int fmt,
                                                           int j, uint32_t* __restrict__ packed, float* a_scale,
                                                           int* status) {
    const FmtTable& t = tabs.f[fmt];
    const float r = *rho;
    const bool rho_ok = r > 0.f && isfinite(r);
    const float s = __fdiv_rn(__fmul_rn(r, tabs.cj[j]), t.qmax);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        *a_scale = rho_ok ? s : __int_as_float(0x7fc00000);
        if (!rho_ok) raise_status(status, kStatusNonfinite);
    }
    float T[7];
#pragma unroll
    for (int i = 0; i < 7; ++i) T[i] = code_threshold(tabs.hb[fmt][i], (tabs.tie_up[fmt] >> i) & 1u, s);
    bool bad = false;
    for (long long v = (long long)blockIdx.x * blockDim.x + threadIdx.x; v < nvec;
         v += (long long)gridDim.x * blockDim.x) {
        const uint4 x = __ldg(X + v);
        const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
        int8_t e[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (shift) {
            const uint2 sh = __ldg(reinterpret_cast<const uint2*>(shift + (v * 8) % K));
            const uint32_t shw[2] = {sh.x, sh.y};
#pragma unroll
            for (int i = 0; i < 8; ++i) e[i] = (int8_t)(shw[i >> 2] >> (8 * (i & 3)));
        }
        uint32_t codes = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float xv = __uint_as_float((i & 1) ? (xw[i >> 1] & 0xffff0000u) : (xw[i >> 1] << 16));
            bad |= !isfinite(xv);
            if (shift) xv = __fmul_rn(xv, pow2i(-(int)e[i]));
            const float ax = fabsf(xv);
            int idx = 0;
#pragma unroll
            for (int k = 0; k < 7; ++k) idx += ax >= T[k] ? 1 : 0;
            codes |= (uint32_t)((signbit(xv) ? 8 : 0) | idx) << (4 * i);
        }
        packed[v] = codes;
    }
    if (bad) raise_status(status, kStatusNonfinite);
}

// The values of 4-bit activation codes as bf16 (exact: every magnitude of
// the three formats has at most 3 significant bits), for the 16-bit tensor
// path of the W4A4 product.  Eight codes per thread: a 4-byte load, a
// 16-byte store.
struct CodeTable16 {
    uint16_t v[16];
};

__global__ void __launch_bounds__(256) act_expand_kernel(const uint32_t* __restrict__ codes, long long nwords,
                                                         CodeTable16 tab, uint4* __restrict__ out) {
    __shared__ uint16_t tv[16];
    if (threadIdx.x < 16) tv[threadIdx.x] = tab.v[threadIdx.x];
    __syncthreads();
    pdl_launch_dependents();
    pdl_wait();  // the codes may come from the previous kernel in the stream
    for (long long w = (long long)blockIdx.x * blockDim.x + threadIdx.x; w < nwords;
         w += (long long)gridDim.x * blockDim.x) {
        const uint32_t c = __ldg(codes + w);
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            o[i] = (uint32_t)tv[(c >> (8 * i)) & 15] | ((uint32_t)tv[(c >> (8 * i + 4)) & 15] << 16);
        out[w] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// ----------------------------------------------------------- host launch

int quantize_grid_blocks(long long total) {
    const long long units = (total + 127) / 128;
    long long blocks = (units + (kQuantThreads / 32) - 1) / (kQuantThreads / 32);
    if (blocks > kSearchBlocksMax) blocks = kSearchBlocksMax;
    if (blocks < 1) blocks = 1;
    return (int)blocks;
}

size_t quantize_ws_bytes(long long total, bool search, bool want_sse) {
    if (!search && !want_sse) return 0;
    return (size_t)quantize_grid_blocks(total) * 24 * sizeof(double);
}

// Launched after the packing pass.  The GEMM kernels start copying packed
// codes and scales before the kernel ahead of them in the stream has
// finished (programmatic dependent launch); with this empty launch in
// between, a GEMM that follows fp4_quantize directly reads codes whose
// kernel completed a full kernel boundary earlier.
__global__ void stream_boundary_kernel() {}

cudaError_t launch_quantize(const float* W, int N, int K, int group, int fmt, int bias_search,
                            const int8_t* shift, int sdt, uint8_t* packed, void* scales, int32_t* choice,
                            double* sse, void* ws, const FmtTables& tabs, int* status, cudaStream_t st) {
    QuantParams p;
    p.W = W;
    p.shift = shift;
    p.total = (long long)N * K;
    p.K = K;
    p.group = group;
    p.sdt = sdt;
    p.packed = packed;
    p.scales = scales;
    p.status = status;
    const int f0 = fmt < 0 ? 0 : fmt, f1 = fmt < 0 ? 2 : fmt;
    const int jn = bias_search ? 8 : 1;
    const bool search = (f0 != f1) || jn > 1;
    const int blocks = quantize_grid_blocks(p.total);
    // the packing pass takes kUnroll units per warp iteration
    const long long pack_units = ((p.total + 127) / 128 + kUnroll - 1) / kUnroll;
    int pblocks = (int)((pack_units + (kQuantThreads / 32) - 1) / (kQuantThreads / 32));
    pblocks = pblocks < 1 ? 1 : (pblocks > kSearchBlocksMax ? kSearchBlocksMax : pblocks);
    double* wsd = reinterpret_cast<double*>(ws);
    if (search) {
        search_kernel<<<blocks, kQuantThreads, 0, st>>>(p, tabs, f0, f1, jn, wsd);
        search_finalize_kernel<<<1, 32, 0, st>>>(wsd, blocks, f0, f1, jn, choice, sse);
        quantize_kernel<<<pblocks, kQuantThreads, 0, st>>>(p, tabs, 0, 0, choice, nullptr, nullptr);
    } else {
        quantize_kernel<<<pblocks, kQuantThreads, 0, st>>>(p, tabs, f0, 0, nullptr, choice, sse ? wsd : nullptr);
        if (sse) sse_single_finalize_kernel<<<1, 32, 0, st>>>(wsd, pblocks, f0, 0, sse);
    }
    stream_boundary_kernel<<<1, 32, 0, st>>>();
    return cudaGetLastError();
}

// --------------------------------------------------------------- dequant
// W_hat[n,k] = fl32(v(code) * s): one thread per 8 elements (one 32-bit
// word of codes).
__global__ void dequantize_kernel(const uint32_t* packed, const void* scales, int sdt, FmtTable t,
                                  long long words, int K, int group, float* out) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < words;
         i += (long long)gridDim.x * blockDim.x) {
        const uint32_t w = packed[i];
        const long long e0 = i * 8;
        const long long row = e0 / K;
        const int k0 = (int)(e0 % K);
        const int G = K / group;
        const float s = load_scale(scales, sdt, (size_t)row * G + k0 / group);
        float r[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int c = (w >> (4 * q)) & 15;
            const float v = t.mag[c & 7];
            r[q] = __fmul_rn((c & 8) ? -v : v, s);
        }
        float4* o = reinterpret_cast<float4*>(out + e0);
        o[0] = make_float4(r[0], r[1], r[2], r[3]);
        o[1] = make_float4(r[4], r[5], r[6], r[7]);
    }
}

cudaError_t launch_dequantize(const uint8_t* packed, const void* scales, int sdt, const FmtTable& t, int N,
                              int K, int group, float* out, cudaStream_t st) {
    const long long words = (long long)N * K / 8;
    long long blocks = (words + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    dequantize_kernel<<<(int)blocks, 256, 0, st>>>(reinterpret_cast<const uint32_t*>(packed), scales, sdt, t,
                                                   words, K, group, out);
    return cudaGetLastError();
}


// ------------------------------------------- granularity / activations: host

static long long blk_count(int N, int K, int group, int gran, int heads) {
    if (gran == FP4_GRAN_GROUP) return (long long)N * (K / group);
    return gran == FP4_GRAN_CHANNEL ? N : heads;
}

static size_t up256(size_t b) { return (b + 255) & ~(size_t)255; }

size_t quantize_blocks_ws_bytes(int N, int K, int group, int gran, int heads, bool search) {
    if (gran == FP4_GRAN_GROUP || (long long)N * K == 0) return 0;
    const long long nb = blk_count(N, K, group, gran, heads);
    size_t b = up256((size_t)nb * 4);
    if (search) b += up256((size_t)N * K / 128 * 8 * sizeof(double)) + up256((size_t)nb);
    return b;
}

cudaError_t launch_quantize_blocks(const float* W, int N, int K, int group, int gran, int heads, int fmt, int j,
                                   const int8_t* shift, int sdt, uint8_t* packed, void* scales, int8_t* jmap,
                                   void* ws, const FmtTables& tabs, int* status, cudaStream_t st) {
    BlkParams bp;
    QuantParams& p = bp.q;
    p.W = W;
    p.shift = shift;
    p.total = (long long)N * K;
    p.K = K;
    p.group = group;
    p.sdt = sdt;
    p.packed = packed;
    p.scales = scales;
    p.status = status;
    bp.gran = gran;
    bp.rows_per_block = gran == FP4_GRAN_HEAD ? N / heads : 1;
    bp.blockA = nullptr;
    bp.jsel = nullptr;
    bp.jmap = jmap;
    bp.j = j;
    const long long nb = blk_count(N, K, group, gran, heads);
    const int blocks = quantize_grid_blocks(p.total);
    cudaError_t e = cudaSuccess;
    if (gran != FP4_GRAN_GROUP) {
        uint8_t* w8 = static_cast<uint8_t*>(ws);
        float* blockA = reinterpret_cast<float*>(w8);
        e = cudaMemsetAsync(blockA, 0, (size_t)nb * 4, st);
        if (e != cudaSuccess) return e;
        block_absmax_kernel<<<blocks, kQuantThreads, 0, st>>>(p, bp.rows_per_block, reinterpret_cast<unsigned*>(blockA));
        bp.blockA = blockA;
        if (j < 0) {
            double* usse = reinterpret_cast<double*>(w8 + up256((size_t)nb * 4));
            int8_t* jsel = jmap ? jmap
                                : reinterpret_cast<int8_t*>(w8 + up256((size_t)nb * 4) +
                                                            up256((size_t)p.total / 128 * 8 * sizeof(double)));
            block_sse_kernel<<<blocks, kQuantThreads, 0, st>>>(p, tabs, fmt, bp.rows_per_block, blockA, usse);
            const long long upb = (long long)bp.rows_per_block * (K / 128);
            block_choose_kernel<<<(int)((nb * 32 + 255) / 256), 256, 0, st>>>(usse, upb, (int)nb, jsel);
            bp.jsel = jsel;
            bp.jmap = nullptr;
        } else if (jmap) {
            e = cudaMemsetAsync(jmap, j, (size_t)nb, st);
            if (e != cudaSuccess) return e;
            bp.jmap = nullptr;
        }
    }
    quantize_blocks_kernel<<<blocks, kQuantThreads, 0, st>>>(bp, tabs, fmt);
    stream_boundary_kernel<<<1, 32, 0, st>>>();
    return cudaGetLastError();
}

cudaError_t launch_act_quantize(const uint16_t* X, int M, int K, const int8_t* shift, const float* rho,
                                const FmtTables& tabs, int fmt, int j, uint8_t* packed, float* a_scale, int* status,
                                cudaStream_t st) {
    const long long nvec = (long long)M * K / 8;
    long long blocks = (nvec + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (blocks < 1) blocks = 1;
    act_quantize_kernel<<<(int)blocks, 256, 0, st>>>(reinterpret_cast<const uint4*>(X), nvec, K, shift, rho, tabs, fmt,
                                                      j, reinterpret_cast<uint32_t*>(packed), a_scale, status);
    return cudaGetLastError();
}

cudaError_t launch_act_expand(const uint8_t* codes, long long count, const FmtTable& t, uint16_t* out,
                              cudaStream_t st) {
    CodeTable16 tab;
    for (int c = 0; c < 16; ++c) {
        const float v = (c & 8) ? -t.mag[c & 7] : t.mag[c & 7];
        uint32_t b;
        memcpy(&b, &v, 4);
        tab.v[c] = (uint16_t)(b >> 16);  // exact: at most 3 significant bits
    }
    const long long nwords = count / 8;
    long long blocks = (nwords + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (blocks < 1) blocks = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, act_expand_kernel, reinterpret_cast<const uint32_t*>(codes), nwords, tab,
                                       reinterpret_cast<uint4*>(out));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace fp4
