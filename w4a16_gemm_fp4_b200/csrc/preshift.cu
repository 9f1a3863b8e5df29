// preshift.cu -- pre-shifted exponent bias on sm_100a (LLM-FP4 summary page
// "首个支持4-bit浮点量化的LLM来了", section on the pre-shifted exponent
// bias): per-channel activation maxima from calibration data are split into
// one per-tensor real factor rho and a per-channel power of two 2^e_k; the
// power of two is folded into the weights (quantize.cu), rho stays on the
// activations and is re-applied in the GEMM epilogue.
//
//   c_k  = max_m |X[m,k]|,  rho = max_k c_k (1 if X == 0)
//   e_k  = ceil(log2(c_k / rho)) in [-126, 0]  (exact, from binary exponents)
//   X~   = bf16_rne(fl32(fl32(X * 2^-e_k) / rho))
//
// All three passes are HBM-bound streams over X (bf16, 16-byte vectors).
#include "common.cuh"

#include <atomic>

namespace fp4 {

constexpr int kColsPerBlock = 512;  // 256 threads x 2 bf16 columns

// Partial column maxima over a slab of rows: part[slab][k].
__global__ void __launch_bounds__(256) colmax_kernel(const uint16_t* X, int M, int K, int rows_per_slab,
                                                     float* part, int* status) {
    const int k = blockIdx.x * kColsPerBlock + 2 * threadIdx.x;
    const int slab = blockIdx.y;
    const int m0 = slab * rows_per_slab;
    const int m1 = min(M, m0 + rows_per_slab);
    if (k >= K) return;
    float a0 = 0.f, a1 = 0.f;
    bool bad = false;
    const uint32_t* src = reinterpret_cast<const uint32_t*>(X);
    for (int m = m0; m < m1; ++m) {
        const uint32_t v = __ldg(src + (((size_t)m * K + k) >> 1));
        const float x0 = __uint_as_float(v << 16), x1 = __uint_as_float(v & 0xffff0000u);
        bad |= !isfinite(x0) || !isfinite(x1);
        a0 = fmaxf(a0, fabsf(x0));
        a1 = fmaxf(a1, fabsf(x1));
    }
    if (bad) raise_status(status, kStatusNonfinite);
    part[(size_t)slab * K + k] = a0;
    part[(size_t)slab * K + k + 1] = a1;
}

// One block: c_k = max over slabs, rho = max_k c_k, then e_k.
__global__ void __launch_bounds__(1024) calib_finalize_kernel(float* part, int slabs, int K, int8_t* shift,
                                                              float* rho_out) {
    __shared__ float red[32];
    __shared__ float rho_s;
    float mx = 0.f;
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
        float c = part[k];
        for (int s = 1; s < slabs; ++s) c = fmaxf(c, part[(size_t)s * K + k]);
        part[k] = c;
        mx = fmaxf(mx, c);
    }
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        float r = 0.f;
        for (int i = 0; i < (int)(blockDim.x >> 5); ++i) r = fmaxf(r, red[i]);
        if (r == 0.f) r = 1.f;
        rho_s = r;
        *rho_out = r;
    }
    __syncthreads();
    const float rho = rho_s;
    int q2;
    const float f2 = frexpf(rho, &q2);
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
        const float c = part[k];
        int e = 0;
        if (c > 0.f) {
            int q1;
            const float f1 = frexpf(c, &q1);
            e = q1 - q2 + (f1 > f2 ? 1 : 0);
            e = max(-126, min(0, e));
        }
        shift[k] = (int8_t)e;
    }
}

// X~ = bf16(fl32(fl32(X * 2^-e_k) / rho)), 8 elements (16 B) per thread.
__global__ void __launch_bounds__(256) preshift_apply_kernel(const uint4* X, long long vecs, int K,
                                                             const int8_t* shift, const float* rho_p, uint4* Xt) {
    const float rho = *rho_p;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < vecs;
         i += (long long)gridDim.x * blockDim.x) {
        const uint4 v = __ldg(X + i);
        const int k0 = (int)((i * 8) % K);
        const uint2 sh = __ldg(reinterpret_cast<const uint2*>(shift + k0));
        const uint32_t in[4] = {v.x, v.y, v.z, v.w};
        const uint32_t sw[2] = {sh.x, sh.y};
        uint32_t out[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float r[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float x = __uint_as_float(h ? (in[q] & 0xffff0000u) : (in[q] << 16));
                const int e = (int)(int8_t)((sw[q >> 1] >> (8 * ((2 * q + h) & 3))) & 0xff);
                const float p = __int_as_float((127 - e) << 23);  // 2^-e, e in [-126, 0]
                r[h] = __fdiv_rn(__fmul_rn(x, p), rho);
            }
            out[q] = pack_bf16x2(r[0], r[1]);
        }
        Xt[i] = make_uint4(out[0], out[1], out[2], out[3]);
    }
}

int calib_slabs(int M, int K) {
    const int colblocks = (K + kColsPerBlock - 1) / kColsPerBlock;
    int slabs = (2 * 148 + colblocks - 1) / colblocks;
    slabs = max(1, min(slabs, max(1, M / 16)));
    return slabs;
}

size_t preshift_ws_bytes(int M, int K) { return (size_t)calib_slabs(M, K) * K * sizeof(float); }

cudaError_t launch_calibrate(const uint16_t* X, int M, int K, int8_t* shift, float* rho, void* ws, int* status,
                             cudaStream_t st) {
    const int slabs = calib_slabs(M, K);
    const int rows = (M + slabs - 1) / slabs;
    dim3 grid((K + kColsPerBlock - 1) / kColsPerBlock, slabs);
    float* part = reinterpret_cast<float*>(ws);
    colmax_kernel<<<grid, 256, 0, st>>>(X, M, K, rows, part, status);
    calib_finalize_kernel<<<1, 1024, 0, st>>>(part, slabs, K, shift, rho);
    return cudaGetLastError();
}

cudaError_t launch_apply(const uint16_t* X, int M, int K, const int8_t* shift, const float* rho, uint16_t* Xt,
                         cudaStream_t st) {
    const long long vecs = (long long)M * K / 8;
    long long blocks = (vecs + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (blocks < 1) blocks = 1;
    preshift_apply_kernel<<<(int)blocks, 256, 0, st>>>(reinterpret_cast<const uint4*>(X), vecs, K, shift, rho,
                                                       reinterpret_cast<uint4*>(Xt));
    return cudaGetLastError();
}

}  // namespace fp4

// ------------------------------------------------- allocation-free variant
// fp4_preshift_calibrate_noalloc: the same two kernels, with the per-slab
// column maxima kept in a buffer that is part of the library image instead
// of a caller-provided workspace.  Some callers have no way to obtain device
// memory at the point where they calibrate: an inference runtime that plans
// all of its device memory at start-up and forbids allocation afterwards, or
// a plug-in that is handed tensors but no allocator.  They use this entry.
//
// The buffer holds kNoAllocFloats fp32 values (256 KB), which bounds K at
// kNoAllocFloats (one slab of column maxima per column at least).  Every
// GPU that loads the library holds this buffer until the process exits.
// Calls share it: two calls whose kernels overlap on a GPU (different
// streams without ordering between them) race on it.  Nothing in it needs
// to start at zero: the column-maximum kernel writes every entry the
// finalize kernel reads, and each call overwrites what the previous left.
namespace fp4 {

constexpr int kNoAllocFloats = 65536;
static __device__ __align__(256) float g_calib_scratch[kNoAllocFloats];

// Host code must not use g_calib_scratch as a device address (on the host
// the name stands for a host-side shadow); the device address is fetched
// once per device, with that device current, and cached.  The cache is
// atomic so that host threads calling on different streams may race on the
// first lookup (both store the same address).  A cached address belongs to
// the context that was current at the lookup, like the library's other
// per-device state: a process that resets a device must not call the
// library on it again.
static std::atomic<float*> g_scratch_ptrs[64];

static float* noalloc_scratch_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    float* ptr = g_scratch_ptrs[dev].load(std::memory_order_acquire);
    if (!ptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_calib_scratch) != cudaSuccess) return nullptr;
        ptr = reinterpret_cast<float*>(p);
        g_scratch_ptrs[dev].store(ptr, std::memory_order_release);
    }
    return ptr;
}


int noalloc_max_k() { return kNoAllocFloats; }

cudaError_t launch_calibrate_noalloc(const uint16_t* X, int M, int K, int8_t* shift, float* rho, int* status,
                                     cudaStream_t st) {
    float* part = noalloc_scratch_ptr();
    if (!part) return cudaErrorInvalidDevice;
    // fewer row slabs than the workspace variant when K is large: the
    // column maxima are exact in any grouping, so the results are the same
    int slabs = calib_slabs(M, K);
    if (slabs > kNoAllocFloats / K) slabs = kNoAllocFloats / K;
    const int rows = (M + slabs - 1) / slabs;
    slabs = (M + rows - 1) / rows;
    dim3 grid((K + kColsPerBlock - 1) / kColsPerBlock, slabs);
    colmax_kernel<<<grid, 256, 0, st>>>(X, M, K, rows, part, status);
    calib_finalize_kernel<<<1, 1024, 0, st>>>(part, slabs, K, shift, rho);
    return cudaGetLastError();
}

}  // namespace fp4
