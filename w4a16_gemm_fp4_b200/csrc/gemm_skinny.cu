// Skinny W4A16 GEMM, group 128, M <= 16 tokens:
//   Y[m, n] = bf16( rho * sum_g s[n, g] * sum_{k in g} X[m, k] * v(code[n, k]) )
// (LLM-FP4 summary page, efficient matrix multiplication: the 4-bit products
// are formed on the exact code values and each group scale multiplies a
// partial sum; the pre-shifted bias is already folded into the weights.)
//
// At a few tokens the GEMM is a stream over the packed weights, so the
// kernel is built around keeping HBM busy:
//   * one persistent CTA per SM takes an even share of all (tile, chunk)
//     units -- a chunk is 16 KB of codes: 128 rows x 2 groups, or 256 rows x
//     1 group when a row has an odd number of groups -- so every SM streams
//     the same number of bytes;
//   * a TMA producer keeps a ring of chunks in flight (the codes and the
//     chunk's slice of the activations); the codes of the first ring-full
//     are requested before the dependency wait, so they stream while the
//     previous kernel in the stream is finishing;
//   * a scale warp copies the chunk's group scales into the slot as the
//     slot is refilled (cp.async), so they land with the codes;
//   * converter warps rewrite the chunk's activations into the order the
//     MMA fragments pair the codes (f16 with a per-chunk power-of-two token
//     factor for E2M1, re-paired bf16 otherwise), so that every shared
//     access of the consumers is conflict-free;
//   * sixteen consumer warps each own 16 rows x 1 group of every chunk: one
//     16-byte shared load per row gives a thread 32 codes, which become
//     exact values in registers (hardware e2m1 -> f16 for E2M1, bf16 by bit
//     placement otherwise) straight in the A fragments of m16n8k16 warp
//     MMAs; the group's MMAs accumulate in fresh registers (four independent
//     chains) that are multiplied by the group scale and the token factor in
//     fp32 and added to the running sum;
//   * a tile that ends inside a CTA's share is stored directly; a tile split
//     between CTAs leaves one partial per CTA in the workspace, and the CTA
//     that completes the tile's count adds the partials in CTA order, so the
//     result does not depend on timing.
// The tensor-core work is tiny next to the stream (at most 16 token
// columns), so warp MMAs fed from registers beat staging the dequantized
// weights for tcgen05: nothing is written back to shared or tensor memory.
#include "common.cuh"

namespace fp4 {

struct SkParams {
    const void* scales;
    int sdt;
    int M, N, K;
    const float* x_scale;    // rho or null
    uint16_t* Y;
    float* part;             // two partial tiles per CTA: [2 * P][M][TR]
    int* cnt;                // per-tile count of published partials (zero between calls)
    int C, P;                // code chunks, CTAs
    int* status;
    unsigned long long timeout_ns;
    int act;                 // output activation (apply_act)
};

template <int NT, int CG>
struct SkCfg {
    static constexpr int NTOK = 8 * NT;                  // token columns of the MMAs
    static constexpr int TR = 256 / CG;                  // rows of a tile
    static constexpr int RB = 64 * CG;                   // bytes of a chunk row
    static constexpr int CBYTES = TR * RB;               // codes of a chunk (16 KB)
    static constexpr int XBYTES = CG * 4 * NTOK * 64;    // activations of a chunk (raw or fragment order)
    static constexpr int SBYTES = CG * TR * 4;           // scales of a chunk as stored (f32 at most)
    static constexpr int FBYTES = NTOK * 4;              // f32 token factors of a chunk
    static constexpr int SLOT = CBYTES + 2 * XBYTES + SBYTES + FBYTES;
    static constexpr int NS = (208 * 1024) / SLOT > 16 ? 16 : (208 * 1024) / SLOT;  // ring slots
    static constexpr int NCW = 16;                       // consumer warps: 16 rows x 1 group each
    static constexpr int RBLK = TR / 16;                 // row blocks of a chunk
    static constexpr int CW = NT == 1 ? 2 : 4;           // activation converter warps
    static constexpr int W0 = 2 + CW;                    // first consumer warp
    static constexpr int THREADS = (W0 + NCW) * 32;
    static constexpr int RPL = TR / 32;                  // rows per scale-warp lane
    static constexpr int SD = 4;                         // chunks of scales in flight per scale-warp lane
    static constexpr int CMB = CG == 2 ? RBLK * 32 * 4 * NT * 4 : 16;  // group-1 sums handed to group 0
    static constexpr int SMEM = 1024 + NS * SLOT + CMB + 3 * NS * 8 + 16;
    static_assert(RBLK * CG == NCW, "one row block and group per consumer warp");
    static_assert(CBYTES == 16384 && XBYTES % 1024 == 0, "slot alignment");
    static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

enum { kSkF16 = 0, kSkBf16 = 1 };

template <int XM>
__device__ __forceinline__ void mma_16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    if constexpr (XM == kSkBf16)
        asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    else
        asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 32 codes (16 bytes of one weight row) -> 16 A-operand words of exact code
// values.  E2M1: the hardware e2m1 -> f16 convert, word R = the natural pair
// (2R, 2R+1) of the 32 (two codes per instruction, the cheapest path).  The
// other formats: bf16 by bit placement, word R = 4q + j holds the pair
// (8q + j, 8q + j + 4).  The activations are paired the same way.
template <int XM, int MANT>
__device__ __forceinline__ void codes_to_frag(const uint4 v, uint32_t o[16]) {
    if constexpr (XM == kSkF16) {
        e2m1_to_f16x8(v.x, o[0], o[1], o[2], o[3]);
        e2m1_to_f16x8(v.y, o[4], o[5], o[6], o[7]);
        e2m1_to_f16x8(v.z, o[8], o[9], o[10], o[11]);
        e2m1_to_f16x8(v.w, o[12], o[13], o[14], o[15]);
    } else {
        dequant8_exact<MANT>(v.x, o);
        dequant8_exact<MANT>(v.y, o + 4);
        dequant8_exact<MANT>(v.z, o + 8);
        dequant8_exact<MANT>(v.w, o + 12);
    }
}

// Atomic add with acquire-release semantics at GPU scope: publishes the
// writes this thread has observed (its CTA's, after a barrier) and sees
// those published by the earlier adders.
__device__ __forceinline__ int atomic_add_acq_rel(int* p, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ int sk_owner(int j, int C, int P) {  // CTA whose share holds chunk j
    return (int)(((long long)(j + 1) * P - 1) / C);
}

template <int NT, int CG, int XM, int MANT>
__global__ void __launch_bounds__(SkCfg<NT, CG>::THREADS, 1)
    gemm_skinny_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       SkParams p) {
    using C = SkCfg<NT, CG>;
    constexpr int TR = C::TR;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base (offset arithmetic keeps the shared address space)
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* codes = smem;                                       // [NS][CBYTES], swizzled rows
    uint8_t* xraw = codes + C::NS * C::CBYTES;                   // [NS][NTOK][128 CG] bf16 as loaded
    uint8_t* xfrag = xraw + C::NS * C::XBYTES;                   // [NS][XBYTES] fragment order
    float* scs = reinterpret_cast<float*>(xfrag + C::NS * C::XBYTES);  // [NS] x ([TR][CG] scales as stored)
    float* xfs = scs + C::NS * CG * TR;                          // [NS][NTOK] token factors
    float* cmb = xfs + C::NS * C::NTOK;                          // [RBLK][32][4 NT]
    uint64_t* ready = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(cmb) + C::CMB);
    uint64_t* xland = ready + C::NS;
    uint64_t* empty = xland + C::NS;
    volatile int* reduce_flag = reinterpret_cast<volatile int*>(empty + C::NS);
    const uint32_t codes_a = smem_u32(codes), xraw_a = smem_u32(xraw), xfrag_a = smem_u32(xfrag),
                   scs_a = smem_u32(scs), xfs_a = smem_u32(xfs);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    const int G = p.K >> 7, cpt = G / CG;
    const int j0 = (int)((long long)c * p.C / p.P), j1 = (int)((long long)(c + 1) * p.C / p.P);
    const int nch = j1 - j0;
    const uint64_t to = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(&ready[s], 1 + 32 + 1);  // codes (with the byte count), 32 scale lanes, a converter
            mbar_init(&xland[s], 1);
            mbar_init(&empty[s], C::NCW);
        }
        fence_mbar_init();
        prefetch_tmap(&tmW);
        prefetch_tmap(&tmX);
    }
    __syncthreads();
    pdl_launch_dependents();

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (elect_one()) {
            const int pre = nch < C::NS ? nch : C::NS;
            // Weights are inputs that no kernel still running may write (the
            // previous kernel in the stream triggers this launch early only
            // when it is one of these GEMMs), so the first ring-full of codes
            // is requested before the dependency wait.
            for (int j = 0; j < pre; ++j) {
                const int jj = j0 + j;
                mbar_arrive_expect_tx(&ready[j], C::CBYTES);
                tma_load_2d(codes + j * C::CBYTES, &tmW, (jj % cpt) * C::RB, (jj / cpt) * TR, &ready[j]);
            }
            pdl_wait();  // the activations may come from the previous kernel
            for (int j = 0; j < pre; ++j) {
                const int jj = j0 + j;
                mbar_arrive_expect_tx(&xland[j], C::XBYTES);
                tma_load_3d(xraw + j * C::XBYTES, &tmX, 0, (jj % cpt) * 2 * CG, 0, &xland[j]);
            }
            int j = pre;
            for (; j < nch; ++j) {
                const int s = j % C::NS, jj = j0 + j;
                if (!mbar_wait_sleep(&empty[s], ((uint32_t)(j / C::NS) & 1u) ^ 1u, to)) {
                    raise_status(p.status, kStatusTimeout);
                    break;
                }
                mbar_arrive_expect_tx(&ready[s], C::CBYTES);
                tma_load_2d(codes + s * C::CBYTES, &tmW, (jj % cpt) * C::RB, (jj / cpt) * TR, &ready[s]);
                mbar_arrive_expect_tx(&xland[s], C::XBYTES);
                tma_load_3d(xraw + s * C::XBYTES, &tmX, 0, (jj % cpt) * 2 * CG, 0, &xland[s]);
            }
            // every copy issued must land before the CTA leaves
            for (int i = j - C::NS < 0 ? 0 : j - C::NS; i < j; ++i)
                if (!mbar_wait_sleep(&xland[i % C::NS], (uint32_t)(i / C::NS) & 1u, to) ||
                    !mbar_wait_sleep(&ready[i % C::NS], (uint32_t)(i / C::NS) & 1u, to)) {
                    raise_status(p.status, kStatusTimeout);
                    break;
                }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------ group scales
        // The chunk's scales s[n, g0 .. g0+CG-1] of its TR rows, as stored
        // ([TR][CG] elements of the scale type), land in the slot together
        // with its codes.  lane: rows RPL*lane .. RPL*lane+RPL-1.  Each row's
        // CG scales are 4-byte aligned words (f32, or f16 pairs: g0 and G are
        // even when CG = 2) copied by cp.async, whose completion is one of
        // the slot's arrivals; f16 scales of single-group chunks (2 bytes)
        // go through registers instead, SD chunks ahead.
        constexpr int RPL = C::RPL;
        const int esz = p.sdt == FP4_SCALE_F16 ? 2 : 4;
        const uint8_t* sbase = static_cast<const uint8_t*>(p.scales);
        if (CG * esz >= 4) {
            bool ok = true;
            for (int j = 0; j < nch && ok; ++j) {
                const int s = j % C::NS, jj = j0 + j;
                if (j >= C::NS && !mbar_wait_sleep(&empty[s], ((uint32_t)(j / C::NS) & 1u) ^ 1u, to)) {
                    raise_status(p.status, kStatusTimeout);
                    ok = false;
                    break;
                }
                const int n0 = (jj / cpt) * TR + RPL * lane, g0 = (jj % cpt) * CG;
                const uint32_t dst = smem_u32(reinterpret_cast<uint8_t*>(scs) + s * C::SBYTES +
                                              RPL * lane * CG * esz);
                const int words = CG * esz / 4;  // 4-byte copies per row (scale arrays are 4-byte aligned)
#pragma unroll
                for (int r = 0; r < RPL; ++r) {
                    const bool in = n0 + r < p.N;
                    // rows past N: nothing is read, the piece is zero-filled
                    const uint8_t* src = sbase + (in ? ((size_t)(n0 + r) * G + g0) * esz : 0);
                    for (int w = 0; w < words; ++w)
                        cp_async4_zfill(dst + r * CG * esz + 4 * w, src + (in ? 4 * w : 0), in ? 4 : 0);
                }
                cp_async_arrive_noinc(&ready[s]);
            }
        } else {
            // f16, one group per chunk
            float sv[C::SD][RPL];
            auto fetch = [&](int j, float* v) {
                const int jj = j0 + j, n0 = (jj / cpt) * TR + RPL * lane, g0 = jj % cpt;
#pragma unroll
                for (int r = 0; r < RPL; ++r)
                    v[r] = (j < nch && n0 + r < p.N) ? load_scale(p.scales, p.sdt, (size_t)(n0 + r) * G + g0) : 0.f;
            };
#pragma unroll
            for (int d = 0; d < C::SD; ++d) fetch(d, sv[d]);
            bool ok = true;
            for (int jb = 0; jb < nch && ok; jb += C::SD) {
#pragma unroll
                for (int d = 0; d < C::SD; ++d) {
                    const int j = jb + d;
                    if (j < nch && ok) {
                        const int s = j % C::NS;
                        if (!mbar_wait_sleep(&empty[s], ((uint32_t)(j / C::NS) & 1u) ^ 1u, to)) {
                            raise_status(p.status, kStatusTimeout);
                            ok = false;
                        } else {
                            __half* dst = reinterpret_cast<__half*>(reinterpret_cast<uint8_t*>(scs) + s * C::SBYTES) +
                                          RPL * lane;
#pragma unroll
                            for (int r = 0; r < RPL; ++r) dst[r] = __float2half_rn(sv[d][r]);  // exact: f16 values
                            mbar_arrive(&ready[s]);
                            fetch(j + C::SD, sv[d]);
                        }
                    }
                }
            }
        }
    } else if (warp < C::W0) {
        // ------------------------------------------------ activation converter
        // The chunk's activations ([NTOK][128*CG] bf16 as loaded) go to the
        // order the MMA fragments take them: 16-byte vector vv of token m
        // (group gg = vv / 16, quarter t = (vv / 4) % 4, piece i = vv % 4) is
        // stored at unit ((gg * 4 + i) * NTOK + m) * 4 + t, so that a
        // consumer lane (token q, quarter t) reads its group's 32 values as
        // four 16-byte pieces, eight lanes of a load phase reading 128
        // contiguous bytes.  E2M1: f16 scaled by the power of two that brings
        // the token's largest magnitude in this chunk into [2^14, 2^15)
        // (exact for every element within 2^31 of it; the consumers undo the
        // factor in fp32; a non-finite activation makes its rows non-finite
        // either way).  Other formats: bf16 re-paired from (k0..k7) to
        // (k0,k4) (k1,k5) (k2,k6) (k3,k7).  Padding tokens (M .. NTOK-1) stay
        // zero.
        constexpr int VPT = CG * 16;  // vectors per token and chunk
        constexpr int TPW = 32 / VPT;  // tokens per warp pass: 1 (CG = 2) or 2 (CG = 1)
        const int cv = warp - 2;
        auto unit_of = [&](int m, int vv) {
            return (((vv >> 4) * 4 + (vv & 3)) * C::NTOK + m) * 64 + ((vv >> 2) & 3) * 16;
        };
        for (int s = cv; s < C::NS; s += C::CW) {
            for (int v = p.M * VPT + lane; v < C::NTOK * VPT; v += 32)
                *reinterpret_cast<uint4*>(xfrag + s * C::XBYTES + unit_of(v / VPT, v % VPT)) =
                    make_uint4(0u, 0u, 0u, 0u);
            for (int m = p.M + lane; m < C::NTOK; m += 32) xfs[s * C::NTOK + m] = 0.f;
        }
        const int mm = p.M < C::NTOK ? p.M : C::NTOK;
        const int vv = lane % VPT;  // this lane's vector of each token
        // converter warp cv takes chunks cv, cv + CW, ...: all tokens of a
        // chunk, one vector per lane and token
        for (int j = cv; j < nch; j += C::CW) {
            const int s = j % C::NS;
            // the slot's activations landed, so its previous round was consumed
            if (!__all_sync(0xffffffffu, mbar_wait_sleep(&xland[s], (uint32_t)(j / C::NS) & 1u, to))) {
                if (lane == 0) raise_status(p.status, kStatusTimeout);
                break;
            }
            const uint32_t src = xraw_a + s * C::XBYTES;
            const uint32_t dst = xfrag_a + s * C::XBYTES;
#pragma unroll 4
            for (int m0 = 0; m0 < mm; m0 += TPW) {
                const int m = m0 + lane / VPT;
                const bool has = m < mm;
                const uint4 x = has ? lds128(src + (m * VPT + vv) * 16) : make_uint4(0u, 0u, 0u, 0u);
                uint4 o;
                float f = 1.f;
                if constexpr (XM == kSkF16) {
                    // largest magnitude of the token's slice (bf16 bits order like magnitudes)
                    const uint32_t a0 = x.x & 0x7fff7fffu, a1 = x.y & 0x7fff7fffu, a2 = x.z & 0x7fff7fffu,
                                   a3 = x.w & 0x7fff7fffu;
                    uint32_t mx = max(max(max(a0 & 0xffffu, a0 >> 16), max(a1 & 0xffffu, a1 >> 16)),
                                      max(max(a2 & 0xffffu, a2 >> 16), max(a3 & 0xffffu, a3 >> 16)));
                    if constexpr (VPT == 32) {
                        mx = __reduce_max_sync(0xffffffffu, mx);
                    } else {
#pragma unroll
                        for (int o2 = 1; o2 < VPT; o2 <<= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
                    }
                    const int E = (int)(mx >> 7);  // biased exponent of the maximum
                    int sh = mx == 0 ? 0 : 141 - (E < 1 ? 1 : E);
                    if (sh > 126) sh = 126;
                    o = bf16x8_to_f16x8(x, __int_as_float((127 + sh) << 23));
                    f = __int_as_float((127 - sh) << 23);
                } else {
                    o = make_uint4(prmt(x.x, x.z, 0x5410u), prmt(x.x, x.z, 0x7632u), prmt(x.y, x.w, 0x5410u),
                                   prmt(x.y, x.w, 0x7632u));
                }
                if (has) {
                    sts128(dst + unit_of(m, vv), o);
                    if (vv == 0) sts_f32(xfs_a + (s * C::NTOK + m) * 4, f);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ready[s]);
        }
    } else {
        // --------------------------------------------------------- consumers
        // Warp (rb, gg): rows rb*16 .. rb*16+15 of the chunk, group gg.
        // Lane (q, t) = (lane / 4, lane % 4): MMA row q <-> weight row rA,
        // row q + 8 <-> rB = rA + 8; 16-byte unit t of the group's 64-byte
        // row segment.  With the 128-byte swizzle rows q and q ^ 1 (one
        // shared-load phase) are 4 rows apart, so their units land in
        // different bank halves; with the 64-byte swizzle adjacent rows do.
        const int cw = warp - C::W0, rb = cw % C::RBLK, gg = cw / C::RBLK;
        const int q = lane >> 2, t = lane & 3;
        const int rq = CG == 2 ? (((q & 1) << 2) | (q >> 1)) : q;
        const int rA = rb * 16 + rq, rB = rA + 8;
        const int swz = CG == 2 ? (rA & 7) : ((rA >> 1) & 3);
        const int unit = ((4 * gg + t) ^ swz) << 4;
        const int ctid = threadIdx.x - C::W0 * 32;
        const bool sdt16 = p.sdt == FP4_SCALE_F16;
        pdl_wait();  // rho, the counters and the partials belong to the stream order
        const float rho = p.x_scale ? *p.x_scale : 1.f;
        float tot[NT][4];
#pragma unroll
        for (int jn = 0; jn < NT; ++jn)
#pragma unroll
            for (int k = 0; k < 4; ++k) tot[jn][k] = 0.f;
        const int ft = j0 / cpt;           // first tile of this share
        bool seg_from_start = (j0 % cpt) == 0;
        bool ok = true;
        for (int j = 0; j < nch; ++j) {
            const int s = j % C::NS, jj = j0 + j;
            // after a timeout the loop still walks the pieces (without
            // waiting or computing) so that every consumer warp meets the
            // same named barriers
            if (ok && !__all_sync(0xffffffffu, mbar_wait_sleep(&ready[s], (uint32_t)(j / C::NS) & 1u, to))) {
                if (lane == 0) raise_status(p.status, kStatusTimeout);
                ok = false;
            }
            if (ok) {
                const uint32_t cb = codes_a + s * C::CBYTES;
                const uint32_t xb = xfrag_a + s * C::XBYTES + gg * 4 * C::NTOK * 64;
                const uint4 wa = lds128(cb + rA * C::RB + unit);
                const uint4 wb = lds128(cb + rB * C::RB + unit);
                const uint32_t sp = scs_a + s * C::SBYTES;
                const float sA = sdt16 ? lds_f16_as_f32(sp + (rA * CG + gg) * 2) : lds_f32(sp + (rA * CG + gg) * 4);
                const float sB = sdt16 ? lds_f16_as_f32(sp + (rB * CG + gg) * 2) : lds_f32(sp + (rB * CG + gg) * 4);
                uint32_t A0[16], A1[16];
                codes_to_frag<XM, MANT>(wa, A0);
                codes_to_frag<XM, MANT>(wb, A1);
#pragma unroll
                for (int jn = 0; jn < NT; ++jn) {
                    uint32_t xw[16];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint4 v = lds128(xb + (i * C::NTOK + 8 * jn + q) * 64 + t * 16);
                        xw[4 * i] = v.x;
                        xw[4 * i + 1] = v.y;
                        xw[4 * i + 2] = v.z;
                        xw[4 * i + 3] = v.w;
                    }
                    // four independent accumulator chains (k-step mod 4)
                    float acc[4][4];
#pragma unroll
                    for (int h = 0; h < 4; ++h)
#pragma unroll
                        for (int k = 0; k < 4; ++k) acc[h][k] = 0.f;
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_16816<XM>(acc[k & 3], A0[2 * k], A1[2 * k], A0[2 * k + 1], A1[2 * k + 1], xw[2 * k],
                                      xw[2 * k + 1]);
                    // group scale x the chunk's token factor, in fp32
                    const float f0 = lds_f32(xfs_a + (s * C::NTOK + 8 * jn + 2 * t) * 4),
                                f1 = lds_f32(xfs_a + (s * C::NTOK + 8 * jn + 2 * t + 1) * 4);
                    const float w[4] = {sA * f0, sA * f1, sB * f0, sB * f1};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float a = (acc[0][k] + acc[1][k]) + (acc[2][k] + acc[3][k]);
                        tot[jn][k] = fmaf(w[k], a, tot[jn][k]);
                    }
                }
                __syncwarp();  // every lane's reads of the slot are consumed
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            const int tile = jj / cpt, cc = jj % cpt;
            if (cc != cpt - 1 && j != nch - 1) continue;
            // ----------------------------------------------- end of a tile piece
            // CG = 2: the group-1 warps hand their sums to the group-0 warps
            // of the same rows, which finish the piece
            if constexpr (CG == 2) {
                float* cm = cmb + (rb * 32 + lane) * 4 * NT;
                if (gg == 1) {
#pragma unroll
                    for (int jn = 0; jn < NT; ++jn)
                        *reinterpret_cast<float4*>(cm + 4 * jn) =
                            make_float4(tot[jn][0], tot[jn][1], tot[jn][2], tot[jn][3]);
                }
                named_barrier_sync(1, C::NCW * 32);
                if (gg == 0) {
#pragma unroll
                    for (int jn = 0; jn < NT; ++jn) {
                        const float4 o = *reinterpret_cast<const float4*>(cm + 4 * jn);
                        tot[jn][0] += o.x;
                        tot[jn][1] += o.y;
                        tot[jn][2] += o.z;
                        tot[jn][3] += o.w;
                    }
                }
            }
            const bool owner = gg == 0;  // this warp finishes its rows' piece
            const int n0 = tile * TR;
            if (seg_from_start && cc == cpt - 1) {
                if (owner) {
#pragma unroll
                    for (int jn = 0; jn < NT; ++jn)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int m = 8 * jn + 2 * t + e;
                            const float va = rho * tot[jn][e], vb = rho * tot[jn][2 + e];
                            if (p.act == kActSiluGate) {
                                // rows rA ^ 1 and rB ^ 1 are held by lane ^ 8 (128-byte
                                // swizzle row order) or lane ^ 4 (64-byte)
                                const int o = CG == 2 ? 8 : 4;
                                const float wa = __shfl_xor_sync(0xffffffffu, va, o);
                                const float wb = __shfl_xor_sync(0xffffffffu, vb, o);
                                if (m < p.M && (rA & 1) == 0) {
                                    const int NH = p.N >> 1;
                                    if (n0 + rA + 1 < p.N)
                                        p.Y[(size_t)m * NH + ((n0 + rA) >> 1)] = bf16_bits(silu_gate(va, wa));
                                    if (n0 + rB + 1 < p.N)
                                        p.Y[(size_t)m * NH + ((n0 + rB) >> 1)] = bf16_bits(silu_gate(vb, wb));
                                }
                            } else if (m < p.M) {
                                if (n0 + rA < p.N) p.Y[(size_t)m * p.N + n0 + rA] = bf16_bits(apply_act(va, p.act));
                                if (n0 + rB < p.N) p.Y[(size_t)m * p.N + n0 + rB] = bf16_bits(apply_act(vb, p.act));
                            }
                        }
                }
            } else {
                // A tile split between CTAs: publish this share's partial, count
                // it, and the CTA that completes the count adds all partials in
                // CTA order (the count is left at zero for the next call).
                const int slot = tile == ft ? 0 : 1;
                if (owner) {
                    float* pp = p.part + (size_t)(2 * c + slot) * p.M * TR;
#pragma unroll
                    for (int jn = 0; jn < NT; ++jn)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int m = 8 * jn + 2 * t + e;
                            if (m < p.M) {
                                pp[m * TR + rA] = tot[jn][e];
                                pp[m * TR + rB] = tot[jn][2 + e];
                            }
                        }
                }
                // the barrier makes every consumer's partial visible to thread
                // 0, whose release-acquire add publishes them at GPU scope and
                // (for the last adder) acquires everyone else's
                named_barrier_sync(1, C::NCW * 32);
                const int c0 = sk_owner(tile * cpt, p.C, p.P), c1 = sk_owner((tile + 1) * cpt - 1, p.C, p.P);
                if (ctid == 0) *reduce_flag = ok && atomic_add_acq_rel(p.cnt + tile, 1) == c1 - c0;
                named_barrier_sync(1, C::NCW * 32);
                if (*reduce_flag) {
                    const int quads = p.M * (TR / 4);  // 4 outputs (one token, 4 rows) each
                    for (int qd = ctid; qd < quads; qd += C::NCW * 32) {
                        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
                        for (int z0 = c0; z0 <= c1; z0 += 8) {
                            float4 v[8];
#pragma unroll
                            for (int z = 0; z < 8; ++z) {
                                const int cz = z0 + z;
                                v[z] = make_float4(0.f, 0.f, 0.f, 0.f);
                                if (cz <= c1) {
                                    const int ftz = (int)((long long)cz * p.C / p.P) / cpt;
                                    // L2 loads: the partials were written by other SMs
                                    v[z] = __ldcg(reinterpret_cast<const float4*>(
                                               p.part + (size_t)(2 * cz + (tile == ftz ? 0 : 1)) * p.M * TR) +
                                           qd);
                                }
                            }
#pragma unroll
                            for (int z = 0; z < 8; ++z) {
                                sum.x += v[z].x;
                                sum.y += v[z].y;
                                sum.z += v[z].z;
                                sum.w += v[z].w;
                            }
                        }
                        const int m = qd / (TR / 4), n = n0 + (qd % (TR / 4)) * 4;
                        if (p.act == kActSiluGate) {
                            // the quad is two gate/up pairs
                            uint16_t* dst = p.Y + (size_t)m * (p.N >> 1) + (n >> 1);
                            if (n + 1 < p.N) dst[0] = bf16_bits(silu_gate(rho * sum.x, rho * sum.y));
                            if (n + 3 < p.N) dst[1] = bf16_bits(silu_gate(rho * sum.z, rho * sum.w));
                            continue;
                        }
                        uint16_t* dst = p.Y + (size_t)m * p.N + n;
                        const uint32_t y01 = pack_bf16x2(apply_act(rho * sum.x, p.act), apply_act(rho * sum.y, p.act)),
                                       y23 = pack_bf16x2(apply_act(rho * sum.z, p.act), apply_act(rho * sum.w, p.act));
                        if ((p.N & 3) == 0 && n + 3 < p.N) {
                            *reinterpret_cast<uint2*>(dst) = make_uint2(y01, y23);
                        } else {
                            const uint16_t y[4] = {(uint16_t)(y01 & 0xffffu), (uint16_t)(y01 >> 16),
                                                   (uint16_t)(y23 & 0xffffu), (uint16_t)(y23 >> 16)};
                            for (int e = 0; e < 4; ++e)
                                if (n + e < p.N) dst[e] = y[e];
                        }
                    }
                    if (ctid == 0) p.cnt[tile] = 0;
                }
            }
            // reduce_flag and the hand-off buffer are reused by the next piece
            named_barrier_sync(1, C::NCW * 32);
#pragma unroll
            for (int jn = 0; jn < NT; ++jn)
#pragma unroll
                for (int k = 0; k < 4; ++k) tot[jn][k] = 0.f;
            seg_from_start = true;
        }
    }
}

// ----------------------------------------------------------- host launch

bool encode_2d(CUtensorMap* map, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t inner,
               uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw);
bool encode_3d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t mid,
               uint64_t outer, uint64_t mid_stride, uint64_t outer_stride, uint32_t box_inner, uint32_t box_mid,
               uint32_t box_outer);
int device_sm_count();
constexpr int kSkinnyCounters = 16384;  // tiles a counter block serves

int skinny_max_m() { return 16; }

// Tiles of the skinny GEMM for this shape (128 rows, or 256 when a row has
// an odd number of groups).
int skinny_tiles(int N, int K) {
    const int G = K / 128, TR = G % 2 == 0 ? 128 : 256;
    return (N + TR - 1) / TR;
}

int skinny_max_tiles() { return kSkinnyCounters; }

static int sk_ctas(int N, int K, int ctas, int* chunks_out) {
    const int G = K / 128, CG = G % 2 == 0 ? 2 : 1;
    const int C = skinny_tiles(N, K) * (G / CG);
    int P = ctas > 0 ? ctas : device_sm_count();
    if (P > C) P = C;
    if (P < 1) P = 1;
    if (chunks_out) *chunks_out = C;
    return P;
}

// Workspace of the skinny GEMM: the partial tiles, two per CTA of M x TR
// floats.  The tile counters live in a separate block that is zero between
// calls.
size_t skinny_ws_bytes(int M, int N, int K) {
    if (M <= 0 || M > 16 || N <= 0 || K <= 0 || K % 128) return 0;
    const int P = sk_ctas(N, K, 0, nullptr), TR = (K / 128) % 2 == 0 ? 128 : 256;
    return ((size_t)2 * P * M * TR * 4 + 255) & ~(size_t)255;
}

static cudaLaunchAttribute pdl_attr() {
    cudaLaunchAttribute a;
    a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a.val.programmaticStreamSerializationAllowed = 1;
    return a;
}

template <int NT, int CG, int XM, int MANT>
static cudaError_t launch_sk_t(const CUtensorMap& mw, const CUtensorMap& mx, const SkParams& p, cudaStream_t st) {
    using C = SkCfg<NT, CG>;
    auto kern = gemm_skinny_kernel<NT, CG, XM, MANT>;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_set[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.P, 1, 1);
    cfg.blockDim = dim3(C::THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1] = {pdl_attr()};
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, mw, mx, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int NT, int CG>
static cudaError_t launch_sk_fmt(int fmt, const CUtensorMap& mw, const CUtensorMap& mx, const SkParams& p,
                                 cudaStream_t st) {
    if (fmt == FP4_E2M1) return launch_sk_t<NT, CG, kSkF16, 1>(mw, mx, p, st);
    if (fmt == FP4_E1M2) return launch_sk_t<NT, CG, kSkBf16, 2>(mw, mx, p, st);
    return launch_sk_t<NT, CG, kSkBf16, 0>(mw, mx, p, st);
}

// Skinny GEMM (M <= 16, group 128).  cnt: kSkinnyCounters ints, zero on
// entry and left zero; ws: skinny_ws_bytes(M, N, K) bytes; ctas = 0 takes
// one CTA per SM (at most one per code chunk).
cudaError_t launch_gemm_skinny(const uint16_t* X, int* cnt, void* ws, size_t ws_bytes, const uint8_t* packed,
                               const void* scales, int sdt, int fmt, int M, int N, int K, const float* x_scale,
                               uint16_t* Y, int act, int ctas, int* status, unsigned long long timeout_ns,
                               cudaStream_t st) {
    if (K % 128 != 0 || M <= 0 || M > 16 || N <= 0 || cnt == nullptr) return cudaErrorInvalidValue;
    if (skinny_tiles(N, K) > kSkinnyCounters) return cudaErrorInvalidValue;
    int chunks = 0;
    const int P = sk_ctas(N, K, ctas, &chunks);
    const int G = K / 128, CG = G % 2 == 0 ? 2 : 1, TR = 256 / CG, NT = M <= 8 ? 1 : 2;
    if (ws == nullptr || ws_bytes < (size_t)2 * P * M * TR * 4) return cudaErrorInvalidValue;
    CUtensorMap mw, mx;
    // code chunks: TR rows x CG*64 bytes, 128- or 64-byte swizzle
    if (!encode_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, packed, (uint64_t)K / 2, (uint64_t)N, (uint32_t)(64 * CG),
                   (uint32_t)TR, CG == 2 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    // activation slices: X viewed as [M][K/64][64]; one box = 2*CG runs of 64
    // k for 8*NT token rows (rows past M read as zero)
    if (!encode_3d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, 64, (uint64_t)K / 64, (uint64_t)M, 128,
                   (uint64_t)K * 2, 64, (uint32_t)(2 * CG), (uint32_t)(8 * NT)))
        return cudaErrorInvalidValue;
    SkParams p;
    p.scales = scales;
    p.sdt = sdt;
    p.M = M;
    p.N = N;
    p.K = K;
    p.x_scale = x_scale;
    p.Y = Y;
    p.part = static_cast<float*>(ws);
    p.cnt = cnt;
    p.C = chunks;
    p.P = P;
    p.status = status;
    p.timeout_ns = timeout_ns;
    p.act = act;
    if (CG == 2) return NT == 1 ? launch_sk_fmt<1, 2>(fmt, mw, mx, p, st) : launch_sk_fmt<2, 2>(fmt, mw, mx, p, st);
    return NT == 1 ? launch_sk_fmt<1, 1>(fmt, mw, mx, p, st) : launch_sk_fmt<2, 1>(fmt, mw, mx, p, st);
}

}  // namespace fp4
