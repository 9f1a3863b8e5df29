// gemm_ts.cu -- the decode engine: group-128 W4A16 GEMM for M <= 64 on the
// sm_100a tensor cores with the dequantized weights in TENSOR MEMORY
// (tcgen05.mma, A from TMEM, B from shared memory).
//
// Y[m,n] = bf16( rho * sum_g s[n,g] * sum_{k in g} X[m,k] * v(code[n,k]) )
// (LLM-FP4 summary page "首个支持4-bit浮点量化的LLM来了", efficient matrix
// multiplication: the full-precision group scale stays outside the 4-bit
// product.)  The tensor cores multiply the EXACT code values v by 16-bit
// activations with fp32 accumulation, one TMEM accumulator per 128-k group,
// and each group's sum is scaled by s in fp32 (the fold).  No weight is
// rounded.
//
// Why the weights go to tensor memory.  An MMA that reads its A operand from
// shared memory moves 4 KB (128 rows x 16 k x 2 B) through shared memory per
// K = 16 step on top of the B operand; at small N that read is the floor of
// the instruction (measured: 39 cycles at N = 16, 48 at N = 64).  With A in
// tensor memory an M = 128, K = 16 step takes 10 cycles at N = 16 and runs at
// the full tensor rate from N = 64 (32 cycles) up, and shared memory carries
// only the packed codes (0.5 B per weight) and the activations.
//
// Activations are prepared once per call by a pre-pass into the workspace:
// E2M1 rows scaled by a power of two into the f16 range and rounded to f16
// (x_rows_to_f16_kernel; the codes then dequantize with the hardware
// e2m1x2 -> f16x2 convert), other formats re-paired bf16 rows
// (x_rows_repair_kernel; codes by bit placement to bf16 (k, k+4) pairs).
// Every 128-row tile of the output reads the same activations, so preparing
// them inside the GEMM would repeat that work N/128 times.
//
// Work split (stream-K).  The weights are cut into code chunks of CG groups
// (128 rows x CG*64 bytes) and the chunks, tile by tile, into one contiguous
// range per CTA, one CTA per SM, so every SM streams the same number of
// bytes.  A tile that a CTA covers whole is stored directly; the pieces of a
// tile shared by several CTAs are written as fp32 partial tiles to the
// workspace, and the CTA that finishes a tile's last piece (a per-tile
// counter) adds them in CTA order -- deterministic -- and stores the tile.
// Measured on one B200: with 128-row tiles split over a cluster along K,
// SMs that hosted two CTAs finished ~45% later than the rest and set the
// kernel time; a CTA alone on an SM with 64 KB of codes in flight was bound
// by memory latency, so each CTA here keeps 128 KB in flight.
//
// Roles (one CTA per SM):
//   warp 0        code producer: one thread copies code chunks by TMA;
//   warp 1        TMEM allocator and MMA issuer (one thread): 8 MMAs per
//                 group, then commits that free the A stage and the
//                 activation stage and hand the accumulator to the fold;
//   warp 2        activation producer: one 128-k stage (two 64-k boxes,
//                 128-byte swizzle) per TMA pair;
//   warps 3-10    dequantize: two per TMEM lane quadrant, a thread owns half
//                 of one weight row of a group (64 codes); it reads both
//                 groups of a chunk and releases the chunk at once, converts
//                 the codes into exact 16-bit values in registers and stores
//                 them into its lane of the A stage with tcgen05.st;
//   fold warps    tcgen05.ld the group accumulator and add s * acc to fp32
//                 totals in registers; at the end of each tile piece the
//                 epilogue above.
// A TMA copy costs its issuing thread on the order of a hundred cycles, so
// codes and activations have a producer thread each and the codes travel in
// chunks of two groups (one full 128-byte line per weight row).
// Every mbarrier wait is bounded; a warp decides together (a vote) before
// any warp-collective tcgen05 instruction.  No multicast is used.
#include "common.cuh"

namespace fp4 {

enum { kXF16 = 0, kXBf16 = 1 };  // prepared activations: scaled f16 / re-paired bf16

struct TsParams {
    const uint16_t* xp;    // prepared activations [M][K] (f16 or re-paired bf16)
    const void* scales;
    int sdt;
    int M, N, K;
    const float* x_scale;  // rho (device) or nullptr
    const float* xrow;     // kXF16: per-row factor undoing the f16 scaling
    uint16_t* Y;
    float* part;           // [2 * P][BT][128] fp32 partial tiles
    int* cnt;              // [tiles] pieces finished (zero at entry, left zero)
    int C;                 // code chunks in total (tiles * chunks per tile)
    int P;                 // CTAs
    int* status;
    unsigned long long timeout_ns;
    int act;               // output activation (apply_act)
};

template <int BT, int CG>
struct TsCfg {
    static constexpr int BW = 128;                       // weight rows per tile (MMA M, TMEM lanes)
    static constexpr int XBOX = BT * 128;                // 64 k x BT rows of 16-bit activations
    static constexpr int XBYTES = 2 * XBOX;              // one 128-k activation stage
    static constexpr int RB = 64 * CG;                   // bytes of one weight row in a code chunk
    static constexpr int CBYTES = BW * RB;               // one code chunk
    static constexpr int WCH = 8 * 2 / CG;               // code chunks in flight: 128 KB
    static constexpr int NA = 4;                         // A stages in TMEM, 64 columns each
    static constexpr int NACC = BT <= 32 ? 4 : 2;        // accumulators in TMEM, BT columns each
    // activation stages: their copies share the SM's copy engine with the
    // code chunks, so they are issued several groups ahead
    static constexpr int NX = BT <= 16 ? 8 : (BT <= 32 ? 6 : 4);
    static constexpr int DQW = 8;                        // dequant warps: two per lane quadrant
    static constexpr int FCOLS = BT <= 32 ? BT : 32;     // accumulator columns per fold thread
    static constexpr int NF = 4 * (BT / FCOLS);          // fold warps
    static constexpr int DQ0 = 3, FW0 = DQ0 + DQW;       // warps 0-2: codes, MMA, activations
    static constexpr int THREADS = (FW0 + NF) * 32;
    static constexpr int ACC0 = NA * 64;                 // first accumulator column
    static constexpr int TMEM_NEED = ACC0 + NACC * BT;
    static constexpr int TMEM_COLS = TMEM_NEED <= 256 ? 256 : 512;
    static constexpr int NBAR = 2 * WCH + 2 * NX + 2 * NA + 2 * NACC;
    static constexpr int RING = NX * XBYTES + WCH * CBYTES;
    static constexpr int XROW = NF * FCOLS * 4;          // token factors of each fold warp
    static constexpr int DEP = DQW * 32 * 4;             // per-dequant-thread scratch words (chunk release)
    static constexpr int SB = NF * 32 * 8 * 4;           // per-fold-thread group scales of 8 stages
    static constexpr int SMEM = 1024 + RING + XROW + DEP + SB + NBAR * 8 + 32;
    static_assert(BT == 16 || BT == 32 || BT == 64, "token tile");
    static_assert(CG == 1 || CG == 2, "groups per code chunk");
    static_assert(TMEM_NEED <= 512, "tensor memory");
    static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
    static_assert(THREADS <= 1024, "threads per CTA");
};

// The CTA that owns chunk j when C chunks are split into P contiguous
// ranges [c*C/P, (c+1)*C/P).
__device__ __forceinline__ int chunk_owner(int j, int C, int P) {
    return (int)(((long long)(j + 1) * P - 1) / C);
}

// 8 codes (one word) -> four 32-bit columns of the A stage.
template <int XM, int MANT>
__device__ __forceinline__ void codes_to_a(uint32_t w, uint32_t* o) {
    if constexpr (XM == kXBf16) {
        dequant8_exact<MANT>(w, o);  // (k, k+4) pairs, bf16
    } else {
        e2m1_to_f16x8(w, o[0], o[1], o[2], o[3]);  // (k, k+1) pairs, f16
    }
}

template <int BT, int CG, int XM, int MANT>
__global__ void __launch_bounds__(TsCfg<BT, CG>::THREADS, 1)
    gemm_ts_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, TsParams p) {
    using C = TsCfg<BT, CG>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* xs = smem;                                  // NX x XBYTES: activation stages
    uint8_t* wsr = xs + C::NX * C::XBYTES;               // WCH x CBYTES: code chunks
    float* xrow_s = reinterpret_cast<float*>(wsr + C::WCH * C::CBYTES);  // [NF][FCOLS]
    uint32_t* dep_slots = reinterpret_cast<uint32_t*>(xrow_s + C::XROW / 4);
    float* sbuf = reinterpret_cast<float*>(dep_slots + C::DEP / 4);  // [NF * 32][8]
    uint64_t* bars = reinterpret_cast<uint64_t*>(sbuf + C::SB / 4);
    uint64_t* wfull = bars;                  // code chunk landed
    uint64_t* wempty = wfull + C::WCH;       // code chunk read by the dequant threads
    uint64_t* xfull = wempty + C::WCH;       // activations landed
    uint64_t* xempty = xfull + C::NX;        // MMAs done with the activations
    uint64_t* afull = xempty + C::NX;        // A stage written to TMEM
    uint64_t* aempty = afull + C::NA;        // MMAs done with the A stage
    uint64_t* gfull = aempty + C::NA;        // accumulator complete
    uint64_t* gempty = gfull + C::NACC;      // accumulator folded
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gempty + C::NACC);
    volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    const int G = p.K >> 7;                  // groups per row
    const int cpt = G / CG;                  // chunks per tile
    const int j0 = (int)((long long)c * p.C / p.P), j1 = (int)((long long)(c + 1) * p.C / p.P);
    const int nch = j1 - j0;                 // code chunks of this CTA
    const int nst = nch * CG;                // stages (groups) of this CTA
    const int u0 = j0 * CG;                  // first (tile, group) unit: tile = u / G, group = u % G
    const uint64_t to = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::WCH; ++s) {
            mbar_init(&wfull[s], 1);
            mbar_init(&wempty[s], C::DQW * 32);
        }
        for (int s = 0; s < C::NX; ++s) {
            mbar_init(&xfull[s], 1);
            mbar_init(&xempty[s], 1);
        }
        for (int s = 0; s < C::NA; ++s) {
            mbar_init(&afull[s], C::DQW);
            mbar_init(&aempty[s], 1);
        }
        for (int s = 0; s < C::NACC; ++s) {
            mbar_init(&gfull[s], 1);
            mbar_init(&gempty[s], C::NF);
        }
        fence_mbar_init();
        prefetch_tmap(&tmX);
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
    pdl_wait();  // activations, counters (and everything else) may come from the previous kernel
    pdl_launch_dependents();

    if (warp == 0) {
        // --------------------------------------------------- code producer
        if (elect_one()) {
            int j = 0;
            for (; j < nch; ++j) {
                const int s = j % C::WCH, jj = j0 + j;
                if (!mbar_wait(&wempty[s], ((uint32_t)(j / C::WCH) & 1u) ^ 1u, to)) {
                    raise_status(p.status, kStatusTimeout);
                    break;
                }
                mbar_arrive_expect_tx(&wfull[s], C::CBYTES);
                tma_load_2d(wsr + s * C::CBYTES, &tmW, (jj % cpt) * C::RB, (jj / cpt) * C::BW, &wfull[s]);
            }
            // every copy issued must land before the CTA leaves
            for (int i = j - C::WCH < 0 ? 0 : j - C::WCH; i < j; ++i)
                if (!mbar_wait(&wfull[i % C::WCH], (uint32_t)(i / C::WCH) & 1u, to)) {
                    raise_status(p.status, kStatusTimeout);
                    break;
                }
        }
        __syncwarp();
    } else if (warp == 2) {
        // --------------------------------------------- activation producer
        if (elect_one()) {
            int i = 0;
            for (; i < nst; ++i) {
                const int s = i % C::NX, g = (u0 + i) % G;
                if (!mbar_wait(&xempty[s], ((uint32_t)(i / C::NX) & 1u) ^ 1u, to)) {
                    raise_status(p.status, kStatusTimeout);
                    break;
                }
                mbar_arrive_expect_tx(&xfull[s], C::XBYTES);
                tma_load_2d(xs + s * C::XBYTES, &tmX, g * 128, 0, &xfull[s]);
                tma_load_2d(xs + s * C::XBYTES + C::XBOX, &tmX, g * 128 + 64, 0, &xfull[s]);
            }
            for (int j = i - C::NX < 0 ? 0 : i - C::NX; j < i; ++j)
                if (!mbar_wait(&xfull[j % C::NX], (uint32_t)(j / C::NX) & 1u, to)) {
                    raise_status(p.status, kStatusTimeout);
                    break;
                }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ----------------------------------------------------- MMA issuer
        if (elect_one()) {
            const uint32_t idesc = XM == kXBf16 ? idesc_bf16_f32(C::BW, BT) : idesc_f16_f32(C::BW, BT);
            const uint64_t xdesc0 = sw128_desc(smem_u32(xs));
            constexpr uint32_t kXStep = C::XBYTES >> 4, kXAtom = C::XBOX >> 4;
            int issued = 0;
            for (int i = 0; i < nst; ++i) {
                const int a = i % C::NA, x = i % C::NX, b = i % C::NACC;
                if (!mbar_wait(&afull[a], (uint32_t)(i / C::NA) & 1u, to) ||
                    !mbar_wait(&xfull[x], (uint32_t)(i / C::NX) & 1u, to) ||
                    !mbar_wait(&gempty[b], ((uint32_t)(i / C::NACC) & 1u) ^ 1u, to)) {
                    raise_status(p.status, kStatusTimeout);
                    break;
                }
                tc_fence_after();
                const uint64_t xd = xdesc0 + (uint64_t)(x * kXStep);
                const uint32_t ta = tmem + (uint32_t)(a * 64);
                const uint32_t td = tmem + (uint32_t)(C::ACC0 + b * BT);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc_mma_ts(td, ta + (uint32_t)(8 * kk), xd + (uint64_t)((kk >> 2) * kXAtom + 2 * (kk & 3)), idesc,
                              kk ? 1u : 0u);
                tc_commit(&aempty[a]);
                tc_commit(&xempty[x]);
                tc_commit(&gfull[b]);
                ++issued;
            }
            // TMEM is freed at the end: the last MMAs must have completed
            if (issued > 0) {
                const int last = issued - 1;
                if (!mbar_wait(&gfull[last % C::NACC], (uint32_t)(last / C::NACC) & 1u, to))
                    raise_status(p.status, kStatusTimeout);
            }
        }
        __syncwarp();
    } else if (warp < C::FW0) {
        // ---------------------------------------------------- dequantize
        // thread = half hh (64 k) of weight row r (TMEM lane) in every group.
        // CG = 2: a chunk row is 128 bytes, groups 2j and 2j+1 in 16-byte
        // units 0-3 and 4-7 at unit u ^ (r & 7) (128-byte swizzle).
        // CG = 1: a chunk row is 64 bytes, units 0-3 at u ^ ((r >> 1) & 3)
        // (64-byte swizzle).
        const int dw = warp - C::DQ0;
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const int hh = dw >> 2;
        const int sw = CG == 2 ? (r & 7) : ((r >> 1) & 3);
        const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
        uint32_t* dslot = dep_slots + dw * 32 + lane;
        bool ok = true;
        // 8 words (64 codes) of group stage i -> this thread's 32 columns of its A stage
        auto put = [&](int i, const uint32_t* w) -> bool {
            const int a = i % C::NA;
            uint32_t o[32];
#pragma unroll
            for (int k = 0; k < 8; ++k) codes_to_a<XM, MANT>(w[k], o + 4 * k);
            if (!__all_sync(0xffffffffu, mbar_wait(&aempty[a], ((uint32_t)(i / C::NA) & 1u) ^ 1u, to)))
                return false;
            tmem_st32(tl + (uint32_t)(a * 64 + hh * 32), o);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&afull[a]);
            return true;
        };
        for (int j = 0; j < nch && ok; ++j) {
            const int ws = j % C::WCH;
            if (!__all_sync(0xffffffffu, mbar_wait(&wfull[ws], (uint32_t)(j / C::WCH) & 1u, to))) {
                if (lane == 0) raise_status(p.status, kStatusTimeout);
                break;
            }
            const uint8_t* prow = wsr + ws * C::CBYTES + r * C::RB;
            uint32_t w[CG][8];
#pragma unroll
            for (int g = 0; g < CG; ++g)
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const uint4 v = *reinterpret_cast<const uint4*>(prow + (((4 * g + 2 * hh + u) ^ sw) << 4));
                    w[g][4 * u + 0] = v.x;
                    w[g][4 * u + 1] = v.y;
                    w[g][4 * u + 2] = v.z;
                    w[g][4 * u + 3] = v.w;
                }
            // the chunk's words are in registers: release it before converting
            mbar_arrive_after(&wempty[ws], w[0][0] ^ w[CG - 1][4], dslot);
#pragma unroll
            for (int g = 0; g < CG; ++g)
                if (ok) ok = put(j * CG + g, w[g]);
            if (!ok && lane == 0) raise_status(p.status, kStatusTimeout);
        }
    } else {
        // ---------------------------------------------- fold + epilogue
        const int fw = warp - C::FW0;
        const int q = warp & 3;
        const int cb = (fw >> 2) * C::FCOLS;  // first accumulator column (token) of this thread
        const int r = q * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
        const int ft = u0 / G;                 // first tile of this CTA
        float* xrw = xrow_s + fw * C::FCOLS;
        for (int j = lane; j < C::FCOLS; j += 32) {
            const int m = cb + j;
            xrw[j] = XM == kXF16 ? (m < p.M ? p.xrow[m] : 0.f) : 1.f;
        }
        __syncwarp();
        const float rho = p.x_scale ? *p.x_scale : 1.f;
        float tot[C::FCOLS];
#pragma unroll
        for (int j = 0; j < C::FCOLS; ++j) tot[j] = 0.f;
        bool ok = true;
        int seg_g0 = u0 % G;                   // first group of the current tile piece
        // group scales in batches of 8 stages, each batch loaded one batch
        // ahead and parked in shared memory: a load per stage would put one
        // L2 round trip into every stage
        auto scale_of = [&](int i) -> float {  // s[n, g] of stage i for this thread's row
            const int u = u0 + i, n = (u / G) * C::BW + r;
            return (i < nst && n < p.N) ? load_scale(p.scales, p.sdt, (size_t)n * G + (u % G)) : 0.f;
        };
        float* sb = sbuf + (fw * 32 + lane) * 8;
        float snext[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) snext[k] = scale_of(k);
        for (int i = 0; i < nst; ++i) {
            const int b = i % C::NACC;
            if ((i & 7) == 0) {
#pragma unroll
                for (int k = 0; k < 8; ++k) sb[k] = snext[k];
#pragma unroll
                for (int k = 0; k < 8; ++k) snext[k] = scale_of(i + 8 + k);
            }
            const float sc = sb[i & 7];
            if (ok && !__all_sync(0xffffffffu, mbar_wait(&gfull[b], (uint32_t)(i / C::NACC) & 1u, to))) {
                if (lane == 0) raise_status(p.status, kStatusTimeout);
                ok = false;
            }
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int cc = 0; cc < C::FCOLS; cc += 16) {
                    uint32_t v[16];
                    tmem_ld16(tl + (uint32_t)(C::ACC0 + b * BT + cb + cc), v);
                    tmem_ld_wait();
#pragma unroll
                    for (int k = 0; k < 16; ++k) tot[cc + k] = fmaf(sc, __uint_as_float(v[k]), tot[cc + k]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&gempty[b]);
            }
            const int u = u0 + i, t = u / G, g = u % G;
            if (g != G - 1 && i != nst - 1) continue;
            // ------------------------------------------- end of a tile piece
            const int n = t * C::BW + r;
            if (seg_g0 == 0 && g == G - 1) {
                // the whole tile is this CTA's: store it
                if (p.act == kActSiluGate) {
                    // row n ^ 1, the other half of the gate/up pair, is lane ^ 1
#pragma unroll
                    for (int k = 0; k < C::FCOLS; ++k) {
                        const int m = cb + k;
                        const float v = rho * tot[k] * xrw[k];
                        const float w = __shfl_xor_sync(0xffffffffu, v, 1);
                        if (ok && m < p.M && (n & 1) == 0 && n + 1 < p.N)
                            p.Y[(size_t)m * (p.N >> 1) + (n >> 1)] = bf16_bits(silu_gate(v, w));
                    }
                } else if (ok && n < p.N) {
#pragma unroll
                    for (int k = 0; k < C::FCOLS; ++k) {
                        const int m = cb + k;
                        if (m < p.M) {
                            __nv_bfloat16 y = __float2bfloat16_rn(apply_act(rho * tot[k] * xrw[k], p.act));
                            p.Y[(size_t)m * p.N + n] = *reinterpret_cast<uint16_t*>(&y);
                        }
                    }
                }
            } else {
                // a piece: publish the partial tile, count it, and the CTA that
                // completes the tile adds all pieces in CTA order
                float* slot = p.part + (size_t)(2 * c + (t == ft ? 0 : 1)) * (BT * C::BW);
#pragma unroll
                for (int k = 0; k < C::FCOLS; ++k) slot[(cb + k) * C::BW + r] = ok ? tot[k] * xrw[k] : 0.f;
                __threadfence();
                named_barrier_sync(1, C::NF * 32);
                if (fw == 0 && lane == 0) *last_flag = atomicAdd(p.cnt + t, 1);
                named_barrier_sync(1, C::NF * 32);
                const int c_first = chunk_owner(t * cpt, p.C, p.P);
                const int c_last = chunk_owner((t + 1) * cpt - 1, p.C, p.P);
                if (*last_flag == c_last - c_first) {
                    __threadfence();
                    // this thread: kQB quads (4 rows of one token) at a time; the
                    // loads of up to kSB pieces are issued before any is added
                    // (a dependent load per piece would pay an L2 round trip
                    // each), pieces added in CTA order
                    constexpr int kQB = BT <= 32 ? 2 : 1, kSB = 4;
                    const int nseg = c_last - c_first + 1;
                    for (int q0 = fw * 32 + lane; q0 < BT * 32; q0 += kQB * C::NF * 32) {
                        float4 acc[kQB];
#pragma unroll
                        for (int qb = 0; qb < kQB; ++qb) acc[qb] = make_float4(0.f, 0.f, 0.f, 0.f);
                        for (int z0 = 0; z0 < nseg; z0 += kSB) {
                            float4 v[kQB][kSB];
#pragma unroll
                            for (int qb = 0; qb < kQB; ++qb)
#pragma unroll
                                for (int z = 0; z < kSB; ++z) {
                                    const int qd = q0 + qb * C::NF * 32, cc2 = c_first + z0 + z;
                                    v[qb][z] = make_float4(0.f, 0.f, 0.f, 0.f);
                                    if (qd < BT * 32 && z0 + z < nseg) {
                                        const int ft2 = (int)((long long)cc2 * p.C / p.P) * CG / G;
                                        // L2 loads: the pieces were written by other SMs
                                        v[qb][z] = __ldcg(reinterpret_cast<const float4*>(
                                            p.part + (size_t)(2 * cc2 + (t == ft2 ? 0 : 1)) * (BT * C::BW) +
                                            (qd >> 5) * C::BW + (qd & 31) * 4));
                                    }
                                }
#pragma unroll
                            for (int qb = 0; qb < kQB; ++qb)
#pragma unroll
                                for (int z = 0; z < kSB; ++z) {
                                    acc[qb].x += v[qb][z].x;
                                    acc[qb].y += v[qb][z].y;
                                    acc[qb].z += v[qb][z].z;
                                    acc[qb].w += v[qb][z].w;
                                }
                        }
#pragma unroll
                        for (int qb = 0; qb < kQB; ++qb) {
                            const int qd = q0 + qb * C::NF * 32;
                            if (qd >= BT * 32) continue;
                            const int m = qd >> 5, n4 = t * C::BW + (qd & 31) * 4;
                            const float4 a = acc[qb];
                            if (p.act == kActSiluGate) {
                                // the quad is two gate/up pairs
                                if (m < p.M) {
                                    uint16_t* dst = p.Y + (size_t)m * (p.N >> 1) + (n4 >> 1);
                                    if (n4 + 1 < p.N) dst[0] = bf16_bits(silu_gate(rho * a.x, rho * a.y));
                                    if (n4 + 3 < p.N) dst[1] = bf16_bits(silu_gate(rho * a.z, rho * a.w));
                                }
                                continue;
                            }
                            if (m < p.M && n4 < p.N) {
                                const uint32_t y01 = pack_bf16x2(apply_act(rho * a.x, p.act),
                                                                 apply_act(rho * a.y, p.act)),
                                               y23 = pack_bf16x2(apply_act(rho * a.z, p.act),
                                                                 apply_act(rho * a.w, p.act));
                                uint16_t* dst = p.Y + (size_t)m * p.N + n4;
                                if ((p.N & 3) == 0 && n4 + 3 < p.N) {
                                    *reinterpret_cast<uint2*>(dst) = make_uint2(y01, y23);
                                } else {
                                    const uint16_t y[4] = {(uint16_t)(y01 & 0xffffu), (uint16_t)(y01 >> 16),
                                                           (uint16_t)(y23 & 0xffffu), (uint16_t)(y23 >> 16)};
                                    for (int e = 0; e < 4; ++e)
                                        if (n4 + e < p.N) dst[e] = y[e];
                                }
                            }
                        }
                    }
                    if (fw == 0 && lane == 0) p.cnt[t] = 0;  // leave the counter as found
                }
                named_barrier_sync(1, C::NF * 32);  // last_flag is reused by the next piece
            }
#pragma unroll
            for (int k = 0; k < C::FCOLS; ++k) tot[k] = 0.f;
            seg_g0 = 0;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ----------------------------------------------------------- host launch

bool encode_2d(CUtensorMap* map, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t inner,
               uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw);
size_t xh_bytes(int M, int K);
cudaError_t launch_x_rows_to_f16(const uint16_t* X, int M, int K, uint16_t* Xh, float* xrow, int* zero,
                                 int nzero, cudaStream_t st);

int ts_token_tile(int M) { return M <= 16 ? 16 : (M <= 32 ? 32 : 64); }

int device_sm_count() {
    static int sms[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
        sms[dev] = n;
    }
    return sms[dev];
}

// Layout of the decode engine's workspace: prepared activations (f16 rows,
// or re-paired bf16 rows), their row factors, the partial tiles (two per
// CTA) and the per-tile counters, each at a 256-byte boundary.
struct TsLayout {
    size_t xh, xrow, part, cnt, total;
    int tiles, C, P;
};

static size_t up256(size_t b) { return (b + 255) & ~(size_t)255; }

static TsLayout ts_layout(int M, int N, int K, int ctas) {
    TsLayout L;
    const int BT = ts_token_tile(M), G = K / 128, CG = G % 2 == 0 ? 2 : 1;
    L.tiles = (N + 127) / 128;
    L.C = L.tiles * (G / CG);
    L.P = ctas > 0 ? ctas : device_sm_count();
    if (L.P > L.C) L.P = L.C;
    if (L.P < 1) L.P = 1;
    L.xh = 0;
    L.xrow = xh_bytes(M, K);
    L.part = L.xrow + up256((size_t)M * 4);
    L.cnt = L.part + (size_t)2 * L.P * BT * 128 * 4;
    L.total = L.cnt + up256((size_t)L.tiles * 4);
    return L;
}

size_t ts_ws_bytes(int M, int N, int K) {
    if (M <= 0 || N <= 0 || K <= 0 || K % 128) return 0;
    return ts_layout(M, N, K, 0).total;
}

// Activation pre-pass of bf16 paths: every 16-byte chunk of X re-paired
// from (k0..k7) into (k0,k4) (k1,k5) (k2,k6) (k3,k7), the pair order of
// dequant8_exact (one grid-stride pass, 16-byte loads and stores), and the
// GEMM's tile counters zeroed.  Like the f16 pre-pass it lets the GEMM that
// follows start its set-up right away.
__global__ void __launch_bounds__(256) x_rows_repair_kernel(const uint4* __restrict__ X, long long nvec,
                                                            uint4* __restrict__ Xp, int* zero, int nzero) {
    pdl_launch_dependents();
    pdl_wait();  // X may come from the previous kernel in the stream
    if (zero && blockIdx.x == 0)
        for (int i = threadIdx.x; i < nzero; i += 256) zero[i] = 0;
    for (long long i = blockIdx.x * 256ll + threadIdx.x; i < nvec; i += (long long)gridDim.x * 256) {
        const uint4 x = X[i];
        Xp[i] = make_uint4(prmt(x.x, x.z, 0x5410u), prmt(x.x, x.z, 0x7632u), prmt(x.y, x.w, 0x5410u),
                           prmt(x.y, x.w, 0x7632u));
    }
}

static cudaError_t launch_x_rows_repair(const uint16_t* X, int M, int K, uint16_t* Xp, int* zero, int nzero,
                                        cudaStream_t st) {
    const long long nvec = (long long)M * K / 8;
    long long blocks = (nvec + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (blocks < 1) blocks = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks, 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, x_rows_repair_kernel, reinterpret_cast<const uint4*>(X), nvec,
                                       reinterpret_cast<uint4*>(Xp), zero, nzero);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int BT, int CG, int XM, int MANT>
static cudaError_t launch_ts_t(const CUtensorMap& mx, const CUtensorMap& mw, const TsParams& p, cudaStream_t st) {
    using C = TsCfg<BT, CG>;
    auto kern = gemm_ts_kernel<BT, CG, XM, MANT>;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && !attr_set[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.P, 1, 1);
    cfg.blockDim = dim3(C::THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, mx, mw, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int BT, int CG>
static cudaError_t launch_ts_fmt(int fmt, const CUtensorMap& mx, const CUtensorMap& mw, const TsParams& p,
                                 cudaStream_t st) {
    if (fmt == FP4_E2M1) return launch_ts_t<BT, CG, kXF16, 1>(mx, mw, p, st);
    if (fmt == FP4_E1M2) return launch_ts_t<BT, CG, kXBf16, 2>(mx, mw, p, st);
    return launch_ts_t<BT, CG, kXBf16, 0>(mx, mw, p, st);
}

// Decode engine (M <= 64, group 128).  ws must hold ts_ws_bytes(M, N, K)
// bytes; ctas = 0 takes one CTA per SM (at most one per code chunk).
cudaError_t launch_gemm_ts(const uint16_t* X, void* ws, size_t ws_bytes, const uint8_t* packed, const void* scales,
                           int sdt, int fmt, int M, int N, int K, const float* x_scale, uint16_t* Y, int act,
                           int ctas, int* status, unsigned long long timeout_ns, cudaStream_t st) {
    if (K % 128 != 0 || M <= 0 || M > 64 || N <= 0) return cudaErrorInvalidValue;
    const TsLayout L = ts_layout(M, N, K, ctas);
    if (ws == nullptr || ws_bytes < L.total) return cudaErrorInvalidValue;
    const int BT = ts_token_tile(M), G = K / 128, CG = G % 2 == 0 ? 2 : 1;
    uint8_t* w8 = static_cast<uint8_t*>(ws);
    uint16_t* Xp = reinterpret_cast<uint16_t*>(w8 + L.xh);
    float* xrow = reinterpret_cast<float*>(w8 + L.xrow);
    int* cnt = reinterpret_cast<int*>(w8 + L.cnt);
    CUtensorMap mx, mw;
    if (!encode_2d(&mx, fmt == FP4_E2M1 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Xp,
                   (uint64_t)K, (uint64_t)M, 64, (uint32_t)BT, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    // code chunks: 128 rows x CG*64 bytes, 128- or 64-byte swizzle
    if (!encode_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, packed, (uint64_t)K / 2, (uint64_t)N, (uint32_t)(64 * CG),
                   128, CG == 2 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    TsParams p;
    p.xp = Xp;
    p.scales = scales;
    p.sdt = sdt;
    p.M = M;
    p.N = N;
    p.K = K;
    p.x_scale = x_scale;
    p.xrow = xrow;
    p.Y = Y;
    p.part = reinterpret_cast<float*>(w8 + L.part);
    p.cnt = cnt;
    p.C = L.C;
    p.P = L.P;
    p.status = status;
    p.timeout_ns = timeout_ns;
    p.act = act;
    cudaError_t e = fmt == FP4_E2M1 ? launch_x_rows_to_f16(X, M, K, Xp, xrow, cnt, L.tiles, st)
                                    : launch_x_rows_repair(X, M, K, Xp, cnt, L.tiles, st);
    if (e != cudaSuccess) return e;
    if (CG == 2) {
        switch (BT) {
            case 16: return launch_ts_fmt<16, 2>(fmt, mx, mw, p, st);
            case 32: return launch_ts_fmt<32, 2>(fmt, mx, mw, p, st);
            default: return launch_ts_fmt<64, 2>(fmt, mx, mw, p, st);
        }
    }
    switch (BT) {
        case 16: return launch_ts_fmt<16, 1>(fmt, mx, mw, p, st);
        case 32: return launch_ts_fmt<32, 1>(fmt, mx, mw, p, st);
        default: return launch_ts_fmt<64, 1>(fmt, mx, mw, p, st);
    }
}

}  // namespace fp4
