// gemm_tc.cu -- W4A16 GEMM on the sm_100a tensor cores (tcgen05 + TMEM).
//
// Y[m,n] = bf16( rho * sum_g s[n,g] * sum_{k in g} X[m,k] * v(code[n,k]) )
// (LLM-FP4 summary page "首个支持4-bit浮点量化的LLM来了", efficient matrix
// multiplication: the full-precision group scale stays outside the 4-bit
// product.)  The tensor cores multiply the EXACT code values v (bf16 and
// f16 hold every value of the three formats) by the 16-bit activations with
// fp32 accumulation; each group's partial sum is scaled by s in fp32.  No
// weight is ever rounded, so the only rounding besides fp32 accumulation
// is the final bf16 store (and, on the f16 path, the activations' f16
// subnormal range far below each row's maximum: see x_rows_to_f16_kernel).
//
// Two kernels, both with the product computed transposed, D[n][m] = W . X^T:
// the 128 weight rows of a CTA tile (MMA M) map onto the 128 TMEM lanes, so
// the per-row group scale is a per-lane scalar; BT activation rows are MMA N.
//   gemm_tc_kernel<BT, ACT>   groups of 32 or 64: 64-k stages, four TMEM
//                             group accumulators;
//   gemm_tcg_kernel<BT, F16, ACT>  group 128: one group per stage, one
//                             TMEM accumulator per stage (below); ACT
//                             compiles in the output activations.
//
// Warp roles (2 + DQW + NF warps):
//   warp 0       TMA producer: activation tiles (128-byte swizzle) and the
//                packed code tiles (uint8, 128 rows) into shared-memory rings;
//   warp 1       TMEM allocator and MMA issuer: one thread issues tcgen05.mma
//                (K = 16; A from shared memory or, at group 128, from TMEM)
//                into the group's TMEM accumulator and commits;
//   DQW warps    dequantize codes into exact 16-bit values (byte-plane LUT
//                to bf16, or for E2M1 on the f16 path the hardware
//                e2m1x2 -> f16x2 convert): group 32/64 kernel into K-major
//                128-byte-swizzled shared-memory tiles; group-128 kernel
//                into tensor memory, the MMA's A operand (tcgen05.st);
//   NF warps     fold: for each group, tcgen05.ld the group accumulator and
//                add s[n,g] * it to fp32 totals held in registers, then
//                release the accumulator; finally the epilogue: * rho (and
//                the f16 path's token factor) -> bf16 -> global, directly or
//                through shared memory with the dequant warps' help, or fp32
//                split-K partials reduced across a CTA cluster in
//                distributed shared memory.
// Every mbarrier wait is bounded; a wait that gives up sets
// FP4_DEV_WAIT_TIMEOUT and the CTA winds down normally (its copies awaited,
// TMEM freed).  No multicast is used.
#include "common.cuh"

namespace fp4 {

struct TcParams {
    const void* scales;
    int sdt;
    FmtTable t;
    int M, N, K, group;
    const float* x_scale;
    const float* xrow;   // f16 activations: per-row factor 2^e undoing their scaling (else nullptr)
    uint16_t* Y;
    int splits;          // CTAs along K per output tile (one cluster)
    int* status;
    unsigned long long timeout_ns;
    int act;             // output activation (apply_act)
};

template <int BT>
struct TcCfg {
    static constexpr int BW = 128;           // weight rows per tile (MMA M)
    static constexpr int BK = 64;            // k per k-block (one 128-byte swizzle row of bf16)
    static constexpr int KSUP = 4;           // k-blocks per packed-code stage: 128 bytes per weight row
    static constexpr int XBYTES = BT * 128;  // activation tile of one k-block
    static constexpr int ABYTES = BW * 128;  // dequantized weight tile of one k-block
    static constexpr int WBYTES = BW * 128;  // packed codes of KSUP k-blocks
    // small token tiles (decode-sized problems) keep two CTAs per SM
    static constexpr bool kPair = BT <= 64;
    static constexpr int CTAS_PER_SM = kPair ? 2 : 1;
    static constexpr int AST = kPair ? 2 : 3;                      // dequantized tiles
    static constexpr int XST = BT == 32 ? 6 : (BT == 64 ? 3 : 6);  // activation tiles
    static constexpr int WST = BT == 128 ? 4 : 3;                  // packed-code stages
    static constexpr int NACC = 4;                                 // group accumulators in TMEM
    static constexpr int FCOLS = BT < 64 ? BT : 64;  // accumulator columns per fold thread
    static constexpr int FQ = BT / FCOLS;            // column blocks
    static constexpr int NF = 4 * FQ;                // fold warps
    static constexpr int DQW = kPair ? 4 : 8;        // dequant warps (one or two threads per weight row)
    static constexpr int DQ0 = 2;                    // first dequant warp
    static constexpr int FW0 = DQ0 + DQW;            // first fold warp
    static constexpr int THREADS = (FW0 + NF) * 32;
    static_assert(BT <= 128, "fold totals of wider tiles do not fit in registers");
    static constexpr int TMEM_COLS = NACC * BT;
    static constexpr int RING = AST * ABYTES + XST * XBYTES + WST * WBYTES;
    static constexpr int NBAR = 2 * (XST + WST + AST + NACC);
    static constexpr int DEP = DQW * 32 * 4;  // per-dequant-thread scratch words (stage release)
    static constexpr int SMEM = RING + 1024 + NBAR * 8 + 16 + DEP;
    static_assert(BT * 128 * 4 <= AST * ABYTES + XST * XBYTES, "split-K partials overlay the A and X rings");
};

// The k-steps (16 wide) a CTA issues run from kbeg to kstop; groups split
// them into fragments.  Fragment f covers group gfirst + f.
struct KRange {
    int kbeg, kstop, gfirst, nfrag;
};

__device__ __forceinline__ KRange k_range(const TcParams& p, int kb0, int kb1) {
    KRange r;
    r.kbeg = kb0 * 64;
    r.kstop = min(kb1 * 64, p.K);
    r.gfirst = r.kbeg / p.group;
    r.nfrag = r.kstop > r.kbeg ? (r.kstop - 1) / p.group - r.gfirst + 1 : 0;
    return r;
}

__device__ __forceinline__ uint4 lds128_tc(const void* p) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

// Split-K epilogue: the splits of one output tile form a thread-block
// cluster along z, and each CTA has published its fp32 partial tile
// [BT tokens][128 rows] at the start of its shared memory.  Every CTA sums,
// in rank order, one slice of tokens over the partial tiles of all CTAs of
// the cluster (distributed shared memory) and stores it.  Each thread owns
// quads of 4 adjacent rows of one token (16-byte loads) and issues a quad's
// loads from every rank before the first add, so a slice costs a few round
// trips to the other CTAs rather than one per output.
template <int BT>
__device__ __forceinline__ void cluster_reduce_store(const TcParams& p, uint32_t part, int n0, int m0, int act) {
    constexpr int kQ = 1;
    cluster_sync();
    const int rank = (int)cluster_ctarank();
    const int j0 = rank * BT / p.splits, j1 = (rank + 1) * BT / p.splits;
    const int nq = (j1 - j0) * 32;  // quads of rows in this CTA's slice
    const float rho = p.x_scale ? *p.x_scale : 1.f;
    const bool vec_store = (p.N & 3) == 0;
    for (int q0 = threadIdx.x; q0 < nq; q0 += kQ * blockDim.x) {
        float4 v[kQ][8];
#pragma unroll
        for (int u = 0; u < kQ; ++u) {
            const int q = q0 + u * blockDim.x;
            const int j = j0 + (q >> 5), r = (q & 31) * 4;
            const uint32_t off = part + (uint32_t)((j * 128 + r) * 4);
#pragma unroll
            for (int z = 0; z < 8; ++z)
                v[u][z] = (q < nq && z < p.splits) ? ld_dsmem_f32x4(map_dsmem(off, (uint32_t)z))
                                                   : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kQ; ++u) {
            const int q = q0 + u * blockDim.x;
            if (q >= nq) break;
            const int j = j0 + (q >> 5), r = (q & 31) * 4;
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int z = 0; z < 8; ++z) {
                a.x += v[u][z].x;
                a.y += v[u][z].y;
                a.z += v[u][z].z;
                a.w += v[u][z].w;
            }
            const int m = m0 + j, n = n0 + r;
            if (m >= p.M) continue;
            if (p.xrow) {
                const float f = p.xrow[m];
                a.x *= f;
                a.y *= f;
                a.z *= f;
                a.w *= f;
            }
            if (act == kActSiluGate) {
                // 4 rows = 2 gate/up pairs
                uint16_t* dst = p.Y + (size_t)m * (p.N >> 1) + (n >> 1);
                if (n + 1 < p.N) dst[0] = bf16_bits(silu_gate(rho * a.x, rho * a.y));
                if (n + 3 < p.N) dst[1] = bf16_bits(silu_gate(rho * a.z, rho * a.w));
                continue;
            }
            __nv_bfloat16 y[4] = {__float2bfloat16_rn(apply_act(rho * a.x, act)),
                                  __float2bfloat16_rn(apply_act(rho * a.y, act)),
                                  __float2bfloat16_rn(apply_act(rho * a.z, act)),
                                  __float2bfloat16_rn(apply_act(rho * a.w, act))};
            uint16_t* dst = p.Y + (size_t)m * p.N + n;
            if (vec_store && n + 3 < p.N) {
                uint2 w;
                w.x = (uint32_t)(*reinterpret_cast<uint16_t*>(&y[0])) | ((uint32_t)(*reinterpret_cast<uint16_t*>(&y[1])) << 16);
                w.y = (uint32_t)(*reinterpret_cast<uint16_t*>(&y[2])) | ((uint32_t)(*reinterpret_cast<uint16_t*>(&y[3])) << 16);
                *reinterpret_cast<uint2*>(dst) = w;
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (n + e < p.N) dst[e] = *reinterpret_cast<uint16_t*>(&y[e]);
            }
        }
    }
    cluster_sync();  // no CTA leaves while its partials are being read
}

template <int BT, bool ACT>
__global__ void __launch_bounds__(TcCfg<BT>::THREADS, TcCfg<BT>::CTAS_PER_SM)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, TcParams p) {
    using C = TcCfg<BT>;
    const int act = ACT ? p.act : kActNone;  // activation epilogues: own instantiation
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* as = smem;                         // AST x ABYTES: dequantized weight tiles
    uint8_t* xs = as + C::AST * C::ABYTES;      // XST x XBYTES: activation tiles
    uint8_t* wsr = xs + C::XST * C::XBYTES;     // WST x WBYTES: packed-code stages
    uint64_t* bars = reinterpret_cast<uint64_t*>(wsr + C::WST * C::WBYTES);
    uint64_t* xfull = bars;                 // activation tile landed
    uint64_t* xempty = xfull + C::XST;      // MMAs done with the activation tile
    uint64_t* wfull = xempty + C::XST;      // packed codes landed
    uint64_t* wempty = wfull + C::WST;      // packed codes read by the dequant warps
    uint64_t* afull = wempty + C::WST;      // weight tile dequantized
    uint64_t* aempty = afull + C::AST;      // MMAs done with the weight tile
    uint64_t* gfull = aempty + C::AST;      // group accumulator complete
    uint64_t* gempty = gfull + C::NACC;     // group accumulator folded
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gempty + C::NACC);
    uint32_t* dep_slots = tmem_slot + 4;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * C::BW, m0 = blockIdx.y * BT, split = blockIdx.z;
    const int kblocks = (p.K + C::BK - 1) / C::BK;
    const int kb0 = (int)((long long)split * kblocks / p.splits);
    const int kb1 = (int)((long long)(split + 1) * kblocks / p.splits);
    const int nkb = kb1 - kb0;
    const int nsup = (nkb + C::KSUP - 1) / C::KSUP;
    const KRange kr = k_range(p, kb0, kb1);
    const uint64_t to = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::XST; ++s) {
            mbar_init(&xfull[s], 1);
            mbar_init(&xempty[s], 1);
        }
        for (int s = 0; s < C::WST; ++s) {
            mbar_init(&wfull[s], 1);
            mbar_init(&wempty[s], C::DQW * 32);
        }
        for (int s = 0; s < C::AST; ++s) {
            mbar_init(&afull[s], C::DQW * 32);
            mbar_init(&aempty[s], 1);
        }
        for (int b = 0; b < C::NACC; ++b) {
            mbar_init(&gfull[b], 1);
            mbar_init(&gempty[b], C::NF);
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
    pdl_wait();  // inputs may come from the previous kernel in the stream
    pdl_launch_dependents();

    if (warp == 0) {
        // -------------------------------------------------------- producer
        // One thread feeds both rings without blocking on either: packed
        // codes in stages of 128 weight rows x 128 contiguous bytes (KSUP
        // k-blocks), activations per k-block.  It gives up once neither
        // ring has moved for the timeout.
        if (elect_one()) {
            int xi = 0, wj = 0;
            bool ok = true;
            uint64_t t_last = globaltimer_ns();
            while (ok && (xi < nkb || wj < nsup)) {
                bool moved = false;
                if (wj < nsup && mbar_test_wait(&wempty[wj % C::WST], ((uint32_t)(wj / C::WST) & 1u) ^ 1u)) {
                    const int s = wj % C::WST;
                    mbar_arrive_expect_tx(&wfull[s], C::WBYTES);
                    tma_load_2d(wsr + s * C::WBYTES, &tmW, (kb0 + wj * C::KSUP) * (C::BK / 2), n0, &wfull[s]);
                    ++wj;
                    moved = true;
                }
                if (xi < nkb && mbar_test_wait(&xempty[xi % C::XST], ((uint32_t)(xi / C::XST) & 1u) ^ 1u)) {
                    const int s = xi % C::XST;
                    mbar_arrive_expect_tx(&xfull[s], C::XBYTES);
                    tma_load_2d(xs + s * C::XBYTES, &tmX, (kb0 + xi) * C::BK, m0, &xfull[s]);
                    ++xi;
                    moved = true;
                }
                if (moved) {
                    t_last = globaltimer_ns();
                } else if (globaltimer_ns() - t_last > to) {
                    raise_status(p.status, kStatusTimeout);
                    ok = false;
                } else {
                    __nanosleep(32);
                }
            }
            // wait until every copy this thread issued has landed
            for (int i = xi - C::XST < 0 ? 0 : xi - C::XST; i < xi; ++i)
                if (!mbar_wait(&xfull[i % C::XST], (uint32_t)(i / C::XST) & 1u, to)) {
                    raise_status(p.status, kStatusTimeout);
                    break;
                }
            for (int j = wj - C::WST < 0 ? 0 : wj - C::WST; j < wj; ++j)
                if (!mbar_wait(&wfull[j % C::WST], (uint32_t)(j / C::WST) & 1u, to)) {
                    raise_status(p.status, kStatusTimeout);
                    break;
                }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ----------------------------------------------------- MMA issuer
        // One thread issues every MMA, so its own instruction stream is the
        // limit: stage descriptors are built once and advanced by adding
        // the 16-byte-unit offset of each K = 16 step, ring slots and
        // phases are counters, and group bookkeeping runs only at group
        // boundaries.
        if (elect_one()) {
            const uint32_t idesc = idesc_bf16_f32(C::BW, BT);
            const uint64_t adesc0 = sw128_desc(smem_u32(as)), xdesc0 = sw128_desc(smem_u32(xs));
            constexpr uint32_t kAStep = C::ABYTES >> 4, kXStep = C::XBYTES >> 4;
            static_assert((C::NACC & (C::NACC - 1)) == 0, "accumulator count is a power of two");
            constexpr int kNaccShift = C::NACC == 4 ? 2 : (C::NACC == 2 ? 1 : 0);
            const int gmask = p.group - 1;  // group is a power of two
            int a = 0, x = 0;
            uint32_t aph = 0, xph = 0;
            int frag = -1, b = 0;
            int k = kr.kbeg;
            bool ok = true;
            for (int i = 0; i < nkb && ok; ++i) {
                if (!mbar_wait(&afull[a], aph, to) || !mbar_wait(&xfull[x], xph, to)) {
                    raise_status(p.status, kStatusTimeout);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t ad = adesc0 + (uint64_t)(a * kAStep);
                const uint64_t xd = xdesc0 + (uint64_t)(x * kXStep);
#pragma unroll
                for (int kk = 0; kk < C::BK / 16; ++kk) {
                    if (k < kr.kstop) {
                        const bool first = (k == kr.kbeg) || ((k & gmask) == 0);
                        if (first) {
                            // new group fragment: take the next accumulator once it is folded
                            ++frag;
                            b = frag & (C::NACC - 1);
                            if (!mbar_wait(&gempty[b], ((uint32_t)(frag >> kNaccShift) & 1u) ^ 1u, to)) {
                                raise_status(p.status, kStatusTimeout);
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                        }
                        tc_mma_f16(tmem + (uint32_t)(b * BT), ad + (uint64_t)(2 * kk), xd + (uint64_t)(2 * kk), idesc,
                                   first ? 0u : 1u);
                        if ((k + 16 >= kr.kstop) || (((k + 16) & gmask) == 0)) tc_commit(&gfull[b]);
                        k += 16;
                    }
                }
                tc_commit(&aempty[a]);
                tc_commit(&xempty[x]);
                if (++a == C::AST) {
                    a = 0;
                    aph ^= 1u;
                }
                if (++x == C::XST) {
                    x = 0;
                    xph ^= 1u;
                }
            }
            // TMEM is freed below: the last group commit must have landed
            if (frag >= 0 && !mbar_wait(&gfull[frag & (C::NACC - 1)], (uint32_t)(frag >> kNaccShift) & 1u, to))
                raise_status(p.status, kStatusTimeout);
        }
        __syncwarp();
    } else if (warp >= C::DQ0 && warp < C::FW0) {
        // ---------------------------------------------------- dequantize
        // DQW = 4: one thread per weight row (8 words of codes per k-block);
        // DQW = 8: two threads per row, each one 16-byte half (4 words).
        constexpr int kHalves = C::DQW / 4;
        constexpr int kWords = 8 / kHalves;
        const Bf16Lut lut = make_lut(p.t.mag, 1.f);
        const int tid = (warp - C::DQ0) * 32 + lane;
        const int r = tid & 127;                    // weight row within the tile
        const int hh = tid >> 7;                    // half of the row (DQW = 8)
        const int sw = r & 7;                       // 128-byte swizzle (packed stage and weight tile)
        for (int i = 0; i < nkb; ++i) {
            const int j = i / C::KSUP, sub = i % C::KSUP, ws = j % C::WST, a = i % C::AST;
            if (sub == 0 && !mbar_wait(&wfull[ws], (uint32_t)(j / C::WST) & 1u, to)) {
                raise_status(p.status, kStatusTimeout);
                break;
            }
            if (!mbar_wait(&aempty[a], ((uint32_t)(i / C::AST) & 1u) ^ 1u, to)) {
                raise_status(p.status, kStatusTimeout);
                break;
            }
            // 16-byte chunk c of row r sits at chunk c ^ (r & 7); k-block sub
            // of the stage is chunks 2 sub and 2 sub + 1
            const uint8_t* prow = wsr + ws * C::WBYTES + r * 128;
            uint32_t words[kWords];
            uint32_t dep;
            if (kHalves == 1) {
                const uint4 w0 = lds128_tc(prow + (((2 * sub) ^ sw) << 4));
                const uint4 w1 = lds128_tc(prow + (((2 * sub + 1) ^ sw) << 4));
                words[0] = w0.x; words[1] = w0.y; words[2] = w0.z; words[3] = w0.w;
                words[kWords > 4 ? 4 : 0] = w1.x; words[kWords > 5 ? 5 : 0] = w1.y;
                words[kWords > 6 ? 6 : 0] = w1.z; words[kWords > 7 ? 7 : 0] = w1.w;
                dep = w0.x ^ w1.x;
            } else {
                const uint4 w0 = lds128_tc(prow + (((2 * sub + hh) ^ sw) << 4));
                words[0] = w0.x; words[1] = w0.y; words[2] = w0.z; words[3] = w0.w;
                dep = w0.x;
            }
            // release the packed-code stage as soon as its words are in registers
            if (sub == C::KSUP - 1 || i == nkb - 1) mbar_arrive_after(&wempty[ws], dep, dep_slots + tid);
            uint8_t* arow = as + a * C::ABYTES + r * 128;
            const int c0 = hh * kWords;  // first 16-byte unit (8 k) of this thread
#pragma unroll
            for (int c = 0; c < kWords; ++c) {
                uint32_t v[4];
                dequant8(words[c], lut, v);
                *reinterpret_cast<uint4*>(arow + (((c0 + c) ^ sw) << 4)) = make_uint4(v[0], v[1], v[2], v[3]);
            }
            fence_proxy_async_smem();
            mbar_arrive(&afull[a]);
        }
    } else if (warp >= C::FW0) {
        // ---------------------------------------------- fold + epilogue
        const int fw = warp - C::FW0;
        const int q = warp & 3;                  // TMEM lane quadrant of this warp
        const int cb = (fw >> 2) * C::FCOLS;     // first accumulator column of this thread
        const int r = q * 32 + lane;             // weight row within the tile == TMEM lane
        const int n = n0 + r;
        const bool nvalid = n < p.N;
        const int G = p.K / p.group;
        float tot[C::FCOLS];
#pragma unroll
        for (int j = 0; j < C::FCOLS; ++j) tot[j] = 0.f;
        const uint32_t tlane = tmem + ((uint32_t)(q * 32) << 16);
        bool ok = true;
        float s_next = (nvalid && kr.nfrag > 0) ? load_scale(p.scales, p.sdt, (size_t)n * G + kr.gfirst) : 0.f;
        for (int f = 0; f < kr.nfrag; ++f) {
            const int b = f % C::NACC;
            const float s = s_next;
            if (f + 1 < kr.nfrag)
                s_next = nvalid ? load_scale(p.scales, p.sdt, (size_t)n * G + kr.gfirst + f + 1) : 0.f;
            // the warp decides together whether the wait gave up: the TMEM
            // loads below are warp-collective (.sync.aligned)
            if (!__all_sync(0xffffffffu, mbar_wait(&gfull[b], (uint32_t)(f / C::NACC) & 1u, to))) {
                raise_status(p.status, kStatusTimeout);
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < C::FCOLS; c += 16) {
                uint32_t v[16];
                tmem_ld16(tlane + (uint32_t)(b * BT + cb + c), v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) tot[c + j] = fmaf(s, __uint_as_float(v[j]), tot[c + j]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&gempty[b]);
        }
        if (p.splits == 1) {
            const float rho = p.x_scale ? *p.x_scale : 1.f;
            if (ok && nvalid) {
#pragma unroll
                for (int j = 0; j < C::FCOLS; ++j) {
                    const int m = m0 + cb + j;
                    if (m < p.M) {
                        __nv_bfloat16 y = __float2bfloat16_rn(apply_act(rho * tot[j], act));
                        p.Y[(size_t)m * p.N + n] = *reinterpret_cast<uint16_t*>(&y);
                    }
                }
            }
        } else {
            // split-K: publish this CTA's fp32 partial tile [BT tokens][128 rows]
            // in shared memory over the weight and activation tiles (every
            // MMA, and so every copy and dequantization, has completed once
            // the last group has been folded) for the cluster reduction below
            float* part = reinterpret_cast<float*>(smem);
#pragma unroll
            for (int j = 0; j < C::FCOLS; ++j) part[(cb + j) * 128 + r] = tot[j];
        }
    }

    if (p.splits > 1) cluster_reduce_store<BT>(p, smem_u32(smem), n0, m0, act);

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ---------------------------------------------------------------------------
// Group-128 variant (BT in {16, 32, 64} two CTAs per SM; BT = 128 one).
// A k-block is one group (128 k): the MMA thread issues its 8 K=16 steps
// into the stage's own TMEM accumulator and commits ONCE.  That commit both
// frees the stage (dequantized codes, activations) for reuse and hands the
// accumulator to the fold warps.  A commit costs the issuing thread about
// one tensor-pipe round trip, and at these N an MMA issues in ~50 cycles;
// with 64-k stages and separate commits for stage release and group
// completion the commits, not the MMAs, set the pace.
//
// Stage s and accumulator s are the same index (STG == NACC): the next use
// of a stage needs its accumulator folded first, so a stage barrier can
// never run two phases ahead of the fold warps that wait on it.
// The dequant warps write the weights into tensor memory, the A operand
// of `tcgen05.mma` taken from TMEM, not into shared memory: a stage in
// shared memory carries only the activations.  (Dequantized tiles in shared
// memory cost 32 KB written and read back per stage; that traffic set the
// stage period: prefill 873 -> 969 TFLOP/s when they moved to TMEM.)  TMEM
// per CTA: STG accumulators x BT columns + 2 A stages x 64 (512 columns at
// BT = 128, 256 for each of the two CTAs per SM of the smaller tiles).
template <int BT>
struct TgCfg {
    static constexpr int BW = 128;              // weight rows per tile (MMA M)
    static constexpr int KB = 128;              // k per stage = one group
    static constexpr int XBOX = BT * 128;       // activation box: 64 k x BT rows, 128-byte swizzle
    static constexpr int XBYTES = 2 * XBOX;     // activations of one stage (128 k)
    static constexpr int WBYTES = BW * 64;      // packed codes of one stage: 128 rows x 64 B, 64-byte swizzle
    static constexpr bool kPair = BT <= 64;     // two CTAs per SM for small token tiles
    static constexpr int CTAS_PER_SM = kPair ? 2 : 1;
    static constexpr int STG = BT == 128 ? 3 : 2;  // stages == TMEM accumulators
    static constexpr int WST = BT == 16 ? 4 : (BT == 32 || BT == 128 ? 3 : 2);  // packed-code stages
    static constexpr int FCOLS = BT < 64 ? BT : 64;  // accumulator columns per fold thread
    static constexpr int NF = 4 * (BT / FCOLS);      // fold warps: 4 lane quadrants x column blocks
    static constexpr int DQW = kPair ? 4 : 8;   // dequant warps: one thread per row, or two (halves of k)
    static constexpr int DQ0 = 2;
    static constexpr int FW0 = DQ0 + DQW;
    static constexpr int THREADS = (FW0 + NF) * 32;
    static constexpr int NA = 2;                // A stages in TMEM, 64 columns each
    static constexpr int ACOL = STG * BT;       // first TMEM column of the A stages
    static constexpr int TMEM_NEED = STG * BT + NA * 64;
    static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128 : TMEM_NEED <= 256 ? 256 : 512;
    static constexpr int RING = STG * XBYTES + WST * WBYTES;
    static constexpr int NBAR = 4 * STG + 2 * WST + NA;
    static constexpr int DEP = DQW * 32 * 4;  // per-dequant-thread scratch words (stage release)
    // per fold warp, the f16 path's row factors of its FCOLS tokens
    static constexpr int XFB = NF * FCOLS * 4;
    // the 64-token layout only fits two CTAs per SM without alignment slack:
    // it relies on the 1024-byte-aligned dynamic shared-memory base (checked)
    static constexpr int SLACK = BT == 64 ? 0 : 1024;
    static constexpr int SMEM = RING + SLACK + NBAR * 8 + 16 + DEP + XFB;
    static_assert(!kPair || SMEM + 1024 <= 228 * 1024 / 2, "two CTAs per SM");
    static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
    static_assert(BT * 128 * 4 <= STG * XBYTES, "split-K partials overlay the activation stages");
    static_assert(TMEM_NEED <= (kPair ? 256 : 512), "TMEM per CTA");
};

template <int BT, bool F16, bool ACT>
__global__ void __launch_bounds__(TgCfg<BT>::THREADS, TgCfg<BT>::CTAS_PER_SM)
    gemm_tcg_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, TcParams p) {
    using C = TgCfg<BT>;
    // The activation epilogues are a separate instantiation: compiled into
    // the plain kernel, they cost the 128-token tile its register budget.
    const int act = ACT ? p.act : kActNone;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    if (C::SLACK == 0 && smem != smem_raw) {
        if (threadIdx.x == 0) raise_status(p.status, kStatusLayout);
        return;  // before any barrier, copy or TMEM allocation
    }
    uint8_t* xs = smem;                         // STG x XBYTES: activations
    uint8_t* wsr = xs + C::STG * C::XBYTES;     // WST x WBYTES: packed codes
    uint64_t* bars = reinterpret_cast<uint64_t*>(wsr + C::WST * C::WBYTES);
    uint64_t* xfull = bars;                 // activations landed
    uint64_t* afull = xfull + C::STG;       // codes dequantized
    uint64_t* kdone = afull + C::STG;       // the stage's MMAs completed (stage free, accumulator ready)
    uint64_t* wfull = kdone + C::STG;       // packed codes landed
    uint64_t* wempty = wfull + C::WST;      // packed codes read
    uint64_t* gempty = wempty + C::WST;     // accumulator folded (kdone's one arrival is the commit)
    uint64_t* aempty = gempty + C::STG;     // [NA] the MMAs have read the A stage
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(aempty + C::NA);
    uint32_t* dep_slots = tmem_slot + 4;
    float* xf_slots = reinterpret_cast<float*>(dep_slots + C::DEP / 4);
    volatile int* wide_fail = reinterpret_cast<volatile int*>(tmem_slot + 1);
    // the 128-token tile without split stores through shared memory in
    // 16-byte chunks (rows of N bf16 must be multiples of 16 bytes)
    const bool wide = !C::kPair && p.splits == 1 && (p.N & 7) == 0;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * C::BW, m0 = blockIdx.y * BT, split = blockIdx.z;
    const int kblocks = p.K / C::KB;
    const int kb0 = (int)((long long)split * kblocks / p.splits);
    const int kb1 = (int)((long long)(split + 1) * kblocks / p.splits);
    const int nkb = kb1 - kb0;
    const uint64_t to = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STG; ++s) {
            mbar_init(&xfull[s], 1);
            mbar_init(&afull[s], C::DQW);
            mbar_init(&kdone[s], 1);
            mbar_init(&gempty[s], C::NF);
        }
        for (int a = 0; a < C::NA; ++a) mbar_init(&aempty[a], 1);
        for (int s = 0; s < C::WST; ++s) {
            mbar_init(&wfull[s], 1);
            mbar_init(&wempty[s], C::DQW * 32);
        }
        fence_mbar_init();
        prefetch_tmap(&tmX);
        prefetch_tmap(&tmW);
        *wide_fail = 0;
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // The packed codes are inputs that no kernel still running may write (the
    // previous kernel in the stream triggers this launch early only when it
    // is one of these GEMMs), so the first ring-full of them goes out before
    // the dependency wait; the activations follow after it.
    const int wpre = nkb < C::WST ? nkb : C::WST;
    if (warp == 0 && elect_one()) {
        for (int j = 0; j < wpre; ++j) {
            mbar_arrive_expect_tx(&wfull[j], C::WBYTES);
            tma_load_2d(wsr + j * C::WBYTES, &tmW, (kb0 + j) * (C::KB / 2), n0, &wfull[j]);
        }
    }
    __syncwarp();
    pdl_wait();  // the activations, rho, row factors and the output involve the previous kernel
    pdl_launch_dependents();

    if (warp == 0) {
        // -------------------------------------------------------- producer
        if (elect_one()) {
            int xi = 0, wj = wpre;
            bool ok = true;
            uint64_t t_last = globaltimer_ns();
            while (ok && (xi < nkb || wj < nkb)) {
                bool moved = false;
                if (wj < nkb && mbar_test_wait(&wempty[wj % C::WST], ((uint32_t)(wj / C::WST) & 1u) ^ 1u)) {
                    const int s = wj % C::WST;
                    mbar_arrive_expect_tx(&wfull[s], C::WBYTES);
                    tma_load_2d(wsr + s * C::WBYTES, &tmW, (kb0 + wj) * (C::KB / 2), n0, &wfull[s]);
                    ++wj;
                    moved = true;
                }
                if (xi < nkb && mbar_test_wait(&kdone[xi % C::STG], ((uint32_t)(xi / C::STG) & 1u) ^ 1u)) {
                    const int s = xi % C::STG;
                    mbar_arrive_expect_tx(&xfull[s], C::XBYTES);
                    tma_load_2d(xs + s * C::XBYTES, &tmX, (kb0 + xi) * C::KB, m0, &xfull[s]);
                    tma_load_2d(xs + s * C::XBYTES + C::XBOX, &tmX, (kb0 + xi) * C::KB + 64, m0, &xfull[s]);
                    ++xi;
                    moved = true;
                }
                if (moved) {
                    t_last = globaltimer_ns();
                } else if (globaltimer_ns() - t_last > to) {
                    raise_status(p.status, kStatusTimeout);
                    ok = false;
                } else {
                    __nanosleep(32);
                }
            }
            for (int i = xi - C::STG < 0 ? 0 : xi - C::STG; i < xi; ++i)
                if (!mbar_wait(&xfull[i % C::STG], (uint32_t)(i / C::STG) & 1u, to)) {
                    raise_status(p.status, kStatusTimeout);
                    break;
                }
            for (int j = wj - C::WST < 0 ? 0 : wj - C::WST; j < wj; ++j)
                if (!mbar_wait(&wfull[j % C::WST], (uint32_t)(j / C::WST) & 1u, to)) {
                    raise_status(p.status, kStatusTimeout);
                    break;
                }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ----------------------------------------------------- MMA issuer
        if (elect_one()) {
            // A from TMEM: stage i's weights at columns ACOL + (i % NA) * 64
            const uint32_t idesc = F16 ? idesc_f16_f32(C::BW, BT) : idesc_bf16_f32(C::BW, BT);
            const uint64_t xdesc0 = sw128_desc(smem_u32(xs));
            constexpr uint32_t kXStep = C::XBYTES >> 4, kXAtom = C::XBOX >> 4;
            int committed = 0;
            bool ok = true;
            for (int i = 0; i < nkb && ok; ++i) {
                const int s = i % C::STG, a = i % C::NA;
                if (!mbar_wait(&afull[a], (uint32_t)(i / C::NA) & 1u, to) ||
                    !mbar_wait(&xfull[s], (uint32_t)(i / C::STG) & 1u, to) ||
                    !mbar_wait(&gempty[s], ((uint32_t)(i / C::STG) & 1u) ^ 1u, to)) {
                    raise_status(p.status, kStatusTimeout);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t xd = xdesc0 + (uint64_t)(s * kXStep);
                const uint32_t ta = tmem + (uint32_t)(C::ACOL + a * 64);
                const uint32_t d = tmem + (uint32_t)(s * BT);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc_mma_ts(d, ta + (uint32_t)(8 * kk), xd + (uint64_t)((kk >> 2) * kXAtom + 2 * (kk & 3)), idesc,
                              kk ? 1u : 0u);
                tc_commit(&aempty[a]);
                tc_commit(&kdone[s]);
                ++committed;
            }
            if (committed > 0) {
                const int last = committed - 1;
                if (!mbar_wait(&kdone[last % C::STG], (uint32_t)(last / C::STG) & 1u, to))
                    raise_status(p.status, kStatusTimeout);
            }
        }
        __syncwarp();
    } else if (warp >= C::DQ0 && warp < C::FW0) {
        // ------------------------------------------- dequantize into TMEM
        // DQW = 4: one thread per weight row (16 words = 128 k per stage);
        // DQW = 8: two threads per row, each one 64-k half (8 words).  The
        // row is the thread's TMEM lane, so each warp covers the lane
        // quadrant it may access.  A word (8 codes) becomes 4 columns of
        // 16-bit pairs (k, k+1), the A layout of kind::f16 from TMEM: f16
        // by the hardware e2m1 convert, or bf16 by the byte-plane LUT.
        constexpr int kHalves = C::DQW / 4;
        constexpr int kWords = 16 / kHalves;
        const Bf16Lut lut = make_lut(p.t.mag, 1.f);
        const int dw = warp - C::DQ0;
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const int hh = dw >> 2;
        const int swp = (r >> 1) & 3;  // 64-byte swizzle of the packed stage
        const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
        for (int i = 0; i < nkb; ++i) {
            const int ws = i % C::WST, a = i % C::NA;
            if (!__all_sync(0xffffffffu, mbar_wait(&wfull[ws], (uint32_t)(i / C::WST) & 1u, to))) {
                raise_status(p.status, kStatusTimeout);
                break;
            }
            // 16-byte unit u of the row's 64 bytes sits at unit u ^ ((r >> 1) & 3)
            const uint8_t* prow = wsr + ws * C::WBYTES + r * 64;
            uint32_t words[kWords];
            uint32_t dep = 0;
#pragma unroll
            for (int u = 0; u < kWords / 4; ++u) {
                const uint4 w = lds128_tc(prow + (((u + (kWords / 4) * hh) ^ swp) << 4));
                words[4 * u + 0] = w.x;
                words[4 * u + 1] = w.y;
                words[4 * u + 2] = w.z;
                words[4 * u + 3] = w.w;
                dep ^= w.x;
            }
            // release the packed-code stage once its words are in registers
            mbar_arrive_after(&wempty[ws], dep, dep_slots + dw * 32 + lane);
            if (!__all_sync(0xffffffffu, mbar_wait(&aempty[a], ((uint32_t)(i / C::NA) & 1u) ^ 1u, to))) {
                raise_status(p.status, kStatusTimeout);
                break;
            }
#pragma unroll
            for (int h = 0; h < kWords / 8; ++h) {
                uint32_t o[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    if constexpr (F16)
                        e2m1_to_f16x8(words[8 * h + c], o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
                    else
                        dequant8(words[8 * h + c], lut, o + 4 * c);
                }
                tmem_st32(tl + (uint32_t)(C::ACOL + a * 64 + (hh + h) * 32), o);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&afull[a]);
        }
    } else if (warp >= C::FW0) {
        // ---------------------------------------------- fold + epilogue
        const int fw = warp - C::FW0;
        const int q = warp & 3;                  // TMEM lane quadrant of this warp
        const int cb = (fw >> 2) * C::FCOLS;     // first accumulator column of this thread
        const int r = q * 32 + lane;             // weight row within the tile == TMEM lane
        const int n = n0 + r;
        const bool nvalid = n < p.N;
        const int G = p.K / 128;
        // epilogue inputs, fetched before the stages: rho, and on the f16 path
        // this warp's token factors (in shared memory, read back as broadcasts)
        const float rho = p.x_scale ? *p.x_scale : 1.f;
        float* xfw = xf_slots + fw * C::FCOLS;
        if constexpr (F16) {
            for (int j = lane; j < C::FCOLS; j += 32) {
                const int m = m0 + cb + j;
                xfw[j] = m < p.M ? p.xrow[m] : 0.f;
            }
            __syncwarp();
        }
        float tot[C::FCOLS];
#pragma unroll
        for (int j = 0; j < C::FCOLS; ++j) tot[j] = 0.f;
        const uint32_t tlane = tmem + ((uint32_t)(q * 32) << 16);
        bool ok = true;
        float s_next = (nvalid && nkb > 0) ? load_scale(p.scales, p.sdt, (size_t)n * G + kb0) : 0.f;
        for (int i = 0; i < nkb; ++i) {
            const int s = i % C::STG;
            const float sc = s_next;
            if (i + 1 < nkb) s_next = nvalid ? load_scale(p.scales, p.sdt, (size_t)n * G + kb0 + i + 1) : 0.f;
            // the warp decides together whether the wait gave up: the TMEM
            // loads below are warp-collective (.sync.aligned)
            if (!__all_sync(0xffffffffu, mbar_wait(&kdone[s], (uint32_t)(i / C::STG) & 1u, to))) {
                raise_status(p.status, kStatusTimeout);
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < C::FCOLS; c += 16) {
                uint32_t v[16];
                tmem_ld16(tlane + (uint32_t)(s * BT + cb + c), v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) tot[c + j] = fmaf(sc, __uint_as_float(v[j]), tot[c + j]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&gempty[s]);
        }
        if (wide) {
            // every MMA, and so every copy and dequantization, has completed
            // once the last stage has been folded: the fp32 tile [128 tokens]
            // [128 rows] * rho goes over the activation stages (row =
            // token: the lanes' consecutive weight rows are consecutive words)
            // and all dequant and fold warps store it below.  No loads here:
            // a load per element would serialise on its latency.
            float* ep = reinterpret_cast<float*>(smem);
            if (!ok) *wide_fail = 1;
#pragma unroll
            for (int j = 0; j < C::FCOLS; ++j) ep[(cb + j) * 128 + r] = rho * tot[j];
        } else if (p.splits == 1) {
            if (ok && act == kActSiluGate) {
                // row n ^ 1, the other half of the gate/up pair, is lane ^ 1
#pragma unroll
                for (int j = 0; j < C::FCOLS; ++j) {
                    const int m = m0 + cb + j;
                    const float v = rho * (F16 ? tot[j] * xfw[j] : tot[j]);
                    const float w = __shfl_xor_sync(0xffffffffu, v, 1);
                    if (m < p.M && (n & 1) == 0 && n + 1 < p.N)
                        p.Y[(size_t)m * (p.N >> 1) + (n >> 1)] = bf16_bits(silu_gate(v, w));
                }
            } else if (ok && nvalid) {
#pragma unroll
                for (int j = 0; j < C::FCOLS; ++j) {
                    const int m = m0 + cb + j;
                    if (m < p.M) {
                        const float t = F16 ? tot[j] * xfw[j] : tot[j];
                        __nv_bfloat16 y = __float2bfloat16_rn(apply_act(rho * t, act));
                        p.Y[(size_t)m * p.N + n] = *reinterpret_cast<uint16_t*>(&y);
                    }
                }
            }
        } else {
            // every MMA, and so every copy and dequantization, has completed
            // once the last stage has been folded: the partial tile
            // [BT tokens][128 rows] overlays the activation stages
            float* part = reinterpret_cast<float*>(smem);
#pragma unroll
            for (int j = 0; j < C::FCOLS; ++j) part[(cb + j) * 128 + r] = tot[j];
        }
    }

    if (p.splits > 1) cluster_reduce_store<BT>(p, smem_u32(smem), n0, m0, act);
    if (wide && warp >= C::DQ0) {
        // 16-byte output chunks (8 weight rows of one token) over the dequant
        // and fold warps: the f16 path's token factor, bf16x2 converts and
        // coalesced vector stores, all chunks' loads issued first
        constexpr int kT = (C::DQW + C::NF) * 32, kC = BT * 16 / kT;
        static_assert(BT * 16 % kT == 0, "whole chunks per thread");
        named_barrier_sync(1, kT);
        if (*wide_fail == 0) {
            const float* ep = reinterpret_cast<const float*>(smem);
            const int c0 = (int)threadIdx.x - C::DQ0 * 32;
            float4 a[kC], b[kC];
            float f[kC];
#pragma unroll
            for (int u = 0; u < kC; ++u) {
                const int c = c0 + u * kT, j = c >> 4, m = m0 + j;
                a[u] = *reinterpret_cast<const float4*>(ep + j * 128 + (c & 15) * 8);
                b[u] = *reinterpret_cast<const float4*>(ep + j * 128 + (c & 15) * 8 + 4);
                f[u] = F16 && m < p.M ? p.xrow[m] : 1.f;
            }
#pragma unroll
            for (int u = 0; u < kC; ++u) {
                const int c = c0 + u * kT, j = c >> 4, n = n0 + (c & 15) * 8, m = m0 + j;
                if (m < p.M && n < p.N && act == kActSiluGate) {
                    // 8 rows = 4 gate/up pairs -> 4 outputs (N % 8 == 0 on this path)
                    uint2 o;
                    o.x = pack_bf16x2(silu_gate(a[u].x * f[u], a[u].y * f[u]), silu_gate(a[u].z * f[u], a[u].w * f[u]));
                    o.y = pack_bf16x2(silu_gate(b[u].x * f[u], b[u].y * f[u]), silu_gate(b[u].z * f[u], b[u].w * f[u]));
                    *reinterpret_cast<uint2*>(p.Y + (size_t)m * (p.N >> 1) + (n >> 1)) = o;
                } else if (m < p.M && n < p.N) {
                    uint4 o;
                    o.x = pack_bf16x2(apply_act(a[u].x * f[u], act), apply_act(a[u].y * f[u], act));
                    o.y = pack_bf16x2(apply_act(a[u].z * f[u], act), apply_act(a[u].w * f[u], act));
                    o.z = pack_bf16x2(apply_act(b[u].x * f[u], act), apply_act(b[u].y * f[u], act));
                    o.w = pack_bf16x2(apply_act(b[u].z * f[u], act), apply_act(b[u].w * f[u], act));
                    *reinterpret_cast<uint4*>(p.Y + (size_t)m * p.N + n) = o;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

// ----------------------------------------------------------- host launch

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

bool encode_2d(CUtensorMap* map, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t inner,
                      uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * (uint64_t)elem_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 4-bit codes, packed two per byte in rows of `elems` codes, copied as
// 16 x U4 with 16-byte alignment: every 16 codes (8 bytes) land in a
// 16-byte slot of shared memory, the operand layout of kind::f8f6f4 MMAs.
// Boxes of 128 codes x box_rows rows under the 128-byte swizzle.
bool encode_2d_u4(CUtensorMap* map, const void* base, uint64_t elems, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {elems, rows};
    cuuint64_t strides[1] = {elems / 2};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// A 3-D view {inner, mid, outer} with byte strides {mid_stride, outer_stride},
// no swizzle (used for L2 prefetches of several consecutive segments per row).
bool encode_3d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t mid,
               uint64_t outer, uint64_t mid_stride, uint64_t outer_stride, uint32_t box_inner, uint32_t box_mid,
               uint32_t box_outer) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {inner, mid, outer};
    cuuint64_t strides[2] = {mid_stride, outer_stride};
    cuuint32_t box[3] = {box_inner, box_mid, box_outer};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int tc_token_tile(int M) {
    if (M <= 32) return 32;
    if (M <= 64) return 64;
    return 128;
}

int tc_splits(int M, int N, int K) {
    // split K (a cluster of at most 8 CTAs per output tile) only as far as
    // one wave of CTAs covers the SMs
    const int BT = tc_token_tile(M);
    const long long tiles = (long long)((N + 127) / 128) * ((M + BT - 1) / BT);
    const int kblocks = (K + 63) / 64;
    const long long slots = 148LL * (BT <= 64 ? 2 : 1);
    if (tiles >= slots / 2) return 1;
    long long s = slots / tiles;
    if (s > kblocks / 4) s = kblocks / 4;
    if (s > 8) s = 8;
    return s < 1 ? 1 : (int)s;
}

// The split-K reduction runs in distributed shared memory and needs no
// workspace; the f16 activations of the 128-token tile do (M > 64).
size_t tc_f16_ws_bytes(int M, int K);
size_t tc_ws_bytes(int M, int N, int K) {
    (void)N;
    return M > 64 && K > 0 ? tc_f16_ws_bytes(M, K) : 0;
}

template <int BT>
static cudaError_t launch_tc_bt(const CUtensorMap& mx, const CUtensorMap& mw, const TcParams& p, cudaStream_t st) {
    using C = TcCfg<BT>;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BT, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gemm_tc_kernel<BT, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    dim3 grid((p.N + C::BW - 1) / C::BW, (p.M + BT - 1) / BT, p.splits);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(C::THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = (unsigned)p.splits;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = p.act != kActNone ? cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BT, true>, mx, mw, p)
                                      : cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BT, false>, mx, mw, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// Activations of the f16 tensor path.  Row m of X (bf16) is multiplied by
// 2^sh, the power of two that brings its largest finite magnitude into
// [2^14, 2^15) (sh clamped to [-113, 126]), and rounded to f16; xrow[m] =
// 2^-sh undoes it in the epilogue.  The scaling is exact, and a bf16 value
// (8 significant bits) converts to f16 exactly when its scaled magnitude is
// at least 2^-17: every element within 2^31 of the row's maximum.  Smaller
// ones round to the f16 subnormal grid (error below 2^-25 after scaling,
// i.e. under 2^-39 of the row maximum); infinities and NaNs pass through.
//
// R = 16-byte vectors of the row each thread keeps in registers (one read
// of X); R = 0 reads the row twice (any K).  T threads per row: 256, or 128
// for many rows (twice the bytes in flight per thread, and all of a
// 2048-row prefill resident in one wave).
template <int R, int T>
__global__ void __launch_bounds__(T) x_rows_to_f16_kernel(const uint16_t* __restrict__ X, int K,
                                                          uint16_t* __restrict__ Xh, float* __restrict__ xrow,
                                                          int* zero, int nzero) {
    __shared__ uint32_t wmax[T / 32];
    const int m = blockIdx.x, nv = K >> 3;
    const uint4* src = reinterpret_cast<const uint4*>(X + (size_t)m * K);
    uint4* dst = reinterpret_cast<uint4*>(Xh + (size_t)m * K);
    // the GEMM that follows only sets up (and starts its weights towards L2)
    // before its own dependency wait, so it may be launched right away
    pdl_launch_dependents();
    pdl_wait();  // X may come from the previous kernel in the stream
    // the decode engine's tile counters start at zero
    if (zero && m == 0)
        for (int i = threadIdx.x; i < nzero; i += T) zero[i] = 0;
    uint32_t mx2 = 0;  // per-half maxima of the finite magnitudes (bf16 bits order like the values)
    uint4 v[R > 0 ? R : 1];
    if constexpr (R > 0) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int i = threadIdx.x + r * T;
            v[r] = i < nv ? src[i] : make_uint4(0u, 0u, 0u, 0u);
            mx2 = finite_mag_max2(mx2, v[r].x);
            mx2 = finite_mag_max2(mx2, v[r].y);
            mx2 = finite_mag_max2(mx2, v[r].z);
            mx2 = finite_mag_max2(mx2, v[r].w);
        }
    } else {
        for (int i = threadIdx.x; i < nv; i += T) {
            const uint4 u = src[i];
            mx2 = finite_mag_max2(finite_mag_max2(finite_mag_max2(finite_mag_max2(mx2, u.x), u.y), u.z), u.w);
        }
    }
    uint32_t mx = max(mx2 & 0xffffu, mx2 >> 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = mx;
    __syncthreads();
    mx = wmax[0];
#pragma unroll
    for (int w = 1; w < T / 32; ++w) mx = max(mx, wmax[w]);
    const int E = (int)(mx >> 7);  // biased exponent of the row maximum
    int sh = mx == 0 ? 0 : 141 - (E < 1 ? 1 : E);
    if (sh > 126) sh = 126;
    const float sc = __int_as_float((127 + sh) << 23);
    if (threadIdx.x == 0) xrow[m] = __int_as_float((127 - sh) << 23);
    if constexpr (R > 0) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int i = threadIdx.x + r * T;
            if (i < nv) dst[i] = bf16x8_to_f16x8(v[r], sc);
        }
    } else {
        for (int i = threadIdx.x; i < nv; i += T) dst[i] = bf16x8_to_f16x8(src[i], sc);
    }
}

// Bytes of the f16 activations (16-byte aligned rows) and their row factors.
size_t xh_bytes(int M, int K) { return ((size_t)M * K * 2 + 255) & ~(size_t)255; }

size_t tc_f16_ws_bytes(int M, int K) { return xh_bytes(M, K) + (size_t)M * 4; }

cudaError_t launch_x_rows_to_f16(const uint16_t* X, int M, int K, uint16_t* Xh, float* xrow, int* zero, int nzero,
                                 cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    const bool narrow = M >= 1024;  // 128 threads per row
    cfg.gridDim = dim3((unsigned)M, 1, 1);
    cfg.blockDim = dim3(narrow ? 128 : 256, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int nv = K / 8;
    cudaError_t e;
    if (narrow) {
        if (nv <= 128) e = cudaLaunchKernelEx(&cfg, x_rows_to_f16_kernel<1, 128>, X, K, Xh, xrow, zero, nzero);
        else if (nv <= 256) e = cudaLaunchKernelEx(&cfg, x_rows_to_f16_kernel<2, 128>, X, K, Xh, xrow, zero, nzero);
        else if (nv <= 512) e = cudaLaunchKernelEx(&cfg, x_rows_to_f16_kernel<4, 128>, X, K, Xh, xrow, zero, nzero);
        else if (nv <= 1024) e = cudaLaunchKernelEx(&cfg, x_rows_to_f16_kernel<8, 128>, X, K, Xh, xrow, zero, nzero);
        else if (nv <= 2048) e = cudaLaunchKernelEx(&cfg, x_rows_to_f16_kernel<16, 128>, X, K, Xh, xrow, zero, nzero);
        else e = cudaLaunchKernelEx(&cfg, x_rows_to_f16_kernel<0, 128>, X, K, Xh, xrow, zero, nzero);
    } else {
        if (nv <= 256) e = cudaLaunchKernelEx(&cfg, x_rows_to_f16_kernel<1, 256>, X, K, Xh, xrow, zero, nzero);
        else if (nv <= 512) e = cudaLaunchKernelEx(&cfg, x_rows_to_f16_kernel<2, 256>, X, K, Xh, xrow, zero, nzero);
        else if (nv <= 1024) e = cudaLaunchKernelEx(&cfg, x_rows_to_f16_kernel<4, 256>, X, K, Xh, xrow, zero, nzero);
        else if (nv <= 2048) e = cudaLaunchKernelEx(&cfg, x_rows_to_f16_kernel<8, 256>, X, K, Xh, xrow, zero, nzero);
        else e = cudaLaunchKernelEx(&cfg, x_rows_to_f16_kernel<0, 256>, X, K, Xh, xrow, zero, nzero);
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int BT, bool F16>
static cudaError_t launch_tcg_bt(const CUtensorMap& mx, const CUtensorMap& mw, const TcParams& p, cudaStream_t st) {
    using C = TgCfg<BT>;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(gemm_tcg_kernel<BT, F16, false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gemm_tcg_kernel<BT, F16, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((p.N + C::BW - 1) / C::BW, (p.M + BT - 1) / BT, p.splits);
    cfg.blockDim = dim3(C::THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = (unsigned)p.splits;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = p.act != kActNone ? cudaLaunchKernelEx(&cfg, gemm_tcg_kernel<BT, F16, true>, mx, mw, p)
                                      : cudaLaunchKernelEx(&cfg, gemm_tcg_kernel<BT, F16, false>, mx, mw, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// Token tile and split count of the group-128 small-M variant (0 when it
// does not apply): one wave of two CTAs per SM, at least two 128-k stages
// per split, at most 8 splits (one cluster).
int tcg_token_tile(int M, int K, int group) {
    if (group != 128 || K % 128 != 0) return 0;
    return M <= 16 ? 16 : (M <= 32 ? 32 : (M <= 64 ? 64 : 128));
}

int tcg_splits(int M, int N, int K) {
    const int BT = M <= 16 ? 16 : (M <= 32 ? 32 : (M <= 64 ? 64 : 128));
    const long long tiles = (long long)((N + 127) / 128) * ((M + BT - 1) / BT);
    const int kblocks = K / 128;
    const long long slots = 148LL * (BT <= 64 ? 2 : 1);
    long long s = (slots + tiles - 1) / tiles;
    if (tiles * s > slots + slots / 8) s = slots / tiles;
    if (s > kblocks / 2) s = kblocks / 2;
    if (s > 8) s = 8;
    return s < 1 ? 1 : (int)s;
}

cudaError_t launch_gemm_tc(const uint16_t* X, const uint8_t* packed, const void* scales, int sdt, const FmtTable& t,
                           bool e2m1, int M, int N, int K, int group, const float* x_scale, uint16_t* Y, int act,
                           void* ws, size_t ws_bytes, int splits, int* status, unsigned long long timeout_ns,
                           cudaStream_t st) {
    const int BTg = tcg_token_tile(M, K, group);
    if (BTg > 0) {
        if (splits <= 0) splits = tcg_splits(M, N, K);
        if (splits > K / 128) splits = K / 128;
        if (splits > 8) splits = 8;
        // E2M1 codes: hardware convert to f16 and f16 activations (needs the
        // workspace; without it the bf16 path runs).  Not on the 64-token
        // tile: there the row pre-pass costs what the convert saves (measured
        // on 4096x11008: 17.3 us bf16, 17.9 us f16; at 16 tokens 14.5 -> 12.9)
        const bool f16 = e2m1 && BTg != 64 && ws != nullptr && ws_bytes >= tc_f16_ws_bytes(M, K);
        uint16_t* Xh = f16 ? static_cast<uint16_t*>(ws) : nullptr;
        float* xrow = f16 ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + xh_bytes(M, K)) : nullptr;
        CUtensorMap mx, mw;
        if (!encode_2d(&mx, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                       f16 ? Xh : X, (uint64_t)K, (uint64_t)M, 64, (uint32_t)BTg, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        if (!encode_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, packed, (uint64_t)K / 2, (uint64_t)N, 64, 128,
                       CU_TENSOR_MAP_SWIZZLE_64B))
            return cudaErrorInvalidValue;
        TcParams p;
        p.scales = scales;
        p.sdt = sdt;
        p.t = t;
        p.M = M;
        p.N = N;
        p.K = K;
        p.group = group;
        p.x_scale = x_scale;
        p.xrow = xrow;
        p.Y = Y;
        p.splits = splits;
        p.status = status;
        p.timeout_ns = timeout_ns;
        p.act = act;
        if (f16) {
            cudaError_t e = launch_x_rows_to_f16(X, M, K, Xh, xrow, nullptr, 0, st);
            if (e != cudaSuccess) return e;
            switch (BTg) {
                case 16: return launch_tcg_bt<16, true>(mx, mw, p, st);
                case 32: return launch_tcg_bt<32, true>(mx, mw, p, st);
                default: return launch_tcg_bt<128, true>(mx, mw, p, st);
            }
        }
        switch (BTg) {
            case 16: return launch_tcg_bt<16, false>(mx, mw, p, st);
            case 32: return launch_tcg_bt<32, false>(mx, mw, p, st);
            case 64: return launch_tcg_bt<64, false>(mx, mw, p, st);
            default: return launch_tcg_bt<128, false>(mx, mw, p, st);
        }
    }
    const int BT = tc_token_tile(M);
    const int kblocks = (K + 63) / 64;
    if (splits <= 0) splits = tc_splits(M, N, K);
    if (splits > kblocks) splits = kblocks;
    if (splits > 8) splits = 8;
    CUtensorMap mx, mw;
    if (!encode_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, (uint64_t)K, (uint64_t)M, 64, (uint32_t)BT,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!encode_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, packed, (uint64_t)K / 2, (uint64_t)N, 128, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    TcParams p;
    p.scales = scales;
    p.sdt = sdt;
    p.t = t;
    p.M = M;
    p.N = N;
    p.K = K;
    p.group = group;
    p.x_scale = x_scale;
    p.xrow = nullptr;
    p.Y = Y;
    p.splits = splits;
    p.status = status;
    p.timeout_ns = timeout_ns;
    p.act = act;
    switch (BT) {
        case 32: return launch_tc_bt<32>(mx, mw, p, st);
        case 64: return launch_tc_bt<64>(mx, mw, p, st);
        default: return launch_tc_bt<128>(mx, mw, p, st);
    }
}

}  // namespace fp4

// ------------------------------------------------------- bounded-wait check
namespace fp4 {

// Waits on an mbarrier that nothing ever arrives on; the bounded wait must
// give up after timeout_ns and raise FP4_DEV_WAIT_TIMEOUT.  Used by the
// failure-detection test: it exercises the timeout path without any fault.
__global__ void bounded_wait_probe_kernel(int* status, unsigned long long timeout_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, timeout_ns)) raise_status(status, kStatusTimeout);
}

cudaError_t launch_bounded_wait_probe(int* status, unsigned long long timeout_ns, cudaStream_t st) {
    bounded_wait_probe_kernel<<<1, 32, 0, st>>>(status, timeout_ns);
    return cudaGetLastError();
}

}  // namespace fp4
