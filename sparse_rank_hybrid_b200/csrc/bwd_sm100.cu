// Backward pass of the hybrid attention: gradients of sum(dO * out) with respect to q, k, v and the
// projection(s), the block selection held at the forward's (it is piecewise constant in q and k).  The
// formulas below are the default options' (relu features, RoPE outside the activation, one shared
// projection, plain sum); the feature maps and RoPE orderings go through lr_pair_fwd / lr_pair_bwd
// (common.cuh), separate and per-head projections through the A offsets and the dA reduction, and the
// gated fusion through gate_bwd.cu, which hands the two branches their own output gradients.
//
// Method: the derivative of the forward of RoLA "4.1" (block-sparse softmax attention over the kept
// key blocks plus the low-rank branch), "4.2"/"4.3" (truncated RoPE outside the relu feature map) and
// "B.1" (one query-independent summary per head); RoLA "4.5" and "E.1"/"E.2" train the branch's
// parameters jointly with the backbone, which needs these gradients.
//
// Sparse branch (per query row i over its allowed keys j; lse and O_s from the forward):
//   P_ij = 2^(s_ij log2(e)/sqrt(D) - lse_i),  Delta_i = dO_i . O_s,i,  dP_ij = dO_i . v_j,
//   dS_ij = P_ij (dP_ij - Delta_i),  dq^_i = sum_j dS_ij k^_j / sqrt(D),  dk^_j = sum_i dS_ij q^_i / sqrt(D),
//   dv_j = sum_i P_ij dO_i,  dq = R(p)^T dq^,  dk = R(p)^T dk^.
//   bwd_dq_kernel      one CTA per (query block, head): S = q^ k^T and dP = dO v^T per kept key block
//                      into TMEM, the math warps form dS (fp16) over dP's columns, dQ^ += dS k^ is
//                      accumulated in TMEM (tcgen05.mma kind::f16, operands fp16 in shared memory by TMA).
//   bwd_dkdv_kernel    one CTA per (key block, head), over the query blocks that kept it (inverted
//                      lists, ascending): S^T = k^ q^T and dP^T = v dO^T into TMEM, P^T and dS^T (fp16)
//                      over their columns, dV += P^T dO and dK^ += dS^T q^ accumulated in TMEM.  Each
//                      output row is owned by one CTA: no atomics, deterministic.
// Low-rank branch (u = x A, phi = relu(u), psi = R_r phi, den_i = phi_q,i . z + 1e-6):
//   G_i = S dO_i,  dpsi_q,i = G_i / den_i,  dden_i = -(psi_q,i . G_i) / den_i^2,
//   dphi_q,i = R_r^T dpsi_q,i + dden_i z,  dS = sum_i psi_q,i dO_i^T / den_i,  dz = sum_i dden_i phi_q,i,
//   dpsi_k,j = dS v_j,  dv_j += dS^T psi_k,j,  dphi_k,j = R_r^T dpsi_k,j + dz,
//   du = dphi * [u > 0],  dq += du_q A^T,  dk += du_k A^T,  dA = q^T du_q + k^T du_k.
//   lr_bwd_sm100_kernel (lr_bwd_sm100.cu)   the same on the tensor cores for head_dim 128, rank <= 64;
//   bwd_lr_q_kernel / bwd_lr_k_kernel   CUDA-core fp32 passes over token tiles for the other shapes
//                      (split-L partial sums of dS, dz and dA, summed in a fixed order).
//
// All waits are bounded (see sm100.cuh); a wait that runs out records a timeout in the status word and
// the CTA drains what it issued and returns.
#include "common.cuh"
#include "sm100.cuh"

namespace slra {

namespace {

// Warp roles of the dQ and dK/dV kernels for a block of BLK columns: NQ = BLK / 32 math warps per TMEM
// lane group, each owning 32 of the block's columns (and D / NQ columns of the output rows), then the
// tcgen05.mma issuing warp (lane 0) and a TMA producer warp.
template <int BLK>
struct BwdRoles {
    static constexpr int NQ = BLK / 32;
    static constexpr int kMathWarps = 4 * NQ;
    static constexpr int kMathThreads = 32 * kMathWarps;
    static constexpr int kIssueWarp = kMathWarps;
    static constexpr int kProdWarp = kMathWarps + 1;
    static constexpr int kThreads = kMathThreads + 64;
    static constexpr int HW = 32;  // block columns per math thread
};


__device__ __forceinline__ uint32_t pack_half2_lohi(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// TMEM column (32-bit) of the packed fp16 pair holding keys (columns) 2i, 2i+1 of a 16-key k-step kk,
// when each half of the threads writes its HW keys packed at the start of its own column range
// [h*HW, h*HW + HW/2): k-step kk covers keys [16kk, 16kk + 16) of half h = 16kk / HW.
template <int HW>
__device__ __forceinline__ uint32_t packed_col(int kk) {
    const int h = (16 * kk) / HW;
    return static_cast<uint32_t>(h * HW + (16 * kk - h * HW) / 2);
}

}  // namespace


// Bring this thread's DW columns of a gradient row towards L2 before the row is read back, so the
// read in the epilogue overlaps the last products instead of following them.
template <int DW>
__device__ __forceinline__ void prefetch_cols(const float* row_cols) {
#pragma unroll
    for (int o = 0; o < DW; o += 32)  // 128-byte lines
        asm volatile("prefetch.global.L2 [%0];" ::"l"(row_cols + o));
}

// This thread's DW consecutive TMEM columns of its lane from taddr (warp-collective loads), scaled.
template <int DW>
__device__ __forceinline__ void load_cols(uint32_t taddr, float* vals, float scale) {
    if constexpr (DW >= 32) {
#pragma unroll
        for (int c = 0; c < DW / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(taddr + c * 32, r);
            tmem_ld_wait(r);
#pragma unroll
            for (int i = 0; i < 32; ++i) vals[c * 32 + i] = __uint_as_float(r[i]) * scale;
        }
    } else {
        uint32_t r[16];
        tmem_ld16(taddr, r);
        tmem_ld_wait(r);
#pragma unroll
        for (int i = 0; i < 16; ++i) vals[i] = __uint_as_float(r[i]) * scale;
    }
}

// Rotate the pairs of this thread's DW columns [c0, c0 + DW) back by R(p)^T and store them (fp32) into a
// token-major row, or add them to it when a.accumulate (the row then holds the low-rank branch's part);
// `vals` are the 32-bit TMEM words of those columns, already scaled.
template <int DW>
__device__ __forceinline__ void store_row_unrotated(float* dst_row, const float* vals, int c0, int n,
                                                    const BwdArgs& a, const Geom& g, bool rotate) {
    float4 prev[DW / 4];
#pragma unroll
    for (int t = 0; t < DW / 4; ++t)
        prev[t] = a.accumulate ? *reinterpret_cast<const float4*>(dst_row + c0 + 4 * t)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
    const int pt = n / (g.H * g.W), ph = (n / g.W) % g.H, pw = n % g.W;
#pragma unroll
    for (int t = 0; t < DW / 4; ++t) {  // 4 columns (2 pairs) per float4
        float4 o;
        float* ov = reinterpret_cast<float*>(&o);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int c = 4 * t + 2 * u;  // column within this thread's range
            const int pair = (c0 + c) / 2;
            const float y0 = vals[c], y1 = vals[c + 1];
            if (rotate) {
                const int2 pi = a.pair_info[pair];
                const int pos = pi.x == 0 ? pt : (pi.x == 1 ? ph : pw);
                const double2 cs = __ldg(a.tab + pi.y + pos);
                const float cf = static_cast<float>(cs.x), sf = static_cast<float>(cs.y);
                ov[2 * u] = cf * y0 + sf * y1;       // R^T: rotate back by the pair's angle
                ov[2 * u + 1] = -sf * y0 + cf * y1;
            } else {
                ov[2 * u] = y0;
                ov[2 * u + 1] = y1;
            }
        }
        o.x += prev[t].x;
        o.y += prev[t].y;
        o.z += prev[t].z;
        o.w += prev[t].w;
        *reinterpret_cast<float4*>(dst_row + c0 + 4 * t) = o;
    }
}

// ------------------------------------------------------------------------------------------ dQ
// BwdRoles<BLK>: 4 * BLK / 32 math warps (rows = queries; each 32 key columns of a block), then the
// warp that issues the products and the warp that loads the tiles.
// TMEM (512 columns): S | dP buffer 0 | dP buffer 1 | dQ^.  Each math thread writes its packed dS_j over
// its own 32 of dP_j's columns (already in its registers), so the S columns are free as soon as the
// math warps have loaded S_j and dP_j: S_{j+1} and dP_{j+1} (into the other dP buffer) are computed
// while the math warps work on block j, and dQ^ += dS_j k^_j follows when they are done.  k^ tiles stay
// until their dQ product (three slots), v tiles until their dP product (two slots).
template <int D>
struct DqLayout {
    static constexpr int kTile = 128 * D * 2;  // fp16 [128 rows][D] in 64-column slabs
    static constexpr int kOffQ = 0;
    static constexpr int kOffDo = kTile;
    static constexpr int kOffK = 2 * kTile;  // slots s < 3 at kOffK + s * kTile
    static constexpr int kOffV = 5 * kTile;  // slots s < 2 at kOffV + s * kTile
    static constexpr int kOffBar = 7 * kTile;
    static constexpr int kOffMisc = kOffBar + 256;
    static constexpr int kBytes = kOffMisc + 64;
};

enum : int { kDqBarQdo = 0, kDqBarKFull = 1, kDqBarKEmpty = 4, kDqBarVFull = 7, kDqBarVEmpty = 9,
             kDqBarSp = 11, kDqBarLd = 12, kDqBarDs = 13 /* +2 */, kDqBarFinal = 15, kDqBarDrain = 16,
             kDqNumBars = 17 };

template <int D, int BLK>
__global__ void __launch_bounds__(BwdRoles<BLK>::kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, BwdArgs a,
                  Geom g) {
    using Lay = DqLayout<D>;
    using Roles = BwdRoles<BLK>;
    constexpr int HW = Roles::HW;  // key columns per math thread
    constexpr int NC = HW / 32;
    constexpr int DW = D / Roles::NQ;  // dQ columns per math thread in the epilogue
    constexpr int kSteps = D / 16, kKeySteps = BLK / 16;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kOffMisc + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int alpha = blockIdx.x, bh = blockIdx.y;
    const int b = bh / g.Hh, h = bh % g.Hh;
    const int keep = a.keep;
    const int32_t* my_idx = a.idx + (static_cast<size_t>(bh) * g.nb + alpha) * keep;
    const int row0 = bh * g.Lp;
    const uint64_t tmo = a.timeout_ns;

    if (tid == 0) {
        for (int i = 0; i < kDqNumBars; ++i)
            mbar_init(bars + i, (i == kDqBarLd || i == kDqBarDs || i == kDqBarDs + 1) ? Roles::kMathThreads : 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tQ = tmem + 384;
    auto tP = [&](int j) { return tmem + 128 + (j & 1) * 128; };
    auto fail = [&]() {
        *abort_flag = 1;
        atomicOr(a.status, kDevTimeout);
    };
    auto kslot = [&](int j) { return smem + Lay::kOffK + (j % 3) * Lay::kTile; };
    auto vslot = [&](int j) { return smem + Lay::kOffV + (j & 1) * Lay::kTile; };

    if (warp == Roles::kProdWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && keep > 0) {
            auto load_rows = [&](uint8_t* dst, const CUtensorMap* tm, uint64_t* bar, int row, int rows) {
#pragma unroll
                for (int sl = 0; sl < D / 64; ++sl) tma_load_2d(dst + sl * (rows * 128), tm, bar, sl * 64, row);
            };
            mbar_expect_tx(bars + kDqBarQdo, 2u * 128 * D * 2);
            load_rows(smem + Lay::kOffQ, &tm_q, bars + kDqBarQdo, row0 + alpha * BLK, 128);
            load_rows(smem + Lay::kOffDo, &tm_do, bars + kDqBarQdo, row0 + alpha * BLK, 128);
            int nk = 0, nv = 0;
            bool ok = true;
            for (int j = 0; j < keep && ok; ++j) {
                const int r = row0 + __ldg(my_idx + j) * BLK;
                // k^_j into slot j % 3 once dQ_{j-3} has read it; v_j into slot j % 2 once dP_{j-2} has
                if (j >= 3 && !mbar_wait(bars + kDqBarKEmpty + j % 3, ((j - 3) / 3) & 1, tmo, abort_flag)) {
                    ok = false;
                    break;
                }
                mbar_expect_tx(bars + kDqBarKFull + j % 3, static_cast<uint32_t>(BLK) * D * 2);
                load_rows(kslot(j), &tm_k, bars + kDqBarKFull + j % 3, r, BLK);
                ++nk;
                if (j >= 2 && !mbar_wait(bars + kDqBarVEmpty + (j & 1), ((j - 2) >> 1) & 1, tmo, abort_flag)) {
                    ok = false;
                    break;
                }
                mbar_expect_tx(bars + kDqBarVFull + (j & 1), static_cast<uint32_t>(BLK) * D * 2);
                load_rows(vslot(j), &tm_v, bars + kDqBarVFull + (j & 1), r, BLK);
                ++nv;
            }
            if (!ok) {
                fail();
                volatile int no_abort = 0;  // let every issued copy land (bounded)
                mbar_wait(bars + kDqBarQdo, 0, 10000000ull, &no_abort);
                for (int t = nk - 3 < 0 ? 0 : nk - 3; t < nk; ++t)
                    mbar_wait(bars + kDqBarKFull + t % 3, (t / 3) & 1, 10000000ull, &no_abort);
                for (int t = nv - 2 < 0 ? 0 : nv - 2; t < nv; ++t)
                    mbar_wait(bars + kDqBarVFull + (t & 1), (t >> 1) & 1, 10000000ull, &no_abort);
            }
        }
        __syncwarp();
    } else if (warp == Roles::kIssueWarp) {
        // ------------------------------------------------------------ tcgen05.mma issuer
        if (lane == 0 && keep > 0) {
            const uint32_t idesc_s = idesc_f16_f32(128, BLK, false, false);
            const uint32_t idesc_q = idesc_f16_f32(128, D, false, true);
            const uint32_t q_addr = smem_addr(smem + Lay::kOffQ), do_addr = smem_addr(smem + Lay::kOffDo);
            // S_j = q^ k^T_j and dP_j = dO v^T_j (K-major over the head dimension)
            auto issue_sp = [&](int j) -> bool {
                if (!mbar_wait(bars + kDqBarKFull + j % 3, (j / 3) & 1, tmo, abort_flag) ||
                    !mbar_wait(bars + kDqBarVFull + (j & 1), (j >> 1) & 1, tmo, abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t k_addr = smem_addr(kslot(j)), v_addr = smem_addr(vslot(j));
#pragma unroll
                for (int kk = 0; kk < kSteps; ++kk) {
                    const uint32_t ao = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
                    const uint32_t bo = (kk >> 2) * (BLK * 128) + (kk & 3) * 32;
                    umma_ss(tS, sdesc_sw128(q_addr + ao, 16, 1024), sdesc_sw128(k_addr + bo, 16, 1024), idesc_s,
                            kk > 0 ? 1u : 0u);
                    umma_ss(tP(j), sdesc_sw128(do_addr + ao, 16, 1024), sdesc_sw128(v_addr + bo, 16, 1024), idesc_s,
                            kk > 0 ? 1u : 0u);
                }
                umma_commit(bars + kDqBarVEmpty + (j & 1));
                umma_commit(bars + kDqBarSp);
                return true;
            };
            bool ok = mbar_wait(bars + kDqBarQdo, 0, tmo, abort_flag) && issue_sp(0);
            for (int j = 0; j < keep && ok; ++j) {
                // S_{j+1} and dP_{j+1} once the math warps hold S_j and dP_j in registers
                if (j + 1 < keep) {
                    if (!mbar_wait(bars + kDqBarLd, j & 1, tmo, abort_flag) || !issue_sp(j + 1)) {
                        ok = false;
                        break;
                    }
                }
                // dQ^ += dS_j k^_j: A = dS_j packed over dP_j's columns, B = k^_j MN-major
                if (!mbar_wait(bars + kDqBarDs + (j & 1), (j >> 1) & 1, tmo, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t k_addr = smem_addr(kslot(j));
#pragma unroll
                for (int kk = 0; kk < kKeySteps; ++kk)
                    umma_ts(tQ, tP(j) + packed_col<HW>(kk), sdesc_sw128(k_addr + kk * 2048, BLK * 128, 1024),
                            idesc_q, (j > 0 || kk > 0) ? 1u : 0u);
                umma_commit(bars + kDqBarKEmpty + j % 3);
            }
            if (ok) umma_commit(bars + kDqBarFinal);
            else fail();
            umma_commit(bars + kDqBarDrain);  // drain: every product issued here lands before the CTA leaves
            volatile int no_abort = 0;
            mbar_wait(bars + kDqBarDrain, 0, 10000000ull, &no_abort);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax-gradient warps
        const int lg = warp & 3, hf = warp >> 2;
        const int i_row = lg * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(lg * 32) << 16;
        const int n = alpha * BLK + i_row;
        const bool row_real = i_row < BLK && n < g.L;
        // rows that are not this block's (block 64: the tile's second half) or past L recompute as P = 0
        const float lse_i = row_real ? __ldg(a.lse + static_cast<size_t>(row0) + n) : INFINITY;
        const float delta_i = row_real ? __ldg(a.delta + static_cast<size_t>(row0) + n) : 0.f;
        const float c2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
        const int key0 = hf * HW;
        const int last_valid = keep > 0 ? min(BLK, g.L - __ldg(my_idx + keep - 1) * BLK) : BLK;
        bool ok = true;
        for (int j = 0; j < keep; ++j) {
            ok = __all_sync(0xffffffffu, mbar_wait(bars + kDqBarSp, j & 1, tmo, abort_flag));
            if (!ok) {
                if (lane == 0) fail();
                break;
            }
            tc_fence_after();
            uint32_t sr[NC][32], pr[NC][32];
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                tmem_ld32(tS + lane_base + key0 + c * 32, sr[c]);
                tmem_ld32(tP(j) + lane_base + key0 + c * 32, pr[c]);
            }
            tmem_ld_wait(sr[0]);
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                reg_fence(sr[c]);
                reg_fence(pr[c]);
            }
            tc_fence_before();
            mbar_arrive(bars + kDqBarLd);  // S_j and dP_j are in registers: S may be overwritten
            const bool masked = (j == keep - 1) && last_valid < BLK;
#pragma unroll
            for (int c16 = 0; c16 < HW / 32; ++c16) {
                uint32_t pk[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    float d2[2];
#pragma unroll
                    for (int e2 = 0; e2 < 2; ++e2) {
                        const int e = c16 * 32 + 2 * u + e2;  // key within this half
                        const float sv = __uint_as_float(sr[e >> 5][e & 31]);
                        const float dp = __uint_as_float(pr[e >> 5][e & 31]);
                        float p = ex2_approx(fmaf(sv, c2, -lse_i));
                        if (masked && key0 + e >= last_valid) p = 0.f;
                        d2[e2] = p * (dp - delta_i);
                    }
                    pk[u] = pack_half2_lohi(d2[0], d2[1]);
                }
                tmem_st16(tP(j) + lane_base + key0 + c16 * 16, pk);  // packed over this half's dP columns
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(bars + kDqBarDs + (j & 1));
        }
        // ---- epilogue: dq += R(p)^T dQ^ / sqrt(D), token-major fp32
        if (keep > 0) {
            if (ok && row_real && a.accumulate) prefetch_cols<DW>(a.dq + g.so.row(b, n, h) + hf * DW);
            const bool done = ok && __all_sync(0xffffffffu, mbar_wait(bars + kDqBarFinal, 0, tmo, abort_flag));
            if (done) {
                tc_fence_after();
                float vals[DW];
                const float inv_sqrt_d = 1.f / sqrtf(static_cast<float>(D));
                load_cols<DW>(tQ + lane_base + hf * DW, vals, inv_sqrt_d);
                if (row_real)
                    store_row_unrotated<DW>(a.dq + g.so.row(b, n, h), vals, hf * DW, n, a, g, true);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------------------- dK, dV
// BwdRoles<BLK> math warps (rows = keys; each 32 query columns of a block), then the warp that issues
// the products and the warp that loads the query-side tiles.
// TMEM: S^T | dP^T | dV | dK^.  Each math thread writes its packed P^T and dS^T over its own 32 of
// dP^T's columns (P^T in the first quarter of the block's columns, dS^T in the second), so the S^T
// columns are free once S^T_t and dP^T_t are in registers and S^T_{t+1} is computed during the math of
// block t; dP^T_{t+1} follows the dV and dK products that read block t's packed operands.
template <int D, int BLK>
struct DkvLayout {
    static constexpr int kTile = 128 * D * 2;   // key-side tiles: 128 rows (the MMA's M)
    static constexpr int kQTile = BLK * D * 2;  // query-side tiles: one query block
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kTile;
    static constexpr int kOffQ = 2 * kTile;               // slots s at kOffQ + s * kQTile
    static constexpr int kOffDo = kOffQ + 2 * kQTile;     // slots s at kOffDo + s * kQTile
    static constexpr int kOffLse = kOffDo + 2 * kQTile;   // slots s: [BLK] fp32 lse then [BLK] fp32 delta
    static constexpr int kOffBar = kOffLse + 2 * 2 * BLK * 4;
    static constexpr int kOffMisc = kOffBar + 256;
    static constexpr int kBytes = kOffMisc + 64;
};

enum : int { kKvBarKv = 0, kKvBarQFull = 1, kKvBarQEmpty = 3, kKvBarS = 5, kKvBarP = 6, kKvBarLd = 7,
             kKvBarDs = 8 /* +2 */, kKvBarFinal = 10, kKvBarDrain = 11, kKvNumBars = 12 };

template <int D, int BLK>
__global__ void __launch_bounds__(BwdRoles<BLK>::kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do, BwdArgs a,
                    Geom g) {
    using Lay = DkvLayout<D, BLK>;
    using Roles = BwdRoles<BLK>;
    constexpr int HW = Roles::HW;  // query columns per math thread
    constexpr int NC = HW / 32;
    constexpr int DW = D / Roles::NQ;  // dK, dV columns per math thread in the epilogue
    constexpr int kSteps = D / 16, kQSteps = BLK / 16;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kOffMisc + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int beta = blockIdx.x, bh = blockIdx.y;
    const int b = bh / g.Hh, h = bh % g.Hh;
    const int row0 = bh * g.Lp;
    const int cnt = __ldg(a.inv_cnt + static_cast<size_t>(bh) * g.nb + beta);
    const int32_t* my_inv = a.inv + (static_cast<size_t>(bh) * g.nb + beta) * g.nb;
    const uint64_t tmo = a.timeout_ns;

    if (tid == 0) {
        for (int i = 0; i < kKvNumBars; ++i)
            mbar_init(bars + i, (i == kKvBarLd || i == kKvBarDs || i == kKvBarDs + 1) ? Roles::kMathThreads : 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tP = tmem + 128, tV = tmem + 256, tK = tmem + 384;
    auto fail = [&]() {
        *abort_flag = 1;
        atomicOr(a.status, kDevTimeout);
    };
    auto qslot = [&](int s) { return smem + Lay::kOffQ + s * Lay::kQTile; };
    auto doslot = [&](int s) { return smem + Lay::kOffDo + s * Lay::kQTile; };
    auto lseslot = [&](int s) { return reinterpret_cast<float*>(smem + Lay::kOffLse + s * 2 * BLK * 4); };

    if (warp == Roles::kProdWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && cnt > 0) {
            auto load_rows = [&](uint8_t* dst, const CUtensorMap* tm, uint64_t* bar, int row, int rows) {
#pragma unroll
                for (int sl = 0; sl < D / 64; ++sl) tma_load_2d(dst + sl * (rows * 128), tm, bar, sl * 64, row);
            };
            mbar_expect_tx(bars + kKvBarKv, 2u * 128 * D * 2);
            load_rows(smem + Lay::kOffK, &tm_k, bars + kKvBarKv, row0 + beta * BLK, 128);
            load_rows(smem + Lay::kOffV, &tm_v, bars + kKvBarKv, row0 + beta * BLK, 128);
            int nq = 0;
            bool ok = true;
            for (int t = 0; t < cnt; ++t) {
                const int s = t & 1;
                // slot s once the dV and dK products of block t-2 (its last readers) have completed
                if (t >= 2 && !mbar_wait(bars + kKvBarQEmpty + s, ((t - 2) >> 1) & 1, tmo, abort_flag)) {
                    ok = false;
                    break;
                }
                uint64_t* bar = bars + kKvBarQFull + s;
                mbar_expect_tx(bar, 2u * BLK * D * 2 + 2u * BLK * 4);
                const int qb = __ldg(my_inv + t);
                load_rows(qslot(s), &tm_q, bar, row0 + qb * BLK, BLK);
                load_rows(doslot(s), &tm_do, bar, row0 + qb * BLK, BLK);
                bulk_load(lseslot(s), a.lse + static_cast<size_t>(row0) + qb * BLK, BLK * 4, bar);
                bulk_load(lseslot(s) + BLK, a.delta + static_cast<size_t>(row0) + qb * BLK, BLK * 4, bar);
                ++nq;
            }
            if (!ok) {
                fail();
                volatile int no_abort = 0;
                mbar_wait(bars + kKvBarKv, 0, 10000000ull, &no_abort);
                for (int t = nq - 2 < 0 ? 0 : nq - 2; t < nq; ++t)
                    mbar_wait(bars + kKvBarQFull + (t & 1), (t >> 1) & 1, 10000000ull, &no_abort);
            }
        }
        __syncwarp();
    } else if (warp == Roles::kIssueWarp) {
        // ------------------------------------------------------------ tcgen05.mma issuer
        if (lane == 0 && cnt > 0) {
            const uint32_t idesc_s = idesc_f16_f32(128, BLK, false, false);
            const uint32_t idesc_o = idesc_f16_f32(128, D, false, true);
            const uint32_t k_addr = smem_addr(smem + Lay::kOffK), v_addr = smem_addr(smem + Lay::kOffV);
            auto issue_s = [&](int t) {  // S^T_t = k^ q^T_t
                const uint32_t q_addr = smem_addr(qslot(t & 1));
#pragma unroll
                for (int kk = 0; kk < kSteps; ++kk)
                    umma_ss(tS, sdesc_sw128(k_addr + (kk >> 2) * (128 * 128) + (kk & 3) * 32, 16, 1024),
                            sdesc_sw128(q_addr + (kk >> 2) * (BLK * 128) + (kk & 3) * 32, 16, 1024), idesc_s,
                            kk > 0 ? 1u : 0u);
                umma_commit(bars + kKvBarS);
            };
            auto issue_p = [&](int t) {  // dP^T_t = v dO^T_t
                const uint32_t do_addr = smem_addr(doslot(t & 1));
#pragma unroll
                for (int kk = 0; kk < kSteps; ++kk)
                    umma_ss(tP, sdesc_sw128(v_addr + (kk >> 2) * (128 * 128) + (kk & 3) * 32, 16, 1024),
                            sdesc_sw128(do_addr + (kk >> 2) * (BLK * 128) + (kk & 3) * 32, 16, 1024), idesc_s,
                            kk > 0 ? 1u : 0u);
                umma_commit(bars + kKvBarP);
            };
            bool ok = mbar_wait(bars + kKvBarKv, 0, tmo, abort_flag) && mbar_wait(bars + kKvBarQFull, 0, tmo, abort_flag);
            if (ok) {
                tc_fence_after();
                issue_s(0);
                issue_p(0);
            }
            for (int t = 0; t < cnt && ok; ++t) {
                const int s = t & 1;
                // S^T_{t+1} once the math warps hold S^T_t and dP^T_t in registers
                if (t + 1 < cnt) {
                    if (!mbar_wait(bars + kKvBarLd, t & 1, tmo, abort_flag) ||
                        !mbar_wait(bars + kKvBarQFull + ((t + 1) & 1), ((t + 1) >> 1) & 1, tmo, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_s(t + 1);
                }
                if (!mbar_wait(bars + kKvBarDs + s, (t >> 1) & 1, tmo, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // dV += P^T dO_t and dK^ += dS^T q^_t (A packed over dP^T's columns, B MN-major)
                const uint32_t q_addr = smem_addr(qslot(s)), do_addr = smem_addr(doslot(s));
#pragma unroll
                for (int kk = 0; kk < kQSteps; ++kk) {
                    const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
                    const uint32_t col = packed_col<HW>(kk);
                    umma_ts(tV, tP + col, sdesc_sw128(do_addr + kk * 2048, BLK * 128, 1024), idesc_o, acc);
                    umma_ts(tK, tP + col + HW / 2, sdesc_sw128(q_addr + kk * 2048, BLK * 128, 1024), idesc_o, acc);
                }
                umma_commit(bars + kKvBarQEmpty + s);
                if (t + 1 < cnt) issue_p(t + 1);  // after the products that read dP^T's columns
            }
            if (ok) umma_commit(bars + kKvBarFinal);
            else fail();
            umma_commit(bars + kKvBarDrain);
            volatile int no_abort = 0;
            mbar_wait(bars + kKvBarDrain, 0, 10000000ull, &no_abort);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax-gradient warps (rows = keys)
        const int lg = warp & 3, hf = warp >> 2;
        const int j_row = lg * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(lg * 32) << 16;
        const int n = beta * BLK + j_row;
        const bool row_real = j_row < BLK && n < g.L;
        const float c2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
        const int q0 = hf * HW;  // first query column of this thread's half
        bool ok = true;
        for (int t = 0; t < cnt; ++t) {
            const int s = t & 1;
            // the query block's lse and delta arrived with its tiles (same barrier phase)
            ok = __all_sync(0xffffffffu, mbar_wait(bars + kKvBarQFull + s, (t >> 1) & 1, tmo, abort_flag) &&
                                             mbar_wait(bars + kKvBarS, t & 1, tmo, abort_flag) &&
                                             mbar_wait(bars + kKvBarP, t & 1, tmo, abort_flag));
            if (!ok) {
                if (lane == 0) fail();
                break;
            }
            tc_fence_after();
            const float* lse_s = lseslot(s);
            const float* del_s = lse_s + BLK;
            uint32_t sr[NC][32], pr[NC][32];
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                tmem_ld32(tS + lane_base + q0 + c * 32, sr[c]);
                tmem_ld32(tP + lane_base + q0 + c * 32, pr[c]);
            }
            tmem_ld_wait(sr[0]);
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                reg_fence(sr[c]);
                reg_fence(pr[c]);
            }
            tc_fence_before();
            mbar_arrive(bars + kKvBarLd);  // S^T_t and dP^T_t are in registers: S^T may be overwritten
#pragma unroll
            for (int c16 = 0; c16 < HW / 32; ++c16) {
                uint32_t pk[16], dk16[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    float pp[2], dd[2];
#pragma unroll
                    for (int e2 = 0; e2 < 2; ++e2) {
                        const int e = c16 * 32 + 2 * u + e2;  // query column within this half
                        const float sv = __uint_as_float(sr[e >> 5][e & 31]);
                        const float dp = __uint_as_float(pr[e >> 5][e & 31]);
                        const float p = ex2_approx(fmaf(sv, c2, -lse_s[q0 + e]));  // +inf lse: p = 0
                        pp[e2] = p;
                        dd[e2] = p * (dp - del_s[q0 + e]);
                    }
                    pk[u] = pack_half2_lohi(pp[0], pp[1]);
                    dk16[u] = pack_half2_lohi(dd[0], dd[1]);
                }
                tmem_st16(tP + lane_base + q0 + c16 * 16, pk);            // P^T: first quarter of the half
                tmem_st16(tP + lane_base + q0 + HW / 2 + c16 * 16, dk16);  // dS^T: second quarter
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(bars + kKvBarDs + s);
        }
        // ---- epilogue: dv += sum P^T dO, dk += R(p)^T dK^ / sqrt(D); key blocks nobody kept add zeros
        if (ok && row_real && a.accumulate) {
            prefetch_cols<DW>(a.dv + g.so.row(b, n, h) + hf * DW);
            prefetch_cols<DW>(a.dk + g.so.row(b, n, h) + hf * DW);
        }
        const bool done = cnt == 0 || (ok && __all_sync(0xffffffffu, mbar_wait(bars + kKvBarFinal, 0, tmo, abort_flag)));
        if (done) {
            if (cnt > 0) tc_fence_after();
            const float inv_sqrt_d = 1.f / sqrtf(static_cast<float>(D));
            float vals[DW];
#pragma unroll
            for (int which = 0; which < 2; ++which) {  // 0: dv, 1: dk
                if (cnt > 0) {  // uniform over the CTA: the loads are warp-collective
                    load_cols<DW>((which ? tK : tV) + lane_base + hf * DW, vals, which ? inv_sqrt_d : 1.f);
                } else {
#pragma unroll
                    for (int i = 0; i < DW; ++i) vals[i] = 0.f;
                }
                if (row_real)
                    store_row_unrotated<DW>((which ? a.dk : a.dv) + g.so.row(b, n, h), vals, hf * DW, n, a, g,
                                            which == 1);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------------------------ preparation
// dO (fp32, token-major) -> fp16 head-major copy for the tensor cores (rows past L zero), and
// Delta_i = dO_i . O_s,i (O_s head-major fp32 from the recomputed sparse forward).  One warp per row.
__global__ void bwd_prep_kernel(const float* __restrict__ dout, const float* __restrict__ os, Geom g,
                                __half* __restrict__ doh, float* __restrict__ delta, int* status) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    const long long rows = static_cast<long long>(g.BH()) * g.Lp;
    if (warp >= rows) return;
    const int bh = static_cast<int>(warp / g.Lp), n = static_cast<int>(warp % g.Lp);
    const int b = bh / g.Hh, h = bh % g.Hh;
    const int per = g.D / 32;  // elements per lane: 2 or 4
    float dsum = 0.f;
    bool bad = false;
    __half* dst = doh + static_cast<size_t>(warp) * g.D + lane * per;
    if (n < g.L) {
        const float* src = dout + g.so.row(b, n, h) + lane * per;
        const float* o = os + static_cast<size_t>(warp) * g.D + lane * per;
        for (int e = 0; e < per; e += 2) {
            const float2 x = *reinterpret_cast<const float2*>(src + e);
            const float2 y = *reinterpret_cast<const float2*>(o + e);
            dsum = fmaf(x.x, y.x, fmaf(x.y, y.y, dsum));
            bad |= !(fmaxf(fabsf(x.x), fabsf(x.y)) < 65504.f);
            *reinterpret_cast<__half2*>(dst + e) = __floats2half2_rn(x.x, x.y);
        }
    } else {
        for (int e = 0; e < per; e += 2) *reinterpret_cast<__half2*>(dst + e) = __floats2half2_rn(0.f, 0.f);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
    if (lane == 0) delta[warp] = dsum;
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(status, kDevRange);
}

// Inverted kept-block lists: for key block beta of head bh, the query blocks whose kept list holds
// it, ascending (one CTA of 128 threads per (beta, bh); each thread tests query blocks by binary search
// in their ascending kept lists; an ordered compaction writes them).
__global__ void bwd_invert_kernel(const int32_t* __restrict__ idx, Geom g, int32_t* __restrict__ inv,
                                  int32_t* __restrict__ inv_cnt) {
    __shared__ int warp_tot[4];
    const int beta = blockIdx.x, bh = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int32_t* ib = idx + static_cast<size_t>(bh) * g.nb * g.keep;
    int32_t* out = inv + (static_cast<size_t>(bh) * g.nb + beta) * g.nb;
    int written = 0;
    for (int base = 0; base < g.nb; base += 128) {
        const int al = base + tid;
        bool hit = false;
        if (al < g.nb) {
            const int32_t* row = ib + static_cast<size_t>(al) * g.keep;
            int lo = 0, hi = g.keep - 1;
            while (lo <= hi) {
                const int mid = (lo + hi) >> 1;
                const int x = __ldg(row + mid);
                if (x == beta) { hit = true; break; }
                if (x < beta) lo = mid + 1;
                else hi = mid - 1;
            }
        }
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        if (lane == 0) warp_tot[warp] = __popc(m);
        __syncthreads();
        int before = written;
        for (int w = 0; w < warp; ++w) before += warp_tot[w];
        if (hit) out[before + __popc(m & ((1u << lane) - 1u))] = al;
        written += warp_tot[0] + warp_tot[1] + warp_tot[2] + warp_tot[3];
        __syncthreads();
    }
    if (tid == 0) inv_cnt[static_cast<size_t>(bh) * g.nb + beta] = written;
}

// ------------------------------------------------------------------------------------ low-rank
// Token tile of the CUDA-core passes: 32 tokens (16 when rank > 64, so shared memory fits).
template <int R>
struct LrTile {
    static constexpr int T = R <= 64 ? 32 : 16;
};

// Pass over the queries: per token u = q A, psi and the normaliser feature nf (lr_pair_fwd), den = nf . z,
// G = S dO; dpsi = G / den, dden, du (lr_pair_bwd); split-L partial sums of dS = sum psi dO^T / den,
// dz = sum dden nf and dA_q = q^T du; dq += du A^T.  A: this pass's projection (head h at h * a_stride).
template <int D, int R>
__global__ void __launch_bounds__(256) bwd_lr_q_kernel(const __nv_bfloat16* __restrict__ q,
                                                       const float* __restrict__ dout,
                                                       const __nv_bfloat16* __restrict__ A,
                                                       const float* __restrict__ S, const float* __restrict__ z,
                                                       const double2* __restrict__ tab,
                                                       const int2* __restrict__ pairs, Geom g, int nsplit,
                                                       float* __restrict__ dq, float* __restrict__ ds_part,
                                                       float* __restrict__ dz_part, float* __restrict__ da_part,
                                                       int accumulate) {
    constexpr int TT = LrTile<R>::T;
    extern __shared__ __align__(16) float smf[];
    // A and S padded by one column: the loops below read them with consecutive lanes walking either
    // index, and the padding keeps both walks free of shared-memory bank conflicts
    float* As = smf;                    // [D][R+1]
    float* Ss = As + D * (R + 1);       // [R][D+1]
    float* zs = Ss + R * (D + 1);       // [R]
    float* xs = zs + R;                 // [TT][D+1] q
    float* gs = xs + TT * (D + 1);      // [TT][D+1] dO
    float* us = gs + TT * (D + 1);      // [TT][R+1] u
    float* Gs = us + TT * (R + 1);      // [TT][R+1] G = S dO
    float* ws = Gs + TT * (R + 1);      // [TT][R] psi / den
    float* dus = ws + TT * R;           // [TT][R+1] du
    float* phs = dus + TT * (R + 1);    // [TT][R] phi
    float* dens = phs + TT * R;         // [TT] den
    float* ddens = dens + TT;           // [TT] dden
    constexpr int G = 256 / D;          // row groups of the D-wide accumulations
    constexpr int NA = R / G;
    const int tid = threadIdx.x;
    const int split = blockIdx.x, bh = blockIdx.y;
    const int b = bh / g.Hh, h = bh % g.Hh;
    const int ntiles = (g.L + TT - 1) / TT;
    const int per = (ntiles + nsplit - 1) / nsplit;
    const int t0 = split * per, t1 = min(ntiles, t0 + per);
    const __nv_bfloat16* Ah = A + static_cast<size_t>(h) * g.a_stride;
    for (int e = tid; e < D * R; e += 256) As[(e / R) * (R + 1) + e % R] = __bfloat162float(Ah[e]);
    for (int e = tid; e < R * D; e += 256) Ss[(e / D) * (D + 1) + e % D] = S[static_cast<size_t>(bh) * R * D + e];
    if (tid < R) zs[tid] = z[static_cast<size_t>(bh) * R + tid];
    // (cos, sin) of pair p at token n; no rotation without the low-rank RoPE
    auto rot = [&](int p, int n, float& cf, float& sf) {
        if (g.norope) {
            cf = 1.f;
            sf = 0.f;
            return;
        }
        const int2 pi = pairs[p];
        const double2 cs = tab[pi.y + token_axis_pos(n, pi.x, g.H, g.W)];
        cf = static_cast<float>(cs.x);
        sf = static_cast<float>(cs.y);
    };
    const int e_own = tid % D, cg = tid / D;
    float acc_s[NA], acc_a[NA];  // dS[c][e_own], dA[e_own][c] for c = cg + G i
#pragma unroll
    for (int i = 0; i < NA; ++i) acc_s[i] = acc_a[i] = 0.f;
    float acc_z = 0.f;
    for (int tile = t0; tile < t1; ++tile) {
        const int n0 = tile * TT;
        __syncthreads();
        for (int e = tid; e < TT * (D / 2); e += 256) {
            const int tt = e / (D / 2), dp = e % (D / 2);
            const int n = n0 + tt;
            float2 xf = make_float2(0.f, 0.f), gf = make_float2(0.f, 0.f);
            if (n < g.L) {
                xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(q + g.sq.row(b, n, h) + 2 * dp));
                gf = *reinterpret_cast<const float2*>(dout + g.so.row(b, n, h) + 2 * dp);
            }
            xs[tt * (D + 1) + 2 * dp] = xf.x; xs[tt * (D + 1) + 2 * dp + 1] = xf.y;
            gs[tt * (D + 1) + 2 * dp] = gf.x; gs[tt * (D + 1) + 2 * dp + 1] = gf.y;
        }
        __syncthreads();
        // u = q A and G = S dO, thread per (token, feature)
        for (int o = tid; o < TT * R; o += 256) {
            const int tt = o / R, c = o % R;
            const float* xr = xs + tt * (D + 1);
            const float* gr = gs + tt * (D + 1);
            float u = 0.f, gg = 0.f;
#pragma unroll 8
            for (int d = 0; d < D; ++d) {
                u = fmaf(xr[d], As[d * (R + 1) + c], u);
                gg = fmaf(Ss[c * (D + 1) + d], gr[d], gg);
            }
            us[tt * (R + 1) + c] = u;
            Gs[tt * (R + 1) + c] = gg;
        }
        __syncthreads();
        // per token: den = nf . z + 1e-6, dden = -(psi . G) / den^2 (one warp per token); nf kept for dz
        {
            const int warp = tid >> 5, lane = tid & 31;
            for (int tt = warp; tt < TT; tt += 8) {
                const int n = n0 + tt;
                const int nt = n < g.L ? n : 0;
                float dz_ = 0.f, dot = 0.f;
                for (int p = lane; p < R / 2; p += 32) {
                    float cf, sf;
                    rot(p, nt, cf, sf);
                    const LrPair P = lr_pair_fwd(us[tt * (R + 1) + 2 * p], us[tt * (R + 1) + 2 * p + 1], cf, sf,
                                                 g.act, g.inside);
                    phs[tt * R + 2 * p] = P.nf0;
                    phs[tt * R + 2 * p + 1] = P.nf1;
                    dz_ = fmaf(P.nf0, zs[2 * p], fmaf(P.nf1, zs[2 * p + 1], dz_));
                    dot = fmaf(P.psi0, Gs[tt * (R + 1) + 2 * p], fmaf(P.psi1, Gs[tt * (R + 1) + 2 * p + 1], dot));
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    dz_ += __shfl_xor_sync(0xffffffffu, dz_, o);
                    dot += __shfl_xor_sync(0xffffffffu, dot, o);
                }
                if (lane == 0) {
                    const float den = dz_ + 1e-6f;
                    dens[tt] = den;
                    ddens[tt] = n < g.L ? -dot / (den * den) : 0.f;
                }
            }
        }
        __syncthreads();
        // per (token, pair): psi / den; du from dpsi = G / den and dnf = dden z
        for (int o = tid; o < TT * (R / 2); o += 256) {
            const int tt = o / (R / 2), p = o % (R / 2);
            const int n = n0 + tt;
            const int nt = n < g.L ? n : 0;
            float cf, sf;
            rot(p, nt, cf, sf);
            const float den = dens[tt], dd = ddens[tt];
            const LrPair P = lr_pair_fwd(us[tt * (R + 1) + 2 * p], us[tt * (R + 1) + 2 * p + 1], cf, sf, g.act,
                                         g.inside);
            ws[tt * R + 2 * p] = n < g.L ? P.psi0 / den : 0.f;
            ws[tt * R + 2 * p + 1] = n < g.L ? P.psi1 / den : 0.f;
            const float g0 = Gs[tt * (R + 1) + 2 * p] / den, g1 = Gs[tt * (R + 1) + 2 * p + 1] / den;
            float du0, du1;
            lr_pair_bwd(P, g0, g1, dd * zs[2 * p], dd * zs[2 * p + 1], cf, sf, g.inside, du0, du1);
            const bool live = n < g.L;
            dus[tt * (R + 1) + 2 * p] = live ? du0 : 0.f;
            dus[tt * (R + 1) + 2 * p + 1] = live ? du1 : 0.f;
        }
        __syncthreads();
        // partial sums: dS[c][e] += sum_t w[t][c] dO[t][e]; dA[d][c] += sum_t q[t][d] du[t][c]; dz
#pragma unroll 4
        for (int tt = 0; tt < TT; ++tt) {
            const float go = gs[tt * (D + 1) + e_own], xo = xs[tt * (D + 1) + e_own];
#pragma unroll
            for (int i = 0; i < NA; ++i) {
                acc_s[i] = fmaf(ws[tt * R + cg + G * i], go, acc_s[i]);
                acc_a[i] = fmaf(xo, dus[tt * (R + 1) + cg + G * i], acc_a[i]);
            }
        }
        if (tid < R)
            for (int tt = 0; tt < TT; ++tt) acc_z = fmaf(ddens[tt], phs[tt * R + tid], acc_z);
        // dq += du A^T, thread per (token, dim)
        for (int o = tid; o < TT * D; o += 256) {
            const int tt = o / D, d = o % D;
            const int n = n0 + tt;
            if (n >= g.L) continue;
            float s = 0.f;
#pragma unroll 8
            for (int c = 0; c < R; ++c) s = fmaf(dus[tt * (R + 1) + c], As[d * (R + 1) + c], s);
            float* dst = dq + g.so.row(b, n, h) + d;
            *dst = accumulate ? *dst + s : s;
        }
    }
    const size_t slot = static_cast<size_t>(bh) * nsplit + split;
#pragma unroll
    for (int i = 0; i < NA; ++i) {
        ds_part[slot * R * D + (cg + G * i) * D + e_own] = acc_s[i];
        da_part[slot * D * R + e_own * R + cg + G * i] = acc_a[i];
    }
    if (tid < R) dz_part[slot * R + tid] = acc_z;
}

// Pass over the keys: per token u = k A, psi (lr_pair_fwd); dpsi = dS v; dv += dS^T psi; du from dpsi and
// dnf = dz (lr_pair_bwd); dk += du A^T; split-L partial sums of dA_k = k^T du.  A: the key projection.
template <int D, int R>
__global__ void __launch_bounds__(256) bwd_lr_k_kernel(const __nv_bfloat16* __restrict__ k,
                                                       const __nv_bfloat16* __restrict__ v,
                                                       const __nv_bfloat16* __restrict__ A,
                                                       const float* __restrict__ dS, const float* __restrict__ dz,
                                                       const double2* __restrict__ tab,
                                                       const int2* __restrict__ pairs, Geom g, int nsplit,
                                                       float* __restrict__ dk, float* __restrict__ dv,
                                                       float* __restrict__ da_part, int accumulate) {
    constexpr int TT = LrTile<R>::T;
    extern __shared__ __align__(16) float smf[];
    float* As = smf;                    // [D][R+1] (padded as in the query pass)
    float* Ss = As + D * (R + 1);       // [R][D+1] dS
    float* zs = Ss + R * (D + 1);       // [R] dz
    float* xs = zs + R;                 // [TT][D+1] k
    float* vs = xs + TT * (D + 1);      // [TT][D+1] v
    float* us = vs + TT * (D + 1);      // [TT][R+1] u
    float* ps = us + TT * (R + 1);      // [TT][R+1] dpsi, then du
    float* psis = ps + TT * (R + 1);    // [TT][R+1] psi
    constexpr int G = 256 / D;
    constexpr int NA = R / G;
    const int tid = threadIdx.x;
    const int split = blockIdx.x, bh = blockIdx.y;
    const int b = bh / g.Hh, h = bh % g.Hh;
    const int ntiles = (g.L + TT - 1) / TT;
    const int per = (ntiles + nsplit - 1) / nsplit;
    const int t0 = split * per, t1 = min(ntiles, t0 + per);
    const __nv_bfloat16* Ah = A + static_cast<size_t>(h) * g.a_stride;
    for (int e = tid; e < D * R; e += 256) As[(e / R) * (R + 1) + e % R] = __bfloat162float(Ah[e]);
    for (int e = tid; e < R * D; e += 256) Ss[(e / D) * (D + 1) + e % D] = dS[static_cast<size_t>(bh) * R * D + e];
    if (tid < R) zs[tid] = dz[static_cast<size_t>(bh) * R + tid];
    const int e_own = tid % D, cg = tid / D;
    float acc_a[NA];
#pragma unroll
    for (int i = 0; i < NA; ++i) acc_a[i] = 0.f;
    for (int tile = t0; tile < t1; ++tile) {
        const int n0 = tile * TT;
        __syncthreads();
        for (int e = tid; e < TT * (D / 2); e += 256) {
            const int tt = e / (D / 2), dp = e % (D / 2);
            const int n = n0 + tt;
            float2 xf = make_float2(0.f, 0.f), vf = make_float2(0.f, 0.f);
            if (n < g.L) {
                xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(k + g.sk.row(b, n, h) + 2 * dp));
                vf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(v + g.sv.row(b, n, h) + 2 * dp));
            }
            xs[tt * (D + 1) + 2 * dp] = xf.x; xs[tt * (D + 1) + 2 * dp + 1] = xf.y;
            vs[tt * (D + 1) + 2 * dp] = vf.x; vs[tt * (D + 1) + 2 * dp + 1] = vf.y;
        }
        __syncthreads();
        // u = k A and dpsi = dS v, thread per (token, feature)
        for (int o = tid; o < TT * R; o += 256) {
            const int tt = o / R, c = o % R;
            const float* xr = xs + tt * (D + 1);
            const float* vr = vs + tt * (D + 1);
            float u = 0.f, dp = 0.f;
#pragma unroll 8
            for (int d = 0; d < D; ++d) {
                u = fmaf(xr[d], As[d * (R + 1) + c], u);
                dp = fmaf(Ss[c * (D + 1) + d], vr[d], dp);
            }
            us[tt * (R + 1) + c] = u;
            ps[tt * (R + 1) + c] = dp;
        }
        __syncthreads();
        // per (token, pair): psi; du from dpsi and dnf = dz (written over dpsi)
        for (int o = tid; o < TT * (R / 2); o += 256) {
            const int tt = o / (R / 2), p = o % (R / 2);
            const int n = n0 + tt;
            const int nt = n < g.L ? n : 0;
            float cf = 1.f, sf = 0.f;
            if (!g.norope) {
                const int2 pi = pairs[p];
                const double2 cs = tab[pi.y + token_axis_pos(nt, pi.x, g.H, g.W)];
                cf = static_cast<float>(cs.x);
                sf = static_cast<float>(cs.y);
            }
            const LrPair P = lr_pair_fwd(us[tt * (R + 1) + 2 * p], us[tt * (R + 1) + 2 * p + 1], cf, sf, g.act,
                                         g.inside);
            psis[tt * (R + 1) + 2 * p] = P.psi0;
            psis[tt * (R + 1) + 2 * p + 1] = P.psi1;
            float du0, du1;
            lr_pair_bwd(P, ps[tt * (R + 1) + 2 * p], ps[tt * (R + 1) + 2 * p + 1], zs[2 * p], zs[2 * p + 1], cf, sf,
                        g.inside, du0, du1);
            const bool live = n < g.L;
            ps[tt * (R + 1) + 2 * p] = live ? du0 : 0.f;
            ps[tt * (R + 1) + 2 * p + 1] = live ? du1 : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int tt = 0; tt < TT; ++tt) {
            const float xo = xs[tt * (D + 1) + e_own];
#pragma unroll
            for (int i = 0; i < NA; ++i) acc_a[i] = fmaf(xo, ps[tt * (R + 1) + cg + G * i], acc_a[i]);
        }
        // dv += dS^T psi and dk += du A^T, thread per (token, dim)
        for (int o = tid; o < TT * D; o += 256) {
            const int tt = o / D, d = o % D;
            const int n = n0 + tt;
            if (n >= g.L) continue;
            float sv = 0.f, sk = 0.f;
#pragma unroll 8
            for (int c = 0; c < R; ++c) {
                sv = fmaf(Ss[c * (D + 1) + d], psis[tt * (R + 1) + c], sv);
                sk = fmaf(ps[tt * (R + 1) + c], As[d * (R + 1) + c], sk);
            }
            const long long r = g.so.row(b, n, h) + d;
            dv[r] = accumulate ? dv[r] + sv : sv;
            dk[r] = accumulate ? dk[r] + sk : sk;
        }
    }
    const size_t slot = static_cast<size_t>(bh) * nsplit + split;
#pragma unroll
    for (int i = 0; i < NA; ++i) da_part[slot * D * R + e_own * R + cg + G * i] = acc_a[i];
}

// ---- register-tiled passes for rank <= 64 (32-token tiles): lane = token of the tile; each warp owns
// FC = R/8 consecutive features (for the products over the head dimension) or D/8 consecutive dims (for
// the products over the features), so A, S and dS are read as warp-wide broadcast vectors and the
// per-token operands as conflict-free gathers (rows padded to D+1 / R+1), and a token's rotation pairs
// stay inside one thread.
// N consecutive floats from shared memory: 16-byte loads when N is a multiple of 4 (src 16-B aligned),
// else 8-byte loads (src 8-B aligned, N even).
template <int N>
__device__ __forceinline__ void ld_bcast(float (&dst)[N], const float* src) {
    if constexpr (N % 4 == 0) {
#pragma unroll
        for (int i = 0; i < N; i += 4) {
            const float4 v = *reinterpret_cast<const float4*>(src + i);
            dst[i] = v.x;
            dst[i + 1] = v.y;
            dst[i + 2] = v.z;
            dst[i + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; i += 2) {
            const float2 v = *reinterpret_cast<const float2*>(src + i);
            dst[i] = v.x;
            dst[i + 1] = v.y;
        }
    }
}

template <int D, int R>
__global__ void __launch_bounds__(256) bwd_lr_q_tiled_kernel(const __nv_bfloat16* __restrict__ q,
                                                             const float* __restrict__ dout,
                                                             const __nv_bfloat16* __restrict__ A,
                                                             const float* __restrict__ S, const float* __restrict__ z,
                                                             const double2* __restrict__ tab,
                                                             const int2* __restrict__ pairs, Geom g, int nsplit,
                                                             float* __restrict__ dq, float* __restrict__ ds_part,
                                                             float* __restrict__ dz_part, float* __restrict__ da_part,
                                                             int accumulate) {
    constexpr int TT = 32, FC = R / 8, DC = D / 8;
    static_assert(R <= 64 && FC % 2 == 0, "rank 16..64");
    extern __shared__ __align__(16) float smf[];
    float* Au = smf;                   // [D][R]   A
    float* At = Au + D * R;            // [R][D]   A^T
    float* St = At + R * D;            // [D][R]   S^T
    float* zs = St + D * R;            // [R]
    float* xs = zs + R;                // [TT][D+1] q
    float* gs = xs + TT * (D + 1);     // [TT][D+1] dO
    float* ws = gs + TT * (D + 1);     // [TT][R]   psi / den
    float* dus = ws + TT * R;          // [TT][R+1] du
    float* phs = dus + TT * (R + 1);   // [TT][R]   phi
    float* red = phs + TT * R;         // [8][2][TT] per-warp partial dots
    float* dd = red + 8 * 2 * TT;      // [TT] dden
    float* duc = dd + TT;              // [TT][R]   du, unpadded (vector reads in the partial sums)
    constexpr int G = 256 / D;
    constexpr int NA = R / G;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int split = blockIdx.x, bh = blockIdx.y;
    const int b = bh / g.Hh, h = bh % g.Hh;
    const int ntiles = (g.L + TT - 1) / TT;
    const int per = (ntiles + nsplit - 1) / nsplit;
    const int t0 = split * per, t1 = min(ntiles, t0 + per);
    const __nv_bfloat16* Ah = A + static_cast<size_t>(h) * g.a_stride;
    for (int e = tid; e < D * R; e += 256) {
        const float a = __bfloat162float(Ah[e]);
        Au[e] = a;
        At[(e % R) * D + e / R] = a;
    }
    for (int e = tid; e < R * D; e += 256) St[(e % D) * R + e / D] = S[static_cast<size_t>(bh) * R * D + e];
    if (tid < R) zs[tid] = z[static_cast<size_t>(bh) * R + tid];
    // partial sums: thread (e_own, cg) owns features [cg * NA, cg * NA + NA) of column e_own
    const int e_own = tid % D, cg = tid / D;
    float acc_s[NA], acc_a[NA];
#pragma unroll
    for (int i = 0; i < NA; ++i) acc_s[i] = acc_a[i] = 0.f;
    float acc_z = 0.f;
    const int c0 = warp * FC, d0 = warp * DC;
    // the next tile's q and dO are loaded into registers while this tile is computed
    constexpr int NL = TT * (D / 2) / 256;
    __nv_bfloat162 pq[NL];
    float2 pg[NL];
    auto fetch = [&](int tile) {
#pragma unroll
        for (int l = 0; l < NL; ++l) {
            const int e = tid + 256 * l, tt = e / (D / 2), dp = e % (D / 2);
            const int n = tile * TT + tt;
            if (tile < t1 && n < g.L) {
                pq[l] = *reinterpret_cast<const __nv_bfloat162*>(q + g.sq.row(b, n, h) + 2 * dp);
                pg[l] = *reinterpret_cast<const float2*>(dout + g.so.row(b, n, h) + 2 * dp);
            } else {
                pq[l] = __floats2bfloat162_rn(0.f, 0.f);
                pg[l] = make_float2(0.f, 0.f);
            }
        }
    };
    fetch(t0);
    for (int tile = t0; tile < t1; ++tile) {
        const int n0 = tile * TT;
        __syncthreads();
#pragma unroll
        for (int l = 0; l < NL; ++l) {
            const int e = tid + 256 * l, tt = e / (D / 2), dp = e % (D / 2);
            const float2 xf = __bfloat1622float2(pq[l]);
            xs[tt * (D + 1) + 2 * dp] = xf.x; xs[tt * (D + 1) + 2 * dp + 1] = xf.y;
            gs[tt * (D + 1) + 2 * dp] = pg[l].x; gs[tt * (D + 1) + 2 * dp + 1] = pg[l].y;
        }
        __syncthreads();
        fetch(tile + 1);
        const int n = n0 + lane;
        const bool live = n < g.L;
        const int nt = live ? n : 0;
        // this token's (cos, sin) of the warp's pairs, loaded before the products that hide their latency
        float cf[FC / 2], sf[FC / 2];
        {
            double2 cs[FC / 2];
#pragma unroll
            for (int pp = 0; pp < FC / 2; ++pp) {
                const int2 pi = __ldg(pairs + c0 / 2 + pp);
                cs[pp] = g.norope ? make_double2(1.0, 0.0) : __ldg(tab + pi.y + token_axis_pos(nt, pi.x, g.H, g.W));
            }
#pragma unroll
            for (int pp = 0; pp < FC / 2; ++pp) {
                cf[pp] = static_cast<float>(cs[pp].x);
                sf[pp] = static_cast<float>(cs[pp].y);
            }
        }
        // u = q A and G = S dO for token `lane`, features [c0, c0 + FC)
        float u[FC], gg[FC];
#pragma unroll
        for (int f = 0; f < FC; ++f) u[f] = gg[f] = 0.f;
        const float* xr = xs + lane * (D + 1);
        const float* gr = gs + lane * (D + 1);
#pragma unroll 4
        for (int d = 0; d < D; ++d) {
            float av[FC], sv[FC];
            ld_bcast(av, Au + d * R + c0);
            ld_bcast(sv, St + d * R + c0);
            const float x = xr[d], go = gr[d];
#pragma unroll
            for (int f = 0; f < FC; ++f) {
                u[f] = fmaf(x, av[f], u[f]);
                gg[f] = fmaf(sv[f], go, gg[f]);
            }
        }
        // psi and the normaliser feature nf, partial den = nf . z and psi . G over this warp's features
        LrPair P[FC / 2];
        float den_p = 0.f, dot_p = 0.f;
#pragma unroll
        for (int pp = 0; pp < FC / 2; ++pp) {
            P[pp] = lr_pair_fwd(u[2 * pp], u[2 * pp + 1], cf[pp], sf[pp], g.act, g.inside);
            den_p = fmaf(P[pp].nf0, zs[c0 + 2 * pp], fmaf(P[pp].nf1, zs[c0 + 2 * pp + 1], den_p));
            dot_p = fmaf(P[pp].psi0, gg[2 * pp], fmaf(P[pp].psi1, gg[2 * pp + 1], dot_p));
        }
        red[(warp * 2 + 0) * TT + lane] = den_p;
        red[(warp * 2 + 1) * TT + lane] = dot_p;
        __syncthreads();
        float den = 1e-6f, dot = 0.f;
        {
            float dsum = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                dsum += red[(w * 2 + 0) * TT + lane];
                dot += red[(w * 2 + 1) * TT + lane];
            }
            den += dsum;
        }
        const float dden = live ? -dot / (den * den) : 0.f;
        if (warp == 0) dd[lane] = dden;
        // psi / den for dS; du from dpsi = G / den and dnf = dden z for dq and dA; nf for dz
#pragma unroll
        for (int pp = 0; pp < FC / 2; ++pp) {
            const int c = c0 + 2 * pp;
            const float g0 = gg[2 * pp] / den, g1 = gg[2 * pp + 1] / den;
            float du0, du1;
            lr_pair_bwd(P[pp], g0, g1, dden * zs[c], dden * zs[c + 1], cf[pp], sf[pp], g.inside, du0, du1);
            du0 = live ? du0 : 0.f;
            du1 = live ? du1 : 0.f;
            ws[lane * R + c] = live ? P[pp].psi0 / den : 0.f;
            ws[lane * R + c + 1] = live ? P[pp].psi1 / den : 0.f;
            dus[lane * (R + 1) + c] = du0;
            dus[lane * (R + 1) + c + 1] = du1;
            duc[lane * R + c] = du0;
            duc[lane * R + c + 1] = du1;
            phs[lane * R + c] = P[pp].nf0;
            phs[lane * R + c + 1] = P[pp].nf1;
        }
        __syncthreads();
        // partial sums: dS[c][e] += sum_t w[t][c] dO[t][e]; dA[d][c] += sum_t q[t][d] du[t][c]; dz
#pragma unroll 2
        for (int tt = 0; tt < TT; ++tt) {
            const float go = gs[tt * (D + 1) + e_own], xo = xs[tt * (D + 1) + e_own];
            float wv[NA], uv[NA];
            ld_bcast(wv, ws + tt * R + cg * NA);
            ld_bcast(uv, duc + tt * R + cg * NA);
#pragma unroll
            for (int i = 0; i < NA; ++i) {
                acc_s[i] = fmaf(wv[i], go, acc_s[i]);
                acc_a[i] = fmaf(xo, uv[i], acc_a[i]);
            }
        }
        if (tid < R)
            for (int tt = 0; tt < TT; ++tt) acc_z = fmaf(dd[tt], phs[tt * R + tid], acc_z);
        // dq += du A^T for token `lane`, dims [d0, d0 + DC)
        if (live) {
            float o[DC];
#pragma unroll
            for (int i = 0; i < DC; ++i) o[i] = 0.f;
            const float* dur = dus + lane * (R + 1);
#pragma unroll 4
            for (int c = 0; c < R; ++c) {
                float av[DC];
                ld_bcast(av, At + c * D + d0);
                const float du = dur[c];
#pragma unroll
                for (int i = 0; i < DC; ++i) o[i] = fmaf(du, av[i], o[i]);
            }
            float* dst = dq + g.so.row(b, n, h) + d0;
#pragma unroll
            for (int i = 0; i < DC; i += 4) {
                float4 v = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
                if (accumulate) {  // the sparse part is there already
                    const float4 p = *reinterpret_cast<const float4*>(dst + i);
                    v.x += p.x; v.y += p.y; v.z += p.z; v.w += p.w;
                }
                *reinterpret_cast<float4*>(dst + i) = v;
            }
        }
    }
    const size_t slot = static_cast<size_t>(bh) * nsplit + split;
#pragma unroll
    for (int i = 0; i < NA; ++i) {
        ds_part[slot * R * D + (cg * NA + i) * D + e_own] = acc_s[i];
        da_part[slot * D * R + e_own * R + cg * NA + i] = acc_a[i];
    }
    if (tid < R) dz_part[slot * R + tid] = acc_z;
}

template <int D, int R>
__global__ void __launch_bounds__(256) bwd_lr_k_tiled_kernel(const __nv_bfloat16* __restrict__ k,
                                                             const __nv_bfloat16* __restrict__ v,
                                                             const __nv_bfloat16* __restrict__ A,
                                                             const float* __restrict__ dS, const float* __restrict__ dz,
                                                             const double2* __restrict__ tab,
                                                             const int2* __restrict__ pairs, Geom g, int nsplit,
                                                             float* __restrict__ dk, float* __restrict__ dv,
                                                             float* __restrict__ da_part, int accumulate) {
    constexpr int TT = 32, FC = R / 8, DC = D / 8;
    static_assert(R <= 64 && FC % 2 == 0, "rank 16..64");
    extern __shared__ __align__(16) float smf[];
    float* Au = smf;                   // [D][R]   A
    float* At = Au + D * R;            // [R][D]   A^T
    float* dSt = At + R * D;           // [D][R]   dS^T
    float* dSs = dSt + D * R;          // [R][D]   dS
    float* zs = dSs + R * D;           // [R]      dz
    float* xs = zs + R;                // [TT][D+1] k
    float* vs = xs + TT * (D + 1);     // [TT][D+1] v
    float* psis = vs + TT * (D + 1);   // [TT][R+1] psi
    float* dus = psis + TT * (R + 1);  // [TT][R+1] du
    float* duc = dus + TT * (R + 1);   // [TT][R]   du, unpadded (vector reads in the partial sums)
    constexpr int G = 256 / D;
    constexpr int NA = R / G;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int split = blockIdx.x, bh = blockIdx.y;
    const int b = bh / g.Hh, h = bh % g.Hh;
    const int ntiles = (g.L + TT - 1) / TT;
    const int per = (ntiles + nsplit - 1) / nsplit;
    const int t0 = split * per, t1 = min(ntiles, t0 + per);
    const __nv_bfloat16* Ah = A + static_cast<size_t>(h) * g.a_stride;
    for (int e = tid; e < D * R; e += 256) {
        const float a = __bfloat162float(Ah[e]);
        Au[e] = a;
        At[(e % R) * D + e / R] = a;
    }
    for (int e = tid; e < R * D; e += 256) {
        const float x = dS[static_cast<size_t>(bh) * R * D + e];
        dSs[e] = x;
        dSt[(e % D) * R + e / D] = x;
    }
    if (tid < R) zs[tid] = dz[static_cast<size_t>(bh) * R + tid];
    const int e_own = tid % D, cg = tid / D;
    float acc_a[NA];
#pragma unroll
    for (int i = 0; i < NA; ++i) acc_a[i] = 0.f;
    const int c0 = warp * FC, d0 = warp * DC;
    // the next tile's k and v are loaded into registers while this tile is computed
    constexpr int NL = TT * (D / 2) / 256;
    __nv_bfloat162 pk[NL], pv[NL];
    auto fetch = [&](int tile) {
#pragma unroll
        for (int l = 0; l < NL; ++l) {
            const int e = tid + 256 * l, tt = e / (D / 2), dp = e % (D / 2);
            const int n = tile * TT + tt;
            if (tile < t1 && n < g.L) {
                pk[l] = *reinterpret_cast<const __nv_bfloat162*>(k + g.sk.row(b, n, h) + 2 * dp);
                pv[l] = *reinterpret_cast<const __nv_bfloat162*>(v + g.sv.row(b, n, h) + 2 * dp);
            } else {
                pk[l] = pv[l] = __floats2bfloat162_rn(0.f, 0.f);
            }
        }
    };
    fetch(t0);
    for (int tile = t0; tile < t1; ++tile) {
        const int n0 = tile * TT;
        __syncthreads();
#pragma unroll
        for (int l = 0; l < NL; ++l) {
            const int e = tid + 256 * l, tt = e / (D / 2), dp = e % (D / 2);
            const float2 xf = __bfloat1622float2(pk[l]), vf = __bfloat1622float2(pv[l]);
            xs[tt * (D + 1) + 2 * dp] = xf.x; xs[tt * (D + 1) + 2 * dp + 1] = xf.y;
            vs[tt * (D + 1) + 2 * dp] = vf.x; vs[tt * (D + 1) + 2 * dp + 1] = vf.y;
        }
        __syncthreads();
        fetch(tile + 1);
        const int n = n0 + lane;
        const bool live = n < g.L;
        const int nt = live ? n : 0;
        float cfs[FC / 2], sfs[FC / 2];  // this token's (cos, sin) of the warp's pairs, loaded early
        {
            double2 cs[FC / 2];
#pragma unroll
            for (int pp = 0; pp < FC / 2; ++pp) {
                const int2 pi = __ldg(pairs + c0 / 2 + pp);
                cs[pp] = g.norope ? make_double2(1.0, 0.0) : __ldg(tab + pi.y + token_axis_pos(nt, pi.x, g.H, g.W));
            }
#pragma unroll
            for (int pp = 0; pp < FC / 2; ++pp) {
                cfs[pp] = static_cast<float>(cs[pp].x);
                sfs[pp] = static_cast<float>(cs[pp].y);
            }
        }
        // u = k A and dpsi = dS v for token `lane`, features [c0, c0 + FC)
        float u[FC], dp[FC];
#pragma unroll
        for (int f = 0; f < FC; ++f) u[f] = dp[f] = 0.f;
        const float* xr = xs + lane * (D + 1);
        const float* vr = vs + lane * (D + 1);
#pragma unroll 4
        for (int d = 0; d < D; ++d) {
            float av[FC], sv[FC];
            ld_bcast(av, Au + d * R + c0);
            ld_bcast(sv, dSt + d * R + c0);
            const float x = xr[d], vo = vr[d];
#pragma unroll
            for (int f = 0; f < FC; ++f) {
                u[f] = fmaf(x, av[f], u[f]);
                dp[f] = fmaf(sv[f], vo, dp[f]);
            }
        }
        // psi; du from dpsi and dnf = dz
#pragma unroll
        for (int pp = 0; pp < FC / 2; ++pp) {
            const int c = c0 + 2 * pp;
            const float cf = cfs[pp], sf = sfs[pp];
            const LrPair P = lr_pair_fwd(u[2 * pp], u[2 * pp + 1], cf, sf, g.act, g.inside);
            psis[lane * (R + 1) + c] = P.psi0;
            psis[lane * (R + 1) + c + 1] = P.psi1;
            float du0, du1;
            lr_pair_bwd(P, dp[2 * pp], dp[2 * pp + 1], zs[c], zs[c + 1], cf, sf, g.inside, du0, du1);
            du0 = live ? du0 : 0.f;
            du1 = live ? du1 : 0.f;
            dus[lane * (R + 1) + c] = du0;
            dus[lane * (R + 1) + c + 1] = du1;
            duc[lane * R + c] = du0;
            duc[lane * R + c + 1] = du1;
        }
        __syncthreads();
#pragma unroll 2
        for (int tt = 0; tt < TT; ++tt) {
            const float xo = xs[tt * (D + 1) + e_own];
            float uv[NA];
            ld_bcast(uv, duc + tt * R + cg * NA);
#pragma unroll
            for (int i = 0; i < NA; ++i) acc_a[i] = fmaf(xo, uv[i], acc_a[i]);
        }
        // dv += dS^T psi and dk += du A^T for token `lane`, dims [d0, d0 + DC)
        if (live) {
            float ov[DC], ok[DC];
#pragma unroll
            for (int i = 0; i < DC; ++i) ov[i] = ok[i] = 0.f;
            const float* pr = psis + lane * (R + 1);
            const float* dur = dus + lane * (R + 1);
#pragma unroll 2
            for (int c = 0; c < R; ++c) {
                float sv[DC], av[DC];
                ld_bcast(sv, dSs + c * D + d0);
                ld_bcast(av, At + c * D + d0);
                const float ps = pr[c], du = dur[c];
#pragma unroll
                for (int i = 0; i < DC; ++i) {
                    ov[i] = fmaf(ps, sv[i], ov[i]);
                    ok[i] = fmaf(du, av[i], ok[i]);
                }
            }
            const long long r = g.so.row(b, n, h) + d0;
#pragma unroll
            for (int i = 0; i < DC; i += 4) {
                float4 x = make_float4(ov[i], ov[i + 1], ov[i + 2], ov[i + 3]);
                float4 y = make_float4(ok[i], ok[i + 1], ok[i + 2], ok[i + 3]);
                if (accumulate) {  // the sparse parts are there already
                    const float4 px = *reinterpret_cast<const float4*>(dv + r + i);
                    const float4 py = *reinterpret_cast<const float4*>(dk + r + i);
                    x.x += px.x; x.y += px.y; x.z += px.z; x.w += px.w;
                    y.x += py.x; y.y += py.y; y.z += py.z; y.w += py.w;
                }
                *reinterpret_cast<float4*>(dv + r + i) = x;
                *reinterpret_cast<float4*>(dk + r + i) = y;
            }
        }
    }
    const size_t slot = static_cast<size_t>(bh) * nsplit + split;
#pragma unroll
    for (int i = 0; i < NA; ++i) da_part[slot * D * R + e_own * R + cg * NA + i] = acc_a[i];
}

// dA [1 + sep][per_head ? Hh : 1][D][R] from the partials [2 passes][B * Hh][ns][D][R]: each projection
// sums the passes that used it (the query pass for Pq, the key pass for Pk, both when they are one
// matrix) over the heads that share it and every split.  A CTA takes 32 consecutive outputs; its 8 warps
// each sum every 8th partial of the fixed (pass, batch, head, split) order, and the 8 sums are added in
// warp order: deterministic, with 8 loads of 128 bytes in flight per output group.
__global__ void __launch_bounds__(256) bwd_da_reduce_kernel(const float* __restrict__ da_part, Geom g, int ns,
                                                            int sep, int per_head, float* __restrict__ dA) {
    __shared__ float red[8][32];
    const int DR = g.D * g.R;
    const int nh = per_head ? g.Hh : 1;
    const int lo = threadIdx.x & 31, sl = threadIdx.x >> 5;
    const int o = blockIdx.x * 32 + lo;
    const int n_out = (1 + sep) * nh * DR;
    float s = 0.f;
    if (o < n_out) {
        const int e = o % DR, hh = (o / DR) % nh, pj = o / (DR * nh);
        const int npass = sep ? 1 : 2, nheads = per_head ? 1 : g.Hh;
        const int per_pass = g.B * nheads * ns, total = npass * per_pass;
        for (int t = sl; t < total; t += 8) {
            const int pass = sep ? pj : t / per_pass;
            const int rem = t % per_pass;
            const int b = rem / (nheads * ns), rem2 = rem % (nheads * ns);
            const int h = per_head ? hh : rem2 / ns, sp = rem2 % ns;
            s += da_part[((static_cast<size_t>(pass) * g.BH() + b * g.Hh + h) * ns + sp) * DR + e];
        }
    }
    red[sl][lo] = s;
    __syncthreads();
    if (sl == 0 && o < n_out) {
        float t = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) t += red[i][lo];
        dA[o] = t;
    }
}

namespace {
cudaError_t launch_da_reduce(const LrBwdArgs& l, const Geom& g, cudaStream_t st) {
    const int n = (1 + l.proj_separate) * (l.proj_per_head ? g.Hh : 1) * g.D * g.R;
    bwd_da_reduce_kernel<<<(n + 31) / 32, 256, 0, st>>>(l.da_part, g, l.nsplit, l.proj_separate, l.proj_per_head,
                                                         l.dA);
    return cudaGetLastError();
}
}  // namespace

// ------------------------------------------------------------------------------------ launchers
size_t lr_bwd_smem(int D, int R, bool qpass) {
    const int TT = R <= 64 ? 32 : 16;
    const int mats = D * (R + 1) + R * (D + 1);  // padded A and S (or dS)
    if (qpass) return sizeof(float) * (mats + R + 2 * TT * (D + 1) + 3 * TT * (R + 1) + 2 * TT * R + 2 * TT);
    return sizeof(float) * (mats + R + 2 * TT * (D + 1) + 3 * TT * (R + 1));
}

size_t lr_bwd_tiled_smem(int D, int R, bool qpass) {
    const int TT = 32;
    if (qpass)  // A, A^T, S^T; z; q, dO tiles; psi/den, du, phi; dot partials, dden; du unpadded
        return sizeof(float) * (3 * D * R + R + 2 * TT * (D + 1) + TT * R + TT * (R + 1) + TT * R + 16 * TT + TT + TT * R);
    // A, A^T, dS^T, dS; dz; k, v; psi, du; du unpadded
    return sizeof(float) * (4 * D * R + R + 2 * TT * (D + 1) + 2 * TT * (R + 1) + TT * R);
}

int lr_bwd_nsplit(const Geom& g) {
    if (lr_bwd_on_tensor_cores(g)) return lowrank_nsplit(g);  // 128-token tiles, about 8 items per CTA
    const int TT = g.R <= 64 ? 32 : 16;
    const long long ntiles = (g.L + TT - 1) / TT;
    long long ns = (2 * 148 + g.BH() - 1) / g.BH();
    ns = ns < 1 ? 1 : (ns > ntiles ? ntiles : ns);
    return static_cast<int>(ns);
}

namespace {
template <int D, int BLK>
cudaError_t launch_bwd_sparse_t(const BwdMaps& m, const BwdArgs& a, const Geom& g, cudaStream_t st) {
    const size_t sq = DqLayout<D>::kBytes + 1024, skv = DkvLayout<D, BLK>::kBytes + 1024;
    cudaError_t e = cudaFuncSetAttribute(bwd_dq_kernel<D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sq);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_dkdv_kernel<D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)skv);
    if (e != cudaSuccess) return e;
    bwd_dq_kernel<D, BLK><<<dim3(g.nb, g.BH()), BwdRoles<BLK>::kThreads, sq, st>>>(m.q128, m.do128, m.kb, m.vb, a, g);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (m.between) cudaEventRecord(m.between, st);
    bwd_dkdv_kernel<D, BLK><<<dim3(g.nb, g.BH()), BwdRoles<BLK>::kThreads, skv, st>>>(m.k128, m.v128, m.qb, m.dob, a,
                                                                                    g);
    return cudaGetLastError();
}

template <int D, int R>
cudaError_t launch_lr_bwd_t(const LrBwdArgs& l, const Geom& g, cudaStream_t st) {
    const int ns = l.nsplit;
    constexpr bool kTiled = R <= 64;  // the register-tiled passes (32-token tiles)
    const size_t smq = kTiled ? lr_bwd_tiled_smem(D, R, true) : lr_bwd_smem(D, R, true);
    const size_t smk = kTiled ? lr_bwd_tiled_smem(D, R, false) : lr_bwd_smem(D, R, false);
    auto qk = kTiled ? bwd_lr_q_tiled_kernel<D, (R <= 64 ? R : 64)> : bwd_lr_q_kernel<D, R>;
    auto kk = kTiled ? bwd_lr_k_tiled_kernel<D, (R <= 64 ? R : 64)> : bwd_lr_k_kernel<D, R>;
    cudaError_t e = cudaFuncSetAttribute(qk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smq);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smk);
    if (e != cudaSuccess) return e;
    qk<<<dim3(ns, g.BH()), 256, smq, st>>>(l.q, l.dout, l.A, l.S, l.z, l.tab, l.pairs, g, ns, l.dq, l.ds_part,
                                           l.dz_part, l.da_part, l.accumulate);  // query projection(s)
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = launch_lowrank_reduce(l.ds_part, l.dz_part, g, ns, l.dS, l.dz, nullptr, nullptr, nullptr, st)) !=
        cudaSuccess)
        return e;
    kk<<<dim3(ns, g.BH()), 256, smk, st>>>(l.k, l.v, l.A + l.key_proj_offset(g), l.dS, l.dz, l.tab, l.pairs, g, ns,
                                           l.dk, l.dv, l.da_part + static_cast<size_t>(g.BH()) * ns * D * R,
                                           l.accumulate);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return launch_da_reduce(l, g, st);
}
}  // namespace

cudaError_t launch_bwd_prep(const float* dout, const float* os, const Geom& g, __half* doh, float* delta, int* status,
                            cudaStream_t st) {
    const long long rows = static_cast<long long>(g.BH()) * g.Lp;
    const long long blocks = (rows * 32 + 255) / 256;
    bwd_prep_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(dout, os, g, doh, delta, status);
    return cudaGetLastError();
}

cudaError_t launch_bwd_invert(const int32_t* idx, const Geom& g, int32_t* inv, int32_t* inv_cnt, cudaStream_t st) {
    bwd_invert_kernel<<<dim3(g.nb, g.BH()), 128, 0, st>>>(idx, g, inv, inv_cnt);
    return cudaGetLastError();
}

cudaError_t launch_bwd_sparse(const BwdMaps& m, const BwdArgs& a, const Geom& g, cudaStream_t st) {
    if (g.D == 128) return g.block == 128 ? launch_bwd_sparse_t<128, 128>(m, a, g, st) : launch_bwd_sparse_t<128, 64>(m, a, g, st);
    return g.block == 128 ? launch_bwd_sparse_t<64, 128>(m, a, g, st) : launch_bwd_sparse_t<64, 64>(m, a, g, st);
}

cudaError_t launch_lr_bwd(const LrBwdArgs& l, const Geom& g, cudaStream_t st) {
    if (lr_bwd_on_tensor_cores(g)) {
        cudaError_t e = launch_lr_bwd_tc(l, g, st);
        if (e != cudaSuccess) return e;
        return launch_da_reduce(l, g, st);
    }
    if (g.D == 128) {
        switch (g.R) {
            case 16: return launch_lr_bwd_t<128, 16>(l, g, st);
            case 32: return launch_lr_bwd_t<128, 32>(l, g, st);
            case 48: return launch_lr_bwd_t<128, 48>(l, g, st);
            case 64: return launch_lr_bwd_t<128, 64>(l, g, st);
            case 80: return launch_lr_bwd_t<128, 80>(l, g, st);
            case 96: return launch_lr_bwd_t<128, 96>(l, g, st);
            case 112: return launch_lr_bwd_t<128, 112>(l, g, st);
            case 128: return launch_lr_bwd_t<128, 128>(l, g, st);
        }
    } else if (g.D == 64) {
        switch (g.R) {
            case 16: return launch_lr_bwd_t<64, 16>(l, g, st);
            case 32: return launch_lr_bwd_t<64, 32>(l, g, st);
            case 48: return launch_lr_bwd_t<64, 48>(l, g, st);
            case 64: return launch_lr_bwd_t<64, 64>(l, g, st);
        }
    }
    return cudaErrorInvalidValue;
}

}  // namespace slra
