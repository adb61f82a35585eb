// Block-sparse softmax attention over the kept key blocks, on the sm_100a tensor cores, with the
// low-rank branch's query-side readout fused into the epilogue.
//
// Method (RoLA, "4.1"): for each query block alpha, exact softmax attention of its queries over the
// union of the kept key blocks K(alpha); plus O_lr,i = psi(q_i)^T S / (phi(q_i) . z + 1e-6) with
// phi = relu(q A) on the raw query and psi its first r coordinates rotated by 3D RoPE ("4.2", "4.3");
// SiLU, identity or tanh in place of relu, and psi = phi without the rotation, are the options of the
// ablation ("5.3").
//
// One CTA per (query block, batch*head), one CTA per SM, warp-specialised (320 threads):
//   warps 0-7  softmax: row i lives in TMEM lane i; warps w and w+4 both reach lanes 32(w%4).. and
//              split the key block in halves, exchanging their row maxima (and at the end their row
//              sums) through shared memory: row max, lazy rescale of O (only when the max grows by
//              more than 2^8), P = 2^(s*log2e/sqrt(D) - m) rounded to bf16 and written back into the
//              TMEM columns of that S buffer;
//   warp 8     TMA producer: q^ tile, then k^ tiles (the fp16 head-major copies) and v tiles (bf16,
//              straight from the caller's token-major v) into two slots each (128-B swizzle), each
//              slot refilled as soon as the product that read it has completed;
//   warp 9     MMA issuer: once the softmax has released P_j, O += P_j v_j (A operand P_j from TMEM,
//              B = v tile MN-major; bf16) and S_{j+2} = q^ k^T_{j+2} (fp16) into the S buffer P_{j-1}
//              occupied (tcgen05.mma kind::f16, M=128, N=block, K=D, fp32 in TMEM), their k-steps
//              issued alternately.
// With three S buffers S_{j+1} is already in TMEM when the softmax finishes S_j, so a key block
// costs about the longer of the softmax and the two products instead of their sum.  The two
// products' k-steps are interleaved one by one: the tensor pipe runs a run of four or more
// products of one kind followed by a run of the other at about half rate, strictly alternating
// ones at full rate.
// TMEM (512 columns): S0 | S1 | S2 | O; the epilogue's phi = q A reuses S0.
// Epilogue (softmax warps): the low-rank readout (head_dim 128: on the tensor cores, accumulated into
// O; head_dim 64: on the CUDA cores in fp32), then O / l staged in shared memory and written by TMA
// stores (fp32 or bf16).
//
// All waits are bounded (see sm100.cuh); a wait that runs out records a timeout in the status word,
// every role leaves its loop, lets what it issued land, and the CTA releases its tensor memory.
#include "common.cuh"
#include "sm100.cuh"

namespace slra {

namespace {

constexpr int kSoftWarps = 8;
constexpr int kSoftThreads = kSoftWarps * 32;
constexpr int kWarpLoad = 8;   // TMA producer
constexpr int kWarpMma = 9;    // tcgen05.mma issuer
constexpr int kThreads = 320;
constexpr int kNumS = 3;        // S buffers
constexpr int kTmemCols = 512;  // S buffers at [128 b, 128 b + 128), O at [384, 384 + D)
constexpr int kColO = 384;
constexpr int kColPhi = 0;      // epilogue: phi in S0 (free once the last P.V has completed)

// Shared memory: q^ tile, two k^ slots, two v slots (each sized for a 128-row block), barriers,
// the row-partial exchange buffer.  The epilogue reuses the tile area.
template <int D>
struct AttnLayout {
    static constexpr int kTile = 128 * D * 2;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kTile;      // slots s at kOffK + s * kTile
    static constexpr int kOffV = kOffK + 2 * kTile;  // slots s at kOffV + s * kTile
    static constexpr int kOffBar = kOffV + 2 * kTile;  // 32 mbarriers
    static constexpr int kOffMisc = kOffBar + 256;     // tmem base, abort flag
    static constexpr int kOffXch = kOffMisc + 64;      // [2 parities][2 halves][128] fp32 row partials
    static constexpr int kBytes = kOffXch + 2048;
};

// mbarrier indices
enum : int {
    kBarQ = 0,
    kBarKFull = 1,    // +slot: k_0, k_1 landed (the first two S)
    kBarKvEmpty = 3,  // +slot: the products that read the slot's k and v tiles have completed
    kBarVFull = 5,    // +slot: v_j and, when there is one, k_{j+2} landed (block j's two products)
    kBarSFull = 9,    // +buffer: S_j in TMEM (and every product issued before it completed)
    kBarPFull = 12,   // +buffer: P_j in TMEM (one arrival per softmax thread)
    kBarODone = 15,   // P.V_{keep-2} has completed (one phase)
    kBarEld = 18,     // epilogue: raw query tile + A^T image
    kBarEz = 19,      // epilogue: S image of each 64-feature chunk
    kBarEmm = 20,     // epilogue products
    kBarDebug = 21,   // test hook: nothing arrives here
    kBarDrain = 22,   // MMA issuer's final commit on the abort path
    kBarOFinal = 23,  // the last P.V has completed (one phase)
    kNumBars = 24
};

// Named barrier 1 over the softmax warps only (the producer and MMA warps never take part).
__device__ __forceinline__ void group_sync() { asm volatile("barrier.cta.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ bool group_sync_or(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.or.pred q, 1, 256, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred))
        : "memory");
    return r != 0;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// (d0, d1) = (a0 * b0 + c0, a1 * b1 + c1) as one packed fp32x2 FMA.
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                      float c1) {
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

// (s0, s1) += (a0, a1) as one packed fp32x2 add.
__device__ __forceinline__ void fadd2(float& s0, float& s1, float a0, float a1) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%0, %1};\n\tmov.b64 rb, {%2, %3};\n\t"
        "add.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "+f"(s0), "+f"(s1)
        : "f"(a0), "f"(a1));
}

// bf16x2 with lo in the low half (the lower key index sits in the lower 16 bits of a TMEM column).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

}  // namespace

// kDefault: relu features with the low-rank RoPE and the plain sum of the branches (the benchmark's
// configuration); the activation, no-RoPE and gated-fusion branches then fold away at compile time.
template <int D, int BLK, bool kDefault>
__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_qraw,
                      const __grid_constant__ CUtensorMap tm_out, const __grid_constant__ CUtensorMap tm_os,
                      AttnArgs a, Geom g) {
    using Lay = AttnLayout<D>;
    const int act = kDefault ? 0 : g.act;        // low-rank feature map
    const int norope = kDefault ? 0 : g.norope;  // 1: no rotation in the low-rank branch
    const int gated = kDefault ? 0 : a.gated;    // 1: gated fusion of the branches instead of their sum
    const int inside = kDefault ? 0 : g.inside;  // 1: the low-rank RoPE before the activation
    constexpr int HW = BLK / 2;   // keys per thread: the two warps of a lane group split the key block
    constexpr int NC = HW / 32;   // 32-column TMEM loads per thread
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kOffBar);
    uint64_t* bar_q = bars + kBarQ;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kOffMisc + 4);
    float* xch = reinterpret_cast<float*>(smem + Lay::kOffXch);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int lg = warp & 3;    // TMEM lane group (rows 32*lg ..), fixed by the warp's rank in its warpgroup
    const int hf = (warp >> 2) & 1;   // softmax warps: which half of the key block (and of O's columns)
    const int i_row = lg * 32 + lane;
    const int alpha = blockIdx.x, bh = blockIdx.y;
    const int b = bh / g.Hh, h = bh % g.Hh;
    const int blk = BLK;
    const int keep = a.keep;
    const uint64_t tmo = a.timeout_ns;
    const int32_t* my_idx = a.idx + (static_cast<size_t>(bh) * g.nb + alpha) * (keep > 0 ? g.keep : 0);

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i)
            mbar_init(bars + i, (i >= kBarPFull && i < kBarPFull + kNumS) ? kSoftThreads : 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tO = tmem + kColO;       // O accumulator
    const uint32_t tPhi = tmem + kColPhi;   // epilogue: phi = q A
    const uint32_t lane_base = static_cast<uint32_t>(lg * 32) << 16;
    const int row0 = bh * g.Lp;  // first row of this head in the head-major buffers

    auto fail = [&]() {
        *abort_flag = 1;
        atomicOr(a.status, kDevTimeout);
    };
    // Test hook: wait on a barrier that nothing arrives at; the bounded wait runs out, records a timeout
    // and every role sees the abort flag before any copy or product has been issued.
    if (a.debug_unsatisfied_wait && tid == 0 && !mbar_wait(bars + kBarDebug, 0, tmo, abort_flag)) fail();
    __syncthreads();

    const bool prefetch_epi = (D == 128) && a.lowrank && keep > 0;
    // epilogue barrier bookkeeping (softmax thread 0 for the loads; every softmax thread for the products)
    int n_eld_issued = 0, n_eld = 0, n_emm_issued = 0, n_emm = 0, n_ez_issued = 0, n_ez = 0;
    uint64_t* bar_eld = bars + kBarEld;
    uint64_t* bar_ez = bars + kBarEz;
    uint64_t* bar_emm = bars + kBarEmm;
    // The low-rank readout's raw query tile and A^T image go to the q tile and k slot 0, the first
    // chunk's S image (rank <= 64) right after them; all are free once the last S has completed.
    auto issue_epilogue_prefetch = [&]() {
        mbar_expect_tx(bar_eld, 32768 + g.R * 256);
        tma_load_4d(smem, &tm_qraw, bar_eld, 0, h, alpha * blk, b);
        tma_load_4d(smem + 16384, &tm_qraw, bar_eld, 64, h, alpha * blk, b);
        // this head's image when the projections are per head
        bulk_load(smem + 32768, a.at_img + (g.a_stride ? static_cast<size_t>(h) * g.R * 256 : 0), g.R * 256, bar_eld);
        ++n_eld_issued;
        if (g.R <= 64) {
            const uint32_t zb = static_cast<uint32_t>((3 * g.R + 63) / 64) * (D * 128);
            mbar_expect_tx(bar_ez, zb);
            bulk_load(smem + 49152, a.sb_img + static_cast<size_t>(bh) * ((g.R + 63) / 64) * kSbChunkBytes, zb,
                      bar_ez);
            ++n_ez_issued;
        }
    };

    float l_run = 0.f;
    // m_run is the row's running max (identical in both halves); l_run sums this half's keys only.
    float m_run = 0.f;
    if (warp == kWarpLoad) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0 && keep > 0 && !*abort_flag) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            auto load_tile = [&](uint64_t* bar, uint8_t* dst, const CUtensorMap* tm, int row, int rows) {
                mbar_expect_tx(bar, static_cast<uint32_t>(rows) * D * 2);
#pragma unroll
                for (int s = 0; s < D / 64; ++s) tma_load_2d(dst + s * (rows * 128), tm, bar, s * 64, row);
            };
            auto kslot = [&](int s) { return smem + Lay::kOffK + s * Lay::kTile; };
            auto vslot = [&](int s) { return smem + Lay::kOffV + s * Lay::kTile; };
            int nk = 0, nv = 0;  // tiles issued
            bool ok = true;
            load_tile(bar_q, smem + Lay::kOffQ, &tm_q, row0 + alpha * blk, 128);
            load_tile(bars + kBarKFull, kslot(0), &tm_k, row0 + __ldg(my_idx) * blk, blk);
            nk = 1;
            if (keep > 1) {
                load_tile(bars + kBarKFull + 1, kslot(1), &tm_k, row0 + __ldg(my_idx + 1) * blk, blk);
                nk = 2;
            }
            // Block j's products read v_j (P.V_j) and k_{j+2} (S_{j+2}): both copies land on one
            // barrier per slot, so the MMA warp checks one barrier for them instead of two.  v_j's
            // bytes are registered without an arrival; the arrival comes with k_{j+2}'s bytes, or
            // alone when there is no k_{j+2}.
            auto add_tile = [&](uint64_t* bar, uint8_t* dst, const CUtensorMap* tm, int row, int rows, bool arrive) {
                if (arrive) mbar_expect_tx(bar, static_cast<uint32_t>(rows) * D * 2);
                else mbar_add_tx(bar, static_cast<uint32_t>(rows) * D * 2);
#pragma unroll
                for (int sl = 0; sl < D / 64; ++sl) tma_load_2d(dst + sl * (rows * 128), tm, bar, sl * 64, row);
            };
            // v_j straight from the caller's token-major bf16 v (tokens past L read as zero)
            auto add_vtile = [&](uint64_t* bar, uint8_t* dst, int j, bool arrive) {
                if (arrive) mbar_expect_tx(bar, static_cast<uint32_t>(blk) * D * 2);
                else mbar_add_tx(bar, static_cast<uint32_t>(blk) * D * 2);
                const int n0 = __ldg(my_idx + j) * blk;
#pragma unroll
                for (int sl = 0; sl < D / 64; ++sl) tma_load_4d(dst + sl * (blk * 128), &tm_v, bar, sl * 64, h, n0, b);
            };
            // Slot s's k and v tiles are read by the products the MMA warp issues together (P.V_j with
            // S_{j+2}), so one commit frees both: v_j and k_{j+2} go into slot s once P.V_{j-2} and S_j
            // have completed (for j < 2: S_j alone, and v_j needs no wait).
            for (int j = 0; j < keep && ok; ++j) {
                const int s = j & 1;
                const bool has_k = j + 2 < keep;
                if (j >= 2 && !mbar_wait(bars + kBarKvEmpty + s, (j >> 1) & 1, tmo, abort_flag)) {
                    ok = false;
                    break;
                }
                add_vtile(bars + kBarVFull + s, vslot(s), j, !has_k);
                ++nv;
                if (has_k) {
                    if (j < 2 && !mbar_wait(bars + kBarKvEmpty + s, 0, tmo, abort_flag)) {
                        mbar_arrive(bars + kBarVFull + s);  // complete the phase v_j's bytes are on
                        ok = false;
                        break;
                    }
                    add_tile(bars + kBarVFull + s, kslot(s), &tm_k, row0 + __ldg(my_idx + j + 2) * blk, blk, true);
                    ++nk;
                }
            }
            if (!ok) {
                fail();
                // let every issued copy land (bounded, ignoring the abort flag)
                volatile int no_abort = 0;
                const uint64_t drain = 10000000ull;
                mbar_wait(bar_q, 0, drain, &no_abort);
                for (int n = 0; n < (nk < 2 ? nk : 2); ++n)  // k_0, k_1 (later k tiles ride with the v tiles)
                    mbar_wait(bars + kBarKFull + n, 0, drain, &no_abort);
                for (int n = nv - 2 < 0 ? 0 : nv - 2; n < nv; ++n)
                    mbar_wait(bars + kBarVFull + (n & 1), (n >> 1) & 1, drain, &no_abort);
            }
        }
        __syncwarp();
    } else if (warp == kWarpMma) {
        // ---------------------------------------------------------------- tcgen05.mma issuer
        if (lane == 0 && keep > 0 && !*abort_flag) {
            const uint32_t idesc_s = idesc_f16_f32(128, blk, false, false);
            const uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);  // P bf16 (TMEM), v bf16
            const uint32_t q_addr = smem_addr(smem + Lay::kOffQ);
            // Operand descriptors per slot, computed once; a k-step adds a compile-time offset to the
            // 14-bit address field (shared-memory addresses stay below 2^18, so it cannot carry out).
            // The issuing warp shares its sub-partition with two busy softmax warps, so every issue
            // slot it saves shows up as tensor-pipe throughput.
            const uint64_t dq = sdesc_sw128(q_addr, 16, 1024);
            const uint64_t dk0 = sdesc_sw128(smem_addr(smem + Lay::kOffK), 16, 1024);
            const uint64_t dk1 = sdesc_sw128(smem_addr(smem + Lay::kOffK + Lay::kTile), 16, 1024);
            const uint64_t dv0 = sdesc_sw128(smem_addr(smem + Lay::kOffV), static_cast<uint32_t>(blk) * 128, 1024);
            const uint64_t dv1 = sdesc_sw128(smem_addr(smem + Lay::kOffV + Lay::kTile), static_cast<uint32_t>(blk) * 128, 1024);
            auto s_step = [&](uint32_t dst, uint64_t dkj, int kk) {  // k-step kk of S = q^ k^T
                const uint32_t qo = static_cast<uint32_t>(((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4);
                const uint32_t ko = static_cast<uint32_t>(((kk >> 2) * (BLK * 128) + (kk & 3) * 32) >> 4);
                umma_ss(dst, dq + qo, dkj + ko, idesc_s, kk > 0 ? 1u : 0u);
            };
            auto pv_step = [&](uint32_t p, uint64_t dvj, int kk, uint32_t acc) {  // k-step kk of O += P v
                umma_ts(tO, p + kk * 8, dvj + static_cast<uint32_t>((kk * 2048) >> 4), idesc_o, acc);
            };
            constexpr int kSSteps = D / 16, kPvSteps = BLK / 16;
            bool ok = mbar_wait(bar_q, 0, tmo, abort_flag);
            for (int j = 0; j < 2 && j < keep && ok; ++j) {  // S_0, S_1 have no P.V to pair with
                ok = mbar_wait(bars + kBarKFull + j, 0, tmo, abort_flag);
                if (ok) {
                    tc_fence_after();
                    const uint32_t dst = tmem + j * 128;
#pragma unroll
                    for (int kk = 0; kk < kSSteps; ++kk) s_step(dst, j ? dk1 : dk0, kk);
                    umma_commit(bars + kBarSFull + j);
                    if (j + 2 < keep) umma_commit(bars + kBarKvEmpty + j);
                }
            }
            for (int j = 0; j < keep && ok; ++j) {
                // P.V_j paired with S_{j+2}, whose buffer held P_{j-1} (read by P.V_{j-1}, issued earlier
                // from this thread: products run in order)
                const bool has_s = j + 2 < keep;
                if (!mbar_wait(bars + kBarPFull + j % kNumS, (j / kNumS) & 1, tmo, abort_flag) ||
                    !mbar_wait(bars + kBarVFull + (j & 1), (j >> 1) & 1, tmo, abort_flag)) {  // v_j, k_{j+2}
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t pj = tmem + (j % kNumS) * 128, s2 = tmem + ((j + 2) % kNumS) * 128;
                const uint64_t dvj = (j & 1) ? dv1 : dv0, dkj = (j & 1) ? dk1 : dk0;
                const uint32_t acc0 = j > 0 ? 1u : 0u;
                if (has_s) {
#pragma unroll
                    for (int t = 0; t < (kSSteps > kPvSteps ? kSSteps : kPvSteps); ++t) {
                        if (t < kPvSteps) pv_step(pj, dvj, t, t > 0 ? 1u : acc0);
                        if (t < kSSteps) s_step(s2, dkj, t);
                    }
                } else {
#pragma unroll
                    for (int t = 0; t < kPvSteps; ++t) pv_step(pj, dvj, t, t > 0 ? 1u : acc0);
                }
                // Two commits per block: a commit tracks every product issued before it, so S_{j+2}'s
                // also reports P.V_j (the softmax's rescale of O waits on it), and one frees both tiles
                // of slot j & 1.  The last two P.V have no S beside them and barriers of their own.
                if (has_s) {
                    umma_commit(bars + kBarSFull + (j + 2) % kNumS);
                    umma_commit(bars + kBarKvEmpty + (j & 1));
                } else {
                    umma_commit(bars + (j == keep - 1 ? kBarOFinal : kBarODone));
                }
            }
            if (!ok) fail();
            // One more commit tracks every product this thread issued; waiting for it (bounded, whatever
            // the abort flag says) means none of them outlives the CTA, however the other roles end.
            umma_commit(bars + kBarDrain);
            volatile int no_abort = 0;
            mbar_wait(bars + kBarDrain, 0, 10000000ull, &no_abort);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax warps
        const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
        // The kept list is ascending, so the only block that can be partial (the sequence's last) can
        // only be the last one visited.
        const int last_valid = keep > 0 ? min(blk, g.L - __ldg(my_idx + keep - 1) * blk) : blk;
        const int key0 = hf * HW;  // first key of this thread's half of the block
        for (int j = 0; j < keep; ++j) {
            const int sb = j % kNumS;
            const uint32_t tSj = tmem + sb * 128;
            // warp-uniform, since the TMEM loads below are warp-collective
            const bool ok = __all_sync(0xffffffffu, mbar_wait(bars + kBarSFull + sb, (j / kNumS) & 1, tmo, abort_flag));
            tc_fence_after();
            if (tid == 0 && ok && j == keep - 1 && prefetch_epi) issue_epilogue_prefetch();  // all S done
            // ---- softmax of row i_row over keys [key0, key0 + HW)
            uint32_t sr[NC][32];
            if (ok) {
#pragma unroll
                for (int c = 0; c < NC; ++c) tmem_ld32(tSj + lane_base + key0 + c * 32, sr[c]);
                tmem_ld_wait(sr[0]);
#pragma unroll
                for (int c = 1; c < NC; ++c) reg_fence(sr[c]);
            }
            constexpr int NE = HW;  // elements this thread owns
            auto el = [&](int e) -> uint32_t& { return sr[e >> 5][e & 31]; };
            if (j == keep - 1 && last_valid < blk) {
#pragma unroll
                for (int e = 0; e < NE; ++e)
                    if (key0 + e >= last_valid) el(e) = __float_as_uint(-INFINITY);
            }
            // row max over this half: four independent chains of 3-input max
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int e = 0; e < NE; e += 8) {
#pragma unroll
                for (int t = 0; t < 4; ++t)
                    mx4[t] = fmax3(mx4[t], __uint_as_float(el(e + 2 * t)), __uint_as_float(el(e + 2 * t + 1)));
            }
            const float mx_half = fmax3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3]));
            float* xj = xch + (j & 1) * 256;  // by parity, so a fast thread's next write cannot meet this read
            xj[hf * 128 + i_row] = mx_half;
            // One barrier exchanges the two halves' maxima, makes the abort decision uniform, and orders
            // every thread's S loads before the P stores below (half 1's P columns overlap half 0's S).
            tc_fence_before();
            if (group_sync_or(!ok)) {
                if (tid == 0) fail();
                break;
            }
            tc_fence_after();
            float mx = fmaxf(mx_half, xj[(hf ^ 1) * 128 + i_row]);  // same value in both halves
            mx *= scale_log2;
            if (j == 0) {
                m_run = mx;
            } else if (__any_sync(0xffffffffu, mx > m_run + 8.0f)) {  // warp-uniform: TMEM access is collective
                // Both warps of the lane group see the same maxima, so they take the same branch; each
                // rescales its half of O's columns once P.V_{j-1} has landed in O.
                // P.V_{j-1} completes with S_{j+1} (issued together, one commit); the last two P.V have
                // no S beside them, and P.V_{keep-2} has a barrier of its own.  S_{j+1}'s buffer has no
                // later phase yet (that would need P_{j+2}).
                const bool landed = __all_sync(
                    0xffffffffu, j + 1 < keep
                                     ? mbar_wait(bars + kBarSFull + (j + 1) % kNumS, ((j + 1) / kNumS) & 1, tmo, abort_flag)
                                     : mbar_wait(bars + kBarODone, 0, tmo, abort_flag));
                tc_fence_after();
                const float m_new = fmaxf(m_run, mx);
                const float alpha_r = ex2_approx(m_run - m_new);
                if (landed) {
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {  // 16 columns at a time (the scores stay in registers)
                        uint32_t o[16];
                        tmem_ld16(tO + lane_base + hf * (D / 2) + c * 16, o);
                        tmem_ld_wait(o);
#pragma unroll
                        for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha_r);
                        tmem_st16(tO + lane_base + hf * (D / 2) + c * 16, o);
                    }
                    tmem_st_wait();
                } else if (lane == 0) {
                    fail();
                }
                l_run *= alpha_r;
                m_run = m_new;
            }
            const float neg_m = -m_run;
            float sums[4][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};  // independent accumulators
            // keys (2i, 2i+1) of this half -> packed bf16x2 TMEM column key0/2 + i, 16 columns at a time
#pragma unroll
            for (int c16 = 0; c16 < NE / 32; ++c16) {
                uint32_t pk[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int i = c16 * 16 + u;
                    float t0, t1;
                    ffma2(t0, t1, __uint_as_float(el(2 * i)), __uint_as_float(el(2 * i + 1)), scale_log2, scale_log2,
                          neg_m, neg_m);
                    const float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
                    fadd2(sums[u & 3][0], sums[u & 3][1], p0, p1);
                    pk[u] = pack_bf16x2(p0, p1);
                }
                tmem_st16(tSj + lane_base + key0 / 2 + c16 * 16, pk);
            }
            tmem_st_wait();
            l_run += ((sums[0][0] + sums[0][1]) + (sums[1][0] + sums[1][1])) +
                     ((sums[2][0] + sums[2][1]) + (sums[3][0] + sums[3][1]));
            tc_fence_before();
            mbar_arrive(bars + kBarPFull + sb);  // P_j of this thread's row half is in TMEM
        }
    }

    // ==================================================================== softmax warps: epilogue
    if (warp < kSoftWarps) {
    if (keep > 0) {  // the last P.V has landed in O
        const bool ok = !*abort_flag && mbar_wait(bars + kBarOFinal, 0, tmo, abort_flag);
        if (group_sync_or(!ok) && tid == 0) fail();
    }
    // Row sum: the two halves' partial sums (fp32 addition commutes, so both get the same total).
    xch[hf * 128 + i_row] = l_run;
    group_sync();
    l_run += xch[(hf ^ 1) * 128 + i_row];
    // the softmax's log-sum-exp per row (log2 units), for a backward pass; rows past L get +inf so that
    // their probabilities recompute as zero
    if (a.lse != nullptr && hf == 0 && i_row < blk && keep > 0) {
        const int n_row = alpha * blk + i_row;
        a.lse[static_cast<size_t>(bh) * g.Lp + n_row] =
            n_row < g.L ? m_run + log2f(l_run) : INFINITY;
    }
    // The producer and MMA warps may raise the abort flag at any time, so every decision that picks a
    // path through the group barriers is taken from one reduction.
    const bool aborted = group_sync_or(*abort_flag != 0);  // also: the exchange buffer is reused below
    tc_fence_after();

    // Kept for a backward pass: the sparse branch's own output O_s = O / l, read before the low-rank
    // readout joins O.  It is staged in the v slots (free once the last P.V has completed; the readout
    // uses the q tile and the k slots) as fp32 boxes of 32 columns and stored head-major; the stores'
    // reads of the staging are waited for with the output's, or in the teardown.
    bool os_committed = false;
    if (a.os_save != nullptr && keep > 0 && !aborted) {
        const float inv_l_s = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
        for (int cc = 0; cc < D / 64; ++cc) {
            const int c = hf * (D / 64) + cc;  // 32-column group of O
            uint32_t o[32];
            tmem_ld32(tO + lane_base + c * 32, o);
            tmem_ld_wait(o);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const uint32_t off = Lay::kOffV + c * 16384 + i_row * 128 + ((u ^ (i_row & 7)) << 4);
                *reinterpret_cast<float4*>(smem + off) =
                    make_float4(__uint_as_float(o[4 * u]) * inv_l_s, __uint_as_float(o[4 * u + 1]) * inv_l_s,
                                __uint_as_float(o[4 * u + 2]) * inv_l_s, __uint_as_float(o[4 * u + 3]) * inv_l_s);
            }
        }
        fence_async_smem();
        group_sync();
        if (tid == 0) {
            for (int bx = 0; bx < D / 32; ++bx)
                for (int rh = 0; rh * 64 < blk; ++rh) {
                    if (alpha * blk + rh * 64 >= g.L) break;
                    tma_store_4d(&tm_os, smem + Lay::kOffV + bx * 16384 + rh * 64 * 128, bx * 32, h,
                                 alpha * blk + rh * 64, b);
                }
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            os_committed = true;
        }
    }

    // ------------------------------------------------------------------ epilogue
    const int n = alpha * blk + i_row;
    const bool row_valid = (i_row < blk) && (n < g.L) && !aborted;
    float inv_l = (keep > 0 && l_run > 0.f) ? 1.f / l_run : 0.f;
    bool o_live = keep > 0;  // O holds the sparse branch (and, below, the low-rank readout)
    // Gated fusion (RoLA 4.4, as read here): out = O_s + g O_lr rms(O_s) / sqrt(mean(O_lr^2) + 1e-6),
    // g = sigmoid(q . Wg + bg) on the raw query.  The readout then goes to TMEM columns of its own
    // (head_dim 128: S buffer 1, free once the last P.V has completed) or stays in registers (64).
    float glogit = 0.f;   // q . Wg + bg of this row
    bool lr_live = false;  // gated: the low-rank output of this row is available
    const uint32_t tLr = tmem + 128;
    if constexpr (D == 128) {
        if (a.lowrank && !aborted) {
            // Low-rank readout on the tensor cores, accumulated straight into O (so out = O / l):
            //   phi = q A        raw bf16 query tile (TMA) x A^T image, into TMEM columns of its own;
            //   psi = R_r(p) act(phi) * l / (act(phi) . z + 1e-6), split into bf16 hi + lo (no R_r
            //         when the low-rank RoPE is off);
            //   O  += psi S      as psi_hi S_hi + psi_hi S_lo + psi_lo S_hi, one 64-feature chunk at a time.
            // The two warps of a lane group share each row: 32-feature column groups of the
            // denominator alternate between them, and so do the rotation pairs.
            const int R = g.R;
            const int nch = (R + 63) / 64;
            uint8_t* X = smem;           // raw query tile, then each chunk's psi operand [128][3*rc]
            uint8_t* Y = smem + 32768;   // A^T image [R][128]
            uint8_t* Z = smem + 49152;   // S image of the current chunk [128][3*rc]
            const bool z_early = R <= 64;  // Y and Z do not overlap: chunk 0's S image loads right away
            auto sb_bytes = [&](int ch) -> uint32_t {
                const int rc = min(64, R - 64 * ch);
                return static_cast<uint32_t>((3 * rc + 63) / 64) * (D * 128);
            };
            const uint8_t* sb_head = a.sb_img + static_cast<size_t>(bh) * nch * kSbChunkBytes;
            // bar_eld: raw query tile + A^T image (prefetched during the last key block when there is
            // one); bar_ez: the S image of each chunk in turn
            if (tid == 0) {
                if (!prefetch_epi) issue_epilogue_prefetch();  // also chunk 0's S image when rank <= 64
                if (mbar_wait(bar_eld, n_eld & 1, tmo, abort_flag)) {
                    ++n_eld;
                    tc_fence_after();
                    const uint32_t idesc_phi = idesc_bf16_f32(128, R);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t ad = sdesc_sw128(smem_addr(X) + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                        const uint64_t bd = sdesc_sw128(smem_addr(Y) + (kk >> 2) * (R * 128) + (kk & 3) * 32, 16, 1024);
                        umma_ss(tPhi, ad, bd, idesc_phi, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(bar_emm);
                    ++n_emm_issued;
                } else {
                    fail();
                }
            }
            bool ok = mbar_wait(bar_emm, n_emm & 1, tmo, abort_flag);
            if (group_sync_or(!ok)) {
                if (tid == 0) fail();
            } else {
                ++n_emm;
                tc_fence_after();
                if (!z_early && tid == 0) {  // the feature product has finished with Y
                    mbar_expect_tx(bar_ez, sb_bytes(0));
                    bulk_load(Z, sb_head, sb_bytes(0), bar_ez);
                    ++n_ez_issued;
                }
                const int n_tab = n < g.L ? n : g.L - 1;  // rows past the sequence: any valid table entry
                const int axis_t = token_axis_pos(n_tab, 0, g.H, g.W), axis_h = token_axis_pos(n_tab, 1, g.H, g.W),
                          axis_w = token_axis_pos(n_tab, 2, g.H, g.W);
                // This thread's 16 rotation pairs of a chunk: features [16hf, 16hf + 16) and
                // [32 + 16hf, 48 + 16hf) (so both warps of a lane group have work when rc <= 32).
                auto feat = [&](int t) { return t < 8 ? 16 * hf + 2 * t : 32 + 16 * hf + 2 * (t - 8); };
                // phi . z over all R features: the unrotated features (RoPE outside the activation), or
                // with the RoPE inside, the rotated-then-activated ones over this thread's pairs
                const float* zh = a.z + static_cast<size_t>(bh) * R;
                float den = 0.f;
                if (!inside) {
#pragma unroll
                    for (int c0 = hf * 32; c0 < 128; c0 += 64) {
                        if (c0 < R) {
                            uint32_t v[32];
                            tmem_ld32(tPhi + lane_base + c0, v);
                            tmem_ld_wait(v);
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (c0 + i < R) den = fmaf(phi_act(__uint_as_float(v[i]), act), __ldg(zh + c0 + i), den);
                        }
                    }
                } else {
                    for (int ch = 0; ch < nch; ++ch) {
                        const int rc = min(64, R - 64 * ch);
                        uint32_t va[16], vb[16];
                        tmem_ld16(tPhi + lane_base + 64 * ch + 16 * hf, va);
                        tmem_ld16(tPhi + lane_base + 64 * ch + 32 + 16 * hf, vb);
                        tmem_ld_wait(va);
                        reg_fence(vb);
#pragma unroll
                        for (int t = 0; t < 16; ++t) {
                            const int f = feat(t);
                            if (f < rc) {
                                const int2 pi = a.pair_info[32 * ch + f / 2];
                                const int ap = pi.x == 0 ? axis_t : (pi.x == 1 ? axis_h : axis_w);
                                const double2 cs = __ldg(a.tab + pi.y + ap);
                                const float cf = static_cast<float>(cs.x), sf = static_cast<float>(cs.y);
                                const float u0 = __uint_as_float(t < 8 ? va[2 * t] : vb[2 * (t - 8)]);
                                const float u1 = __uint_as_float(t < 8 ? va[2 * t + 1] : vb[2 * (t - 8) + 1]);
                                den = fmaf(phi_act(u0 * cf - u1 * sf, act), __ldg(zh + 64 * ch + f), den);
                                den = fmaf(phi_act(u0 * sf + u1 * cf, act), __ldg(zh + 64 * ch + f + 1), den);
                            }
                        }
                    }
                }
                float gpart = 0.f;
                if (gated) {
                    // Wg . q over this thread's half of the raw query row, read from the tile in X
                    // (the tile's barrier has only one phase, long complete)
                    volatile int no_abort = 0;
                    mbar_wait(bar_eld, 0, tmo, &no_abort);
                    const float* gw = a.gate_w + hf * 64;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint4 raw =
                            *reinterpret_cast<const uint4*>(X + hf * 16384 + i_row * 128 + ((j ^ (i_row & 7)) << 4));
                        const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float2 qf = __bfloat1622float2(q2[u]);
                            gpart = fmaf(qf.x, __ldg(gw + 8 * j + 2 * u), gpart);
                            gpart = fmaf(qf.y, __ldg(gw + 8 * j + 2 * u + 1), gpart);
                        }
                    }
                    xch[256 + hf * 128 + i_row] = gpart;
                }
                xch[hf * 128 + i_row] = den;
                group_sync();
                den += xch[(hf ^ 1) * 128 + i_row];  // same total in both halves
                if (gated) glogit = a.gate_b + (gpart + xch[256 + (hf ^ 1) * 128 + i_row]);
                const float l_eff = keep > 0 ? l_run : 1.f;
                // summed into O (out = O / l): psi carries l; gated: the readout alone
                const float scale = (gated ? 1.f : l_eff) / (den + 1e-6f);
                for (int ch = 0; ch < nch && ok; ++ch) {
                    const int rc = min(64, R - 64 * ch);
                    if (ch > 0) {  // the previous chunk's product must have finished with X and Z
                        ok = mbar_wait(bar_emm, n_emm & 1, tmo, abort_flag);
                        if (group_sync_or(!ok)) {
                            if (tid == 0) fail();
                            ok = false;
                            break;
                        }
                        ++n_emm;
                        tc_fence_after();
                        if (tid == 0) {
                            mbar_expect_tx(bar_ez, sb_bytes(ch));
                            bulk_load(Z, sb_head + static_cast<size_t>(ch) * kSbChunkBytes, sb_bytes(ch), bar_ez);
                            ++n_ez_issued;
                        }
                    }
                    // This thread's 16 rotation pairs of the chunk (feat above).  Their (cos, sin) loads
                    // are all issued before any is used; the pair table holds all D/2 rotary pairs, so
                    // pairs past the rank are still valid entries (their results are not stored).  The
                    // pair -> (axis, table offset) map comes from the launch parameters.
                    float2 rot[16];
                    // the second eight lie past the rank when rc <= 32; no rotation without the low-rank RoPE
                    const int nrot = norope ? 0 : (rc > 32 ? 16 : 8);
                    {
                        double2 cs[16];
#pragma unroll
                        for (int t = 0; t < 16; ++t) {
                            if (t < nrot) {
                                const int2 pi = a.pair_info[32 * ch + feat(t) / 2];
                                const int ap = pi.x == 0 ? axis_t : (pi.x == 1 ? axis_h : axis_w);
                                cs[t] = __ldg(a.tab + pi.y + ap);
                            }
                        }
#pragma unroll
                        for (int t = 0; t < 16; ++t)
                            if (t < nrot) rot[t] = make_float2(static_cast<float>(cs[t].x), static_cast<float>(cs[t].y));
                    }
                    uint32_t va[16], vb[16];
                    tmem_ld16(tPhi + lane_base + 64 * ch + 16 * hf, va);
                    tmem_ld16(tPhi + lane_base + 64 * ch + 32 + 16 * hf, vb);
                    tmem_ld_wait(va);
                    reg_fence(vb);
#pragma unroll
                    for (int t = 0; t < 16; ++t) {
                        const int f = feat(t);
                        const int pp = f / 2;
                        if (f < rc) {
                            const uint32_t u0 = t < 8 ? va[2 * t] : vb[2 * (t - 8)];
                            const uint32_t u1 = t < 8 ? va[2 * t + 1] : vb[2 * (t - 8) + 1];
                            // outside: activation, then rotation; inside: rotation, then activation
                            const float x0 = inside ? __uint_as_float(u0) : phi_act(__uint_as_float(u0), act);
                            const float x1 = inside ? __uint_as_float(u1) : phi_act(__uint_as_float(u1), act);
                            const float cf = norope ? 1.f : rot[t].x, sf = norope ? 0.f : rot[t].y;
                            float r0 = x0 * cf - x1 * sf, r1 = x0 * sf + x1 * cf;
                            if (inside) {
                                r0 = phi_act(r0, act);
                                r1 = phi_act(r1, act);
                            }
                            const float y0 = r0 * scale, y1 = r1 * scale;
                            const __nv_bfloat162 hi = __floats2bfloat162_rn(y0, y1);
                            const float2 hf2 = __bfloat1622float2(hi);
                            const __nv_bfloat162 lo = __floats2bfloat162_rn(y0 - hf2.x, y1 - hf2.y);
                            const uint32_t hb = *reinterpret_cast<const uint32_t*>(&hi);
                            const uint32_t lb = *reinterpret_cast<const uint32_t*>(&lo);
                            *reinterpret_cast<uint32_t*>(X + sw128_offset(i_row, 2 * pp, 128)) = hb;
                            *reinterpret_cast<uint32_t*>(X + sw128_offset(i_row, rc + 2 * pp, 128)) = hb;
                            *reinterpret_cast<uint32_t*>(X + sw128_offset(i_row, 2 * rc + 2 * pp, 128)) = lb;
                        }
                    }
                    fence_async_smem();
                    tc_fence_before();
                    group_sync();
                    if (tid == 0 && !*abort_flag) {
                        if (mbar_wait(bar_ez, n_ez & 1, tmo, abort_flag)) {
                            ++n_ez;
                            tc_fence_after();
                            const uint32_t idesc_lr = idesc_bf16_f32(128, D);
                            for (int kk = 0; kk < (3 * rc) / 16; ++kk) {
                                const uint64_t ad = sdesc_sw128(smem_addr(X) + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                                const uint64_t bd = sdesc_sw128(smem_addr(Z) + (kk >> 2) * (D * 128) + (kk & 3) * 32, 16, 1024);
                                const bool acc = gated ? (ch > 0 || kk > 0) : (keep > 0 || ch > 0 || kk > 0);
                                umma_ss(gated ? tLr : tO, ad, bd, idesc_lr, acc ? 1u : 0u);
                            }
                            umma_commit(bar_emm);
                            ++n_emm_issued;
                        } else {
                            fail();
                        }
                    }
                }
                if (ok) {
                    ok = !*abort_flag && mbar_wait(bar_emm, n_emm & 1, tmo, abort_flag);
                    if (group_sync_or(!ok)) {
                        if (tid == 0) fail();
                    } else {
                        ++n_emm;
                        tc_fence_after();
                        if (gated) {
                            lr_live = true;
                        } else {
                            inv_l = 1.f / l_eff;
                            o_live = true;
                        }
                    }
                }
            }
        }
    }
    // head_dim 64: CUDA-core readout; both warps of a lane group compute the row's features and each
    // accumulates its half of the output columns.
    constexpr int DH = D / 2;
    float acc[D == 128 ? 1 : DH];
    float inv_den = 0.f;
    if constexpr (D != 128) {
#pragma unroll
        for (int e = 0; e < DH; ++e) acc[e] = 0.f;
        if (a.lowrank && !aborted) {
            float* As = reinterpret_cast<float*>(smem);  // [D][R] fp32, reuses the tile buffers
            const __nv_bfloat16* Ah = a.A + static_cast<size_t>(h) * g.a_stride;  // this head's query projection
            for (int e = tid; e < D * g.R; e += kSoftThreads) As[e] = __bfloat162float(Ah[e]);
            group_sync();
            if (row_valid) {
                const __nv_bfloat16* qrow = a.q_raw + g.sq.row(b, n, h);
                const float* Sh = a.S + static_cast<size_t>(bh) * g.R * D + hf * DH;
                const float* zh = a.z + static_cast<size_t>(bh) * g.R;
                float den = 0.f;
                for (int c0 = 0; c0 < g.R; c0 += 16) {
                    float phi[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) phi[c] = 0.f;
                    for (int d0 = 0; d0 < D; d0 += 8) {
                        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(qrow + d0));
                        const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float2 qf = __bfloat1622float2(q2[u]);
                            if (gated && c0 == 0) {  // Wg . q (both threads of the row compute all of it)
                                glogit = fmaf(qf.x, __ldg(a.gate_w + d0 + 2 * u), glogit);
                                glogit = fmaf(qf.y, __ldg(a.gate_w + d0 + 2 * u + 1), glogit);
                            }
                            const float* a0 = As + (d0 + 2 * u) * g.R + c0;
                            const float* a1 = a0 + g.R;
#pragma unroll
                            for (int c = 0; c < 16; ++c) phi[c] = fmaf(qf.y, a1[c], fmaf(qf.x, a0[c], phi[c]));
                        }
                    }
                    // outside: activation (the normaliser's features), then rotation; inside: rotation,
                    // then activation, and the normaliser uses the result
                    if (!inside) {
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            phi[c] = phi_act(phi[c], act);
                            den = fmaf(phi[c], __ldg(zh + c0 + c), den);
                        }
                    }
#pragma unroll
                    for (int pp = 0; pp < 8; ++pp) {
                        if (norope) break;
                        const int2 pi = __ldg(a.pairs + (c0 >> 1) + pp);  // (axis, table offset)
                        const double2 cs = __ldg(a.tab + pi.y + token_axis_pos(n, pi.x, g.H, g.W));
                        const float cf = static_cast<float>(cs.x), sf = static_cast<float>(cs.y);
                        const float x0 = phi[2 * pp], x1 = phi[2 * pp + 1];
                        phi[2 * pp] = x0 * cf - x1 * sf;
                        phi[2 * pp + 1] = x0 * sf + x1 * cf;
                    }
                    if (inside) {
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            phi[c] = phi_act(phi[c], act);
                            den = fmaf(phi[c], __ldg(zh + c0 + c), den);
                        }
                    }
#pragma unroll 4
                    for (int c = 0; c < 16; ++c) {
                        const float4* s4 = reinterpret_cast<const float4*>(Sh + (c0 + c) * D);
#pragma unroll
                        for (int e4 = 0; e4 < DH / 4; ++e4) {
                            const float4 sv4 = __ldg(s4 + e4);
                            acc[4 * e4 + 0] = fmaf(phi[c], sv4.x, acc[4 * e4 + 0]);
                            acc[4 * e4 + 1] = fmaf(phi[c], sv4.y, acc[4 * e4 + 1]);
                            acc[4 * e4 + 2] = fmaf(phi[c], sv4.z, acc[4 * e4 + 2]);
                            acc[4 * e4 + 3] = fmaf(phi[c], sv4.w, acc[4 * e4 + 3]);
                        }
                    }
                }
                inv_den = 1.f / (den + 1e-6f);
                glogit += a.gate_b;
            }
            lr_live = true;
        }
    }
    // ---- out = O / l (+ the CUDA-core readout for head_dim 64): each thread writes its half of its
    //      row into a 128-B-swizzled staging tile (conflict-free 16-byte stores), then 64-row TMA stores
    //      write it out; tokens past L are clipped by the tensor map and a 64-token block's second half
    //      is skipped.
    const bool aborted2 = group_sync_or(*abort_flag != 0);  // every product that read the tile buffers has completed
    if (!aborted2) {
        // this thread's 32-column group cc of O (and, gated with head_dim 128, of the readout)
        auto load_group = [&](int cc, uint32_t (&o)[32], uint32_t (&lr)[32]) {
            const int c = hf * (D / 64) + cc;
            if (o_live) tmem_ld32(tO + lane_base + c * 32, o);
            if (D == 128 && gated && lr_live) tmem_ld32(tLr + lane_base + c * 32, lr);
            if (o_live || (D == 128 && gated && lr_live)) {
                tmem_ld_wait(o);
                reg_fence(lr);
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if (!o_live) o[i] = 0u;
                if (D != 128 || !gated || !lr_live) lr[i] = 0u;
            }
        };
        auto lr_value = [&](int cc, int i, const uint32_t (&lr)[32]) -> float {
            if constexpr (D == 128) return __uint_as_float(lr[i]);
            else return acc[cc * 32 + i] * inv_den;
        };
        float gfac = 0.f;  // gated: g * rms(O_s) / sqrt(mean(O_lr^2) + 1e-6) of this row
        if (gated) {
            float ss_s = 0.f, ss_l = 0.f;  // this thread's half of the two sums of squares
#pragma unroll
            for (int cc = 0; cc < D / 64; ++cc) {
                uint32_t o[32], lr[32];
                load_group(cc, o, lr);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float xs = __uint_as_float(o[i]) * inv_l, xl = lr_value(cc, i, lr);
                    ss_s = fmaf(xs, xs, ss_s);
                    ss_l = fmaf(xl, xl, ss_l);
                }
            }
            xch[hf * 128 + i_row] = ss_s;
            xch[256 + hf * 128 + i_row] = ss_l;
            group_sync();
            ss_s += xch[(hf ^ 1) * 128 + i_row];
            ss_l += xch[256 + (hf ^ 1) * 128 + i_row];
            const float gsig = 1.f / (1.f + expf(-glogit));
            gfac = lr_live ? gsig * sqrtf(ss_s / D) / sqrtf(ss_l / D + 1e-6f) : 0.f;
        }
#pragma unroll
        for (int cc = 0; cc < D / 64; ++cc) {
            const int c = hf * (D / 64) + cc;  // 32-column group of O
            uint32_t o[32], lr[32];
            load_group(cc, o, lr);
            float r[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                float x = __uint_as_float(o[i]) * inv_l;
                if (gated) {
                    x = fmaf(gfac, lr_value(cc, i, lr), x);
                } else {
                    if constexpr (D != 128) x += acc[cc * 32 + i] * inv_den;
                }
                r[i] = x;
            }
            if (a.out_bf16) {  // boxes of 64 columns
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int col = c * 32 + 8 * u;
                    uint4 pk;
                    __nv_bfloat162 t0 = __floats2bfloat162_rn(r[8 * u], r[8 * u + 1]);
                    __nv_bfloat162 t1 = __floats2bfloat162_rn(r[8 * u + 2], r[8 * u + 3]);
                    __nv_bfloat162 t2 = __floats2bfloat162_rn(r[8 * u + 4], r[8 * u + 5]);
                    __nv_bfloat162 t3 = __floats2bfloat162_rn(r[8 * u + 6], r[8 * u + 7]);
                    pk.x = *reinterpret_cast<uint32_t*>(&t0);
                    pk.y = *reinterpret_cast<uint32_t*>(&t1);
                    pk.z = *reinterpret_cast<uint32_t*>(&t2);
                    pk.w = *reinterpret_cast<uint32_t*>(&t3);
                    *reinterpret_cast<uint4*>(smem + sw128_offset(i_row, col, 128)) = pk;
                }
            } else {  // boxes of 32 columns: box c holds columns [32c, 32c + 32)
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint32_t off = c * 16384 + i_row * 128 + (((u ^ (i_row & 7))) << 4);
                    *reinterpret_cast<float4*>(smem + off) = make_float4(r[4 * u], r[4 * u + 1], r[4 * u + 2], r[4 * u + 3]);
                }
            }
        }
        fence_async_smem();
        group_sync();
        if (tid == 0) {
            const int cols_per_box = a.out_bf16 ? 64 : 32;
            const int boxes = D / cols_per_box;
            for (int bx = 0; bx < boxes; ++bx)
                for (int rh = 0; rh * 64 < blk; ++rh) {
                    if (alpha * blk + rh * 64 >= g.L) break;
                    tma_store_4d(&tm_out, smem + bx * 16384 + rh * 64 * 128, bx * cols_per_box, h,
                                 alpha * blk + rh * 64, b);
                }
            tma_store_commit_and_wait();
        }
    }
    // ------------------------------------------------------------------ teardown (softmax warps)
    if (os_committed && aborted2) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    if (*abort_flag && tid == 0) {
        // Let the epilogue's copies and products still in flight land before the memory is released.
        // Each wait is bounded (10 ms) and ignores the abort flag.
        volatile int no_abort = 0;
        const uint64_t drain = 10000000ull;
        if (n_eld_issued > n_eld) mbar_wait(bar_eld, n_eld & 1, drain, &no_abort);
        if (n_ez_issued > n_ez) mbar_wait(bar_ez, n_ez & 1, drain, &no_abort);
        if (n_emm_issued > n_emm) mbar_wait(bar_emm, n_emm & 1, drain, &no_abort);
    }
    }  // softmax warps
    // ------------------------------------------------------------------ teardown (all warps)
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

size_t attn_smem_bytes(const Geom& g) {
    return (g.D == 128 ? AttnLayout<128>::kBytes : AttnLayout<64>::kBytes) + 1024;
}

namespace {
template <int D, int BLK, bool kDefault>
cudaError_t launch_attn_v(const AttnMaps& m, const AttnArgs& a, const Geom& g, cudaStream_t st) {
    const size_t sm = attn_smem_bytes(g);
    cudaError_t e = cudaFuncSetAttribute(attn_sm100_kernel<D, BLK, kDefault>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
    if (e != cudaSuccess) return e;
    attn_sm100_kernel<D, BLK, kDefault><<<dim3(g.nb, g.BH()), kThreads, sm, st>>>(m.q, m.k, m.v, m.q_raw, m.out,
                                                                                    m.os, a, g);
    return cudaGetLastError();
}
template <int D, int BLK>
cudaError_t launch_attn_t(const AttnMaps& m, const AttnArgs& a, const Geom& g, cudaStream_t st) {
    return (g.act == 0 && g.norope == 0 && g.inside == 0 && !a.gated) ? launch_attn_v<D, BLK, true>(m, a, g, st)
                                                                      : launch_attn_v<D, BLK, false>(m, a, g, st);
}
}  // namespace

cudaError_t launch_attn(const AttnMaps& m, const AttnArgs& a, const Geom& g, cudaStream_t st) {
    if (g.D == 128) return g.block == 128 ? launch_attn_t<128, 128>(m, a, g, st) : launch_attn_t<128, 64>(m, a, g, st);
    return g.block == 128 ? launch_attn_t<64, 128>(m, a, g, st) : launch_attn_t<64, 64>(m, a, g, st);
}

}  // namespace slra
