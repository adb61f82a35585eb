// Gradients of the low-rank branch on the sm_100a tensor cores (head_dim 128, rank <= 64): the
// derivative of RoLA "4.1"/"4.2"/"4.3"/"B.1"'s branch (default: phi = relu(x A), psi = R_r phi outside
// the activation, S = sum psi_k v^T, z = sum phi_k, O_lr = psi_q S / (phi_q . z + 1e-6)), and of its
// variants: the other feature maps, no low-rank RoPE, the RoPE inside the activation (psi = act(R_r x A),
// the normaliser on psi), separate and per-head projections.  Per rotation pair, lr_pair_fwd /
// lr_pair_bwd (common.cuh) give psi, the normaliser's feature nf and du for each of these.
//
// Persistent CTAs (one per SM, 256 threads: two per token row, each half of the features) walk work
// items = (head, range of 128-token tiles), like the forward summary kernel.  Per tile:
//   query pass  MMA  U = q A, G = dO S^T                                 (token rows in TMEM)
//               threads (row = TMEM lane): psi, nf, den = nf . z + 1e-6, dden = -(psi . G) / den^2,
//               du from dpsi = G / den and dnf = dden z, w = psi / den; dz += dden nf
//               MMA  dS^T += dO^T [w_hi | w_lo],  dA^T += q^T [du_hi | du_lo]   (accumulated over the
//                    item's tiles, d rows in TMEM),  dq = du A^T
//   key pass    MMA  U = k A, dpsi = v dS^T
//               threads: psi, du from dpsi and dnf = dz
//               MMA  dv = psi dS, dk = du A^T, dA^T += k^T [du_hi | du_lo] (accumulated)
// dq, dk, dv leave through shared memory and TMA: stored, or added to the sparse branch's rows.
// Operands that are not exact in bf16 (dO, S, dS, w, du, psi) are split into bf16 hi + lo (x = hi + lo
// to ~2^-16); products take hi*hi + hi*lo + lo*hi with fp32 accumulation.  The item's dS, dA and dz
// partial sums go to split-L buffers that a fixed-order reduction sums.
// All waits are bounded (sm100.cuh); a wait that runs out records a timeout and the CTA drains and exits.
#include "common.cuh"
#include "sm100.cuh"

namespace slra {

namespace {

constexpr int kTok = 128;                  // tokens per tile
constexpr int kD = 128;                    // head dimension
constexpr int kRp = 64;                    // features per hi / lo half of an operand image
constexpr int kTile = kTok * kD * 2;       // bf16 [128][128] in two 64-column slabs of 16 KB
constexpr int kSlab = kTok * 128;          // bytes of one 64-column slab of 128 rows

// instruction descriptor, bf16 A and B, fp32 accumulation, A / B K-major or MN-major
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((static_cast<uint32_t>(N) >> 3) << 17) | ((static_cast<uint32_t>(M) >> 4) << 24);
}

__device__ __forceinline__ uint16_t bf16_bits(float x) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    return *reinterpret_cast<const uint16_t*>(&h);
}
__device__ __forceinline__ float bf16_val(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

// x = hi + lo as two bf16 (hi = RNE(x), lo = RNE(x - hi))
__device__ __forceinline__ void split_bf16(float x, uint16_t& hi, uint16_t& lo) {
    hi = bf16_bits(x);
    lo = bf16_bits(x - bf16_val(hi));
}

// K-major operand [rows][K]: k-step kk (16 elements = 32 B) of a tile stored as 64-column slabs
__device__ __forceinline__ uint64_t kmaj(uint32_t base, int kk, int slab_bytes) {
    return sdesc_sw128(base + (kk >> 2) * slab_bytes + (kk & 3) * 32, 16, 1024);
}
// MN-major operand stored [K rows][MN] (MN contiguous, 64-column slabs of slab_bytes): k-step kk = 16 rows
__device__ __forceinline__ uint64_t mnmaj(uint32_t base, int kk, int slab_bytes) {
    return sdesc_sw128(base + kk * 2048, static_cast<uint32_t>(slab_bytes), 1024);
}

}  // namespace

struct LrTcBwdArgs {
    const float* dout;   // fp32 [B][L][Hh][D] (strides g.so)
    const float* S;      // query pass: S [BH][R][D]
    const float* z;      // query pass: z [BH][R]
    const float* dS;     // key pass: dS [BH][R][D]
    const float* dz;     // key pass: dz [BH][R]
    const __nv_bfloat16* A;  // [D][R]
    const double2* tab;
    int2 pair_info[kMaxPairs];
    float* dq;  // query pass output (plain stores)
    float* dk;  // key pass outputs
    float* dv;
    float* ds_part;  // [BH][nsplit][R][D]
    float* dz_part;  // [BH][nsplit][R]
    float* da_part;  // [BH][nsplit][D][R]
    int nsplit, tiles_per_split;
    int accumulate;  // 1: add dq (dk, dv) to the rows; 0: store them
    int* status;
    unsigned long long timeout_ns;
};

namespace {

// Shared-memory layout of both passes (1024-B aligned sections).
template <int R>
struct LbLayout {
    static constexpr int kAtImg = ((R * 256 + 1023) / 1024) * 1024;  // [R][128] K-major
    static constexpr int kOffX = 0;                                 // q or k tile
    static constexpr int kOffY = kTile;                             // query pass: dO hi; key pass: v
    static constexpr int kOffY2 = 2 * kTile;                        // query pass: dO lo; key pass: dS^T images
    static constexpr int kOffAt = 3 * kTile;  // A^T image [R][128]: B of x A (K-major), B of du A^T (MN-major)
    static constexpr int kOffSi = kOffAt + kAtImg;                  // S or dS images hi, lo: [R][128] each
    static constexpr int kOffW = kOffSi + 2 * kAtImg;               // [128][hi 64 | lo 64]: w or psi
    static constexpr int kOffDu = kOffW + kTile;                    // [128][hi 64 | lo 64]: du
    static constexpr int kOffXch = kOffDu + kTile;                  // [2][2][128] fp32 row partials
    static constexpr int kOffBar = kOffXch + 2048;
    static constexpr int kOffMisc = kOffBar + 64;
    static constexpr int kBytes = kOffMisc + 64;
};

// Build a K-major [rows = R][128] bf16 image of the transpose-free matrix M[c][d] (R x 128, fp32 or
// bf16 source), split into hi and lo images when `lo` is given.
template <int R>
__device__ __forceinline__ void build_rk_image(uint8_t* hi_img, uint8_t* lo_img, const float* src) {
    for (int e = threadIdx.x; e < R * kD; e += 256) {
        const int c = e / kD, d = e % kD;
        uint16_t hb, lb;
        split_bf16(src[e], hb, lb);
        *reinterpret_cast<uint16_t*>(hi_img + sw128_offset(c, d, R)) = hb;
        if (lo_img) *reinterpret_cast<uint16_t*>(lo_img + sw128_offset(c, d, R)) = lb;
    }
}

// Build a K-major [rows = 128 (d)][64 (c)] image of M[c][d] (the transpose of an R x 128 matrix):
// the B operand of a product over the features with N = 128.
template <int R>
__device__ __forceinline__ void build_dk_image(uint8_t* hi_img, uint8_t* lo_img, const float* src) {
    for (int e = threadIdx.x; e < R * kD; e += 256) {
        const int c = e / kD, d = e % kD;
        uint16_t hb, lb;
        split_bf16(src[e], hb, lb);
        *reinterpret_cast<uint16_t*>(hi_img + sw128_offset(d, c, kTok)) = hb;
        if (lo_img) *reinterpret_cast<uint16_t*>(lo_img + sw128_offset(d, c, kTok)) = lb;
    }
}

}  // namespace

// kKey = false: the query pass; true: the key pass.  kRelu: relu features with the RoPE outside the
// activation (the other feature maps' out-of-line code then drops out at compile time).
template <int R, bool kKey, bool kRelu>
__global__ void __launch_bounds__(256, 1)
    lr_bwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_y,
                        const __grid_constant__ CUtensorMap tm_o0, const __grid_constant__ CUtensorMap tm_o1,
                        LrTcBwdArgs a, Geom g) {
    using Lay = LbLayout<R>;
    constexpr int RH = R / 2;  // features per thread
    const int act = kRelu ? 0 : g.act, inside = kRelu ? 0 : g.inside;
    static_assert(R % 16 == 0 && R <= 64, "rank 16..64");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kOffBar);
    uint64_t* bar_ld = bars;       // the tile's TMA loads
    uint64_t* bar_m1 = bars + 1;   // first products
    uint64_t* bar_m2 = bars + 2;   // second products
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kOffMisc + 4);
    float* xch = reinterpret_cast<float*>(smem + Lay::kOffXch);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row = tid & 127, half = tid >> 7;
    const uint64_t tmo = a.timeout_ns;
    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(bars + i, 1);
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
    // TMEM (512 columns): U | G (query pass) or dpsi (key pass) at 0 | 64; query pass: dS^T (hi | lo) at
    // 128, dA^T (hi | lo) at 256, dq at 384; key pass: dA^T at 128, dv at 256, dk at 384
    const uint32_t tU = tmem, tG = tmem + 64, tDS = tmem + 128, tO = tmem + 384;
    const uint32_t tAcc = kKey ? tmem + 128 : tmem + 256;  // dA^T accumulator
    const uint32_t tV = tmem + 256, tK = tmem + 384;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t sx = smem_addr(smem + Lay::kOffX), sy = smem_addr(smem + Lay::kOffY),
                   sy2 = smem_addr(smem + Lay::kOffY2), sat = smem_addr(smem + Lay::kOffAt),
                   ssi = smem_addr(smem + Lay::kOffSi),
                   sw = smem_addr(smem + Lay::kOffW), sdu = smem_addr(smem + Lay::kOffDu);
    const uint32_t id_tok_r = idesc_bf16(128, R, false, false);     // [tokens x R], K = 128 dims
    const uint32_t id_acc = idesc_bf16(128, 2 * kRp, true, true);   // [dims x (hi|lo)], K = tokens
    const uint32_t id_tok_d = idesc_bf16(128, kD, false, false);    // [tokens x dims], K = features
    const uint32_t id_tok_dt = idesc_bf16(128, kD, false, true);    // the same with B = A^T read MN-major
    int n_ld = 0, n_m1 = 0, n_m2 = 0, n_ld_issued = 0, n_m1_issued = 0, n_m2_issued = 0;
    bool aborted = false;
    auto fail = [&]() {
        *abort_flag = 1;
        atomicOr(a.status, kDevTimeout);
    };
    const int ntiles = (g.L + kTok - 1) / kTok;
    const int n_items = g.BH() * a.nsplit;
    int staged_head = -1;  // head whose projection the A images hold
    for (int item = blockIdx.x; item < n_items && !aborted; item += gridDim.x) {
        const int bh = item / a.nsplit, split = item % a.nsplit;
        const int b = bh / g.Hh, h = bh % g.Hh;
        // A^T image [R][128] of this pass's projection (B of x A, and read MN-major the B of du A^T):
        // once when it is shared, again whenever the head changes when there is one per head
        if (staged_head < 0 || (g.a_stride != 0 && h != staged_head)) {
            const __nv_bfloat16* Ah = a.A + static_cast<size_t>(h) * g.a_stride;
            for (int e = tid; e < kD * R; e += 256) {
                const int d = e / R, c = e % R;
                const uint16_t bits = *reinterpret_cast<const uint16_t*>(Ah + e);
                *reinterpret_cast<uint16_t*>(smem + Lay::kOffAt + sw128_offset(c, d, R)) = bits;
            }
            staged_head = h;
        }
        const int t0 = split * a.tiles_per_split, t1 = min(ntiles, t0 + a.tiles_per_split);
        // this head's S (query pass) or dS (key pass) images; every product of the previous item has
        // completed (each tile waits for its second products) and all threads are past its end
        const float* M = (kKey ? a.dS : a.S) + static_cast<size_t>(bh) * R * kD;
        build_rk_image<R>(smem + Lay::kOffSi, smem + Lay::kOffSi + Lay::kAtImg, M);
        if (kKey) build_dk_image<R>(smem + Lay::kOffY2, smem + Lay::kOffY2 + kSlab, M);
        const float* zv = (kKey ? a.dz : a.z) + static_cast<size_t>(bh) * R;
        float zr[RH];
#pragma unroll
        for (int c = 0; c < RH; ++c) zr[c] = __ldg(zv + half * RH + c);
        float dzacc[RH];
#pragma unroll
        for (int c = 0; c < RH; ++c) dzacc[c] = 0.f;
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        for (int tile = t0; tile < t1 && !aborted; ++tile) {
            const int n = tile * kTok + row;
            const bool live = n < g.L;
            // ---- stage the tile: TMA for the bf16 inputs; the query pass splits dO into hi + lo itself
            if (tid == 0) {
                mbar_expect_tx(bar_ld, (kKey ? 2u : 1u) * kTile);
                for (int x = 0; x < 2; ++x) {
                    tma_load_4d(smem + Lay::kOffX + x * kSlab, &tm_x, bar_ld, x * 64, h, tile * kTok, b);
                    if (kKey) tma_load_4d(smem + Lay::kOffY + x * kSlab, &tm_y, bar_ld, x * 64, h, tile * kTok, b);
                }
                ++n_ld_issued;
                // the next tile's inputs towards L2 while this one is computed
                if (tile + 1 < t1)
                    for (int x = 0; x < 2; ++x) {
                        tma_prefetch_l2_4d(&tm_x, x * 64, h, (tile + 1) * kTok, b);
                        if (kKey) tma_prefetch_l2_4d(&tm_y, x * 64, h, (tile + 1) * kTok, b);
                    }
            }
            if (!kKey && tile + 1 < t1 && n + kTok < g.L) {  // and the next tile's dO rows
                const float* nxt = a.dout + g.so.row(b, n + kTok, h) + half * 64;
                asm volatile("prefetch.global.L2 [%0];" ::"l"(nxt));
                asm volatile("prefetch.global.L2 [%0];" ::"l"(nxt + 32));
            }
            if constexpr (!kKey) {
                const float* src = a.dout + g.so.row(b, live ? n : 0, h) + half * 64;
#pragma unroll 4
                for (int c = 0; c < 64; c += 4) {
                    const float4 x4 = live ? *reinterpret_cast<const float4*>(src + c) : make_float4(0.f, 0.f, 0.f, 0.f);
                    const float xv[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
                    for (int u = 0; u < 4; u += 2) {
                        uint16_t h0, l0, h1, l1;
                        split_bf16(xv[u], h0, l0);
                        split_bf16(xv[u + 1], h1, l1);
                        const uint32_t off = sw128_offset(row, half * 64 + c + u, kTok);
                        *reinterpret_cast<uint32_t*>(smem + Lay::kOffY + off) = h0 | (static_cast<uint32_t>(h1) << 16);
                        *reinterpret_cast<uint32_t*>(smem + Lay::kOffY2 + off) = l0 | (static_cast<uint32_t>(l1) << 16);
                    }
                }
                fence_async_smem();
            }
            // the rows this tile's outputs are added to, brought towards L2 while the tile is computed
            if (a.accumulate && live) {
                const size_t r0 = g.so.row(b, n, h) + half * 64;
#pragma unroll
                for (int which = 0; which < (kKey ? 2 : 1); ++which) {
                    const float* rowp = (kKey ? (which ? a.dk : a.dv) : a.dq) + r0;
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(rowp));
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(rowp + 32));
                }
            }
            // (cos, sin) of this row's pairs, loaded while the tile lands
            const int nt = live ? n : 0;
            const int pos_t = nt / (g.H * g.W), pos_h = (nt / g.W) % g.H, pos_w = nt % g.W;
            float cf[RH / 2], sf[RH / 2];
#pragma unroll
            for (int pp = 0; pp < RH / 2; ++pp) {
                const int2 pi = a.pair_info[half * (RH / 2) + pp];
                const double2 cs = g.norope ? make_double2(1.0, 0.0)
                                            : __ldg(a.tab + pi.y + (pi.x == 0 ? pos_t : (pi.x == 1 ? pos_h : pos_w)));
                cf[pp] = static_cast<float>(cs.x);
                sf[pp] = static_cast<float>(cs.y);
            }
            tc_fence_before();
            __syncthreads();
            // ---- first products
            if (tid == 0 && !*abort_flag) {
                if (mbar_wait(bar_ld, n_ld & 1, tmo, abort_flag)) {
                    ++n_ld;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk)  // U = x A
                        umma_ss(tU, kmaj(sx, kk, kSlab), kmaj(sat, kk, R * 128), id_tok_r, kk > 0 ? 1u : 0u);
                    if constexpr (!kKey) {  // G = dO S^T: hi*hi + hi*lo + lo*hi
#pragma unroll
                        for (int kk = 0; kk < kD / 16; ++kk)
                            umma_ss(tG, kmaj(sy, kk, kSlab), kmaj(ssi, kk, R * 128), id_tok_r, kk > 0 ? 1u : 0u);
#pragma unroll
                        for (int kk = 0; kk < kD / 16; ++kk)
                            umma_ss(tG, kmaj(sy, kk, kSlab), kmaj(ssi + Lay::kAtImg, kk, R * 128), id_tok_r, 1u);
#pragma unroll
                        for (int kk = 0; kk < kD / 16; ++kk)
                            umma_ss(tG, kmaj(sy2, kk, kSlab), kmaj(ssi, kk, R * 128), id_tok_r, 1u);
                    } else {  // dpsi = v dS^T: v exact, dS hi + lo
#pragma unroll
                        for (int kk = 0; kk < kD / 16; ++kk)
                            umma_ss(tG, kmaj(sy, kk, kSlab), kmaj(ssi, kk, R * 128), id_tok_r, kk > 0 ? 1u : 0u);
#pragma unroll
                        for (int kk = 0; kk < kD / 16; ++kk)
                            umma_ss(tG, kmaj(sy, kk, kSlab), kmaj(ssi + Lay::kAtImg, kk, R * 128), id_tok_r, 1u);
                    }
                    umma_commit(bar_m1);
                    ++n_m1_issued;
                } else {
                    fail();
                }
            }
            bool ok = mbar_wait(bar_m1, n_m1 & 1, tmo, abort_flag);
            if (__syncthreads_or(!ok)) {
                if (tid == 0) fail();
                aborted = true;
                break;
            }
            ++n_m1;
            tc_fence_after();
            // ---- per-token work: this thread's RH features [half*RH, half*RH + RH)
            float u[RH], gv[RH];
            {
                uint32_t r1[32], r2[32];  // windows past R read unused (in-range) TMEM columns
                tmem_ld32(tU + lane_base + half * RH, r1);
                tmem_ld32(tG + lane_base + half * RH, r2);
                tmem_ld_wait(r1);
                reg_fence(r2);
#pragma unroll
                for (int c = 0; c < RH; ++c) {
                    u[c] = __uint_as_float(r1[c]);
                    gv[c] = __uint_as_float(r2[c]);
                }
            }
            // psi, the normaliser feature nf and du per rotation pair (lr_pair_fwd / lr_pair_bwd: every
            // feature map and RoPE ordering); the pair's forward is recomputed where it is needed again
            float du[RH], w[RH];
            if constexpr (!kKey) {
                float den_p = 0.f, dot_p = 0.f;
#pragma unroll
                for (int pp = 0; pp < RH / 2; ++pp) {
                    const LrPair P = lr_pair_fwd(u[2 * pp], u[2 * pp + 1], cf[pp], sf[pp], act, inside);
                    den_p = fmaf(P.nf0, zr[2 * pp], fmaf(P.nf1, zr[2 * pp + 1], den_p));
                    dot_p = fmaf(P.psi0, gv[2 * pp], fmaf(P.psi1, gv[2 * pp + 1], dot_p));
                }
                xch[(0 * 2 + half) * 128 + row] = den_p;
                xch[(1 * 2 + half) * 128 + row] = dot_p;
                __syncthreads();
                const float den = (xch[(0 * 2 + 0) * 128 + row] + xch[(0 * 2 + 1) * 128 + row]) + 1e-6f;
                const float dot = xch[(1 * 2 + 0) * 128 + row] + xch[(1 * 2 + 1) * 128 + row];
                const float dden = live ? -dot / (den * den) : 0.f;
#pragma unroll
                for (int pp = 0; pp < RH / 2; ++pp) {
                    const LrPair P = lr_pair_fwd(u[2 * pp], u[2 * pp + 1], cf[pp], sf[pp], act, inside);
                    float du0, du1;
                    lr_pair_bwd(P, gv[2 * pp] / den, gv[2 * pp + 1] / den, dden * zr[2 * pp], dden * zr[2 * pp + 1],
                                cf[pp], sf[pp], inside, du0, du1);
                    du[2 * pp] = live ? du0 : 0.f;
                    du[2 * pp + 1] = live ? du1 : 0.f;
                    w[2 * pp] = live ? P.psi0 / den : 0.f;
                    w[2 * pp + 1] = live ? P.psi1 / den : 0.f;
                    dzacc[2 * pp] = fmaf(dden, P.nf0, dzacc[2 * pp]);
                    dzacc[2 * pp + 1] = fmaf(dden, P.nf1, dzacc[2 * pp + 1]);
                }
            } else {
#pragma unroll
                for (int pp = 0; pp < RH / 2; ++pp) {
                    const LrPair P = lr_pair_fwd(u[2 * pp], u[2 * pp + 1], cf[pp], sf[pp], act, inside);
                    w[2 * pp] = live ? P.psi0 : 0.f;  // psi, the A operand of dv
                    w[2 * pp + 1] = live ? P.psi1 : 0.f;
                    float du0, du1;
                    lr_pair_bwd(P, gv[2 * pp], gv[2 * pp + 1], zr[2 * pp], zr[2 * pp + 1], cf[pp], sf[pp], inside,
                                du0, du1);
                    du[2 * pp] = live ? du0 : 0.f;
                    du[2 * pp + 1] = live ? du1 : 0.f;
                }
            }
            // w (psi / den, or psi) and du as bf16 hi | lo operand tiles [128 tokens][hi 64 | lo 64]
#pragma unroll
            for (int c = 0; c < RH; c += 2) {
                const int col = half * RH + c;
                uint16_t wh0, wl0, wh1, wl1, uh0, ul0, uh1, ul1;
                split_bf16(w[c], wh0, wl0);
                split_bf16(w[c + 1], wh1, wl1);
                split_bf16(du[c], uh0, ul0);
                split_bf16(du[c + 1], uh1, ul1);
                *reinterpret_cast<uint32_t*>(smem + Lay::kOffW + sw128_offset(row, col, kTok)) = wh0 | (uint32_t(wh1) << 16);
                *reinterpret_cast<uint32_t*>(smem + Lay::kOffW + sw128_offset(row, kRp + col, kTok)) = wl0 | (uint32_t(wl1) << 16);
                *reinterpret_cast<uint32_t*>(smem + Lay::kOffDu + sw128_offset(row, col, kTok)) = uh0 | (uint32_t(uh1) << 16);
                *reinterpret_cast<uint32_t*>(smem + Lay::kOffDu + sw128_offset(row, kRp + col, kTok)) = ul0 | (uint32_t(ul1) << 16);
            }
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            // ---- second products
            if (tid == 0 && !*abort_flag) {
                tc_fence_after();
                const bool first = tile == t0;
                if constexpr (!kKey) {
                    // dS^T += dO^T [w_hi | w_lo] (dO hi, then lo)
#pragma unroll
                    for (int kk = 0; kk < kTok / 16; ++kk)
                        umma_ss(tDS, mnmaj(sy, kk, kSlab), mnmaj(sw, kk, kSlab), id_acc, (!first || kk > 0) ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < kTok / 16; ++kk)
                        umma_ss(tDS, mnmaj(sy2, kk, kSlab), mnmaj(sw, kk, kSlab), id_acc, 1u);
                    // dq = du A^T: du hi, then lo (K = R features)
#pragma unroll
                    for (int kk = 0; kk < R / 16; ++kk)
                        umma_ss(tO, kmaj(sdu, kk, kSlab), mnmaj(sat, kk, R * 128), id_tok_dt, kk > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < R / 16; ++kk)
                        umma_ss(tO, kmaj(sdu + kSlab, kk, kSlab), mnmaj(sat, kk, R * 128), id_tok_dt, 1u);
                } else {
                    const uint32_t sdst = sy2;  // dS^T images hi, lo: [128][64] K-major each
                    // dv = psi dS: psi_hi dS_hi + psi_hi dS_lo + psi_lo dS_hi
#pragma unroll
                    for (int kk = 0; kk < R / 16; ++kk)
                        umma_ss(tV, kmaj(sw, kk, kSlab), kmaj(sdst, kk, kSlab), id_tok_d, kk > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < R / 16; ++kk)
                        umma_ss(tV, kmaj(sw, kk, kSlab), kmaj(sdst + kSlab, kk, kSlab), id_tok_d, 1u);
#pragma unroll
                    for (int kk = 0; kk < R / 16; ++kk)
                        umma_ss(tV, kmaj(sw + kSlab, kk, kSlab), kmaj(sdst, kk, kSlab), id_tok_d, 1u);
                    // dk = du A^T
#pragma unroll
                    for (int kk = 0; kk < R / 16; ++kk)
                        umma_ss(tK, kmaj(sdu, kk, kSlab), mnmaj(sat, kk, R * 128), id_tok_dt, kk > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < R / 16; ++kk)
                        umma_ss(tK, kmaj(sdu + kSlab, kk, kSlab), mnmaj(sat, kk, R * 128), id_tok_dt, 1u);
                }
                // dA^T += x^T [du_hi | du_lo]
#pragma unroll
                for (int kk = 0; kk < kTok / 16; ++kk)
                    umma_ss(tAcc, mnmaj(sx, kk, kSlab), mnmaj(sdu, kk, kSlab), id_acc, (!first || kk > 0) ? 1u : 0u);
                umma_commit(bar_m2);
                ++n_m2_issued;
            }
            ok = mbar_wait(bar_m2, n_m2 & 1, tmo, abort_flag);
            if (__syncthreads_or(!ok)) {
                if (tid == 0) fail();
                aborted = true;
                break;
            }
            ++n_m2;
            tc_fence_after();
            // ---- outputs of the tile: this thread's 64 columns of the row (query pass: dq; key: dv, dk),
            // staged as fp32 boxes of 32 columns (128-B swizzled, the output map's layout) in tile buffers
            // the products are done with (dq, dv: w and du; dk: the k and v tiles), then stored by the
            // TMA engine, or with `accumulate` added to the rows in memory (one add per element, in L2).
            // The TMEM loads are warp-collective, so every lane takes them; the maps clip rows past L.
#pragma unroll
            for (int which = 0; which < (kKey ? 2 : 1); ++which) {
                const uint32_t src = kKey ? (which ? tK : tV) : tO;
                uint8_t* stg = smem + (which ? Lay::kOffX : Lay::kOffW);
#pragma unroll
                for (int c0 = 0; c0 < 64; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld32(src + lane_base + half * 64 + c0, r);
                    tmem_ld_wait(r);
                    uint8_t* box = stg + (half * 2 + c0 / 32) * 16384 + row * 128;
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        *reinterpret_cast<float4*>(box + ((u ^ (row & 7)) << 4)) =
                            make_float4(__uint_as_float(r[4 * u]), __uint_as_float(r[4 * u + 1]),
                                        __uint_as_float(r[4 * u + 2]), __uint_as_float(r[4 * u + 3]));
                }
            }
            fence_async_smem();
            __syncthreads();
            if (tid == 0) {
#pragma unroll
                for (int which = 0; which < (kKey ? 2 : 1); ++which) {
                    const CUtensorMap* map = which ? &tm_o1 : &tm_o0;
                    const uint8_t* stg = smem + (which ? Lay::kOffX : Lay::kOffW);
                    for (int bx = 0; bx < 4; ++bx)
                        for (int rh = 0; rh < 2; ++rh) {
                            const int n0 = tile * kTok + rh * 64;
                            if (n0 >= g.L) break;
                            if (a.accumulate) tma_reduce_add_4d(map, stg + bx * 16384 + rh * 8192, bx * 32, h, n0, b);
                            else tma_store_4d(map, stg + bx * 16384 + rh * 8192, bx * 32, h, n0, b);
                        }
                }
                tma_store_commit_and_wait();  // the next tile's loads and operands reuse the staging
            }
            tc_fence_before();
            __syncthreads();  // the next tile overwrites the staged operands and the token-row TMEM
            tc_fence_after();
        }
        if (aborted) break;
        // ---- item done: dS (query pass) and dA partial sums from TMEM (d rows), dz from the threads
        const size_t slot = static_cast<size_t>(bh) * a.nsplit + split;
        if (t1 > t0) {
            // row = d (TMEM lane), this thread's features [half*RH, +RH): hi at column c, lo at kRp + c
#pragma unroll
            for (int which = 0; which < (kKey ? 1 : 2); ++which) {
                const uint32_t src = (kKey || which == 1) ? tAcc : tDS;
                uint32_t rh[32], rl[32];
                tmem_ld32(src + lane_base + half * RH, rh);
                tmem_ld32(src + lane_base + kRp + half * RH, rl);
                tmem_ld_wait(rh);
                reg_fence(rl);
#pragma unroll
                for (int c = 0; c < RH; ++c) {
                    const float v = __uint_as_float(rh[c]) + __uint_as_float(rl[c]);
                    const int cc = half * RH + c;
                    if (!kKey && which == 0) a.ds_part[slot * R * kD + static_cast<size_t>(cc) * kD + row] = v;
                    else a.da_part[slot * kD * R + static_cast<size_t>(row) * R + cc] = v;
                }
            }
        } else {
            for (int e = tid; e < R * kD; e += 256) {
                if (!kKey) a.ds_part[slot * R * kD + e] = 0.f;
                a.da_part[slot * kD * R + e] = 0.f;
            }
        }
        if constexpr (!kKey) {
            // dz: the row partials summed over the 128 rows (warp shuffles, then the 4 warps of a half)
            float* zs = reinterpret_cast<float*>(smem + Lay::kOffXch);  // [8 warps][RH] (reuses xch)
            __syncthreads();
#pragma unroll
            for (int c = 0; c < RH; ++c) {
                float v = dzacc[c];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) zs[warp * RH + c] = v;
            }
            __syncthreads();
            if (tid < R) {
                const int hh = tid / RH, c = tid % RH;
                const float* p = zs + (4 * hh) * RH + c;
                a.dz_part[slot * R + tid] = ((p[0] + p[RH]) + p[2 * RH]) + p[3 * RH];
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (aborted && tid == 0) {  // let the copies and products in flight land (bounded, 10 ms each)
        volatile int no_abort = 0;
        if (n_ld_issued > n_ld) mbar_wait(bar_ld, n_ld & 1, 10000000ull, &no_abort);
        if (n_m1_issued > n_m1) mbar_wait(bar_m1, n_m1 & 1, 10000000ull, &no_abort);
        if (n_m2_issued > n_m2) mbar_wait(bar_m2, n_m2 & 1, 10000000ull, &no_abort);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

namespace {
template <int R, bool kRelu>
cudaError_t launch_lr_bwd_tc_r(const LrTcBwdArgs& a, const Geom& g, const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const CUtensorMap& tdq, const CUtensorMap& tdk,
                               const CUtensorMap& tdv, float* dS, float* dz, long long key_off, cudaStream_t st) {
    const size_t sm = static_cast<size_t>(LbLayout<R>::kBytes) + 1024;
    cudaError_t e = cudaFuncSetAttribute(lr_bwd_sm100_kernel<R, false, kRelu>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(lr_bwd_sm100_kernel<R, true, kRelu>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int items = g.BH() * a.nsplit;
    const int grid = items < sms ? items : sms;
    lr_bwd_sm100_kernel<R, false, kRelu><<<grid, 256, sm, st>>>(tq, tq, tdq, tdq, a, g);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = launch_lowrank_reduce(a.ds_part, a.dz_part, g, a.nsplit, dS, dz, nullptr, nullptr, nullptr, st)) !=
        cudaSuccess)
        return e;
    LrTcBwdArgs ak = a;
    ak.A = a.A + key_off;  // the key projection
    ak.dS = dS;
    ak.dz = dz;
    ak.da_part = a.da_part + static_cast<size_t>(g.BH()) * a.nsplit * kD * R;
    lr_bwd_sm100_kernel<R, true, kRelu><<<grid, 256, sm, st>>>(tk, tv, tdv, tdk, ak, g);
    return cudaGetLastError();
}
}  // namespace

// Tensor-core low-rank gradients (head_dim 128, rank <= 64): query pass, reduction of dS and dz, key
// pass.  The dA partials of both passes are left for the caller's fixed-order reduction.
cudaError_t launch_lr_bwd_tc(const LrBwdArgs& l, const Geom& g, cudaStream_t st) {
    const RopeMeta& meta = *l.meta;
    CUtensorMap tq, tk, tv, tdq, tdk, tdv;
    if (!make_map_tokens(&tq, l.q, g.B, g.L, g.Hh, g.D, g.sq, kTok) ||
        !make_map_tokens(&tk, l.k, g.B, g.L, g.Hh, g.D, g.sk, kTok) ||
        !make_map_tokens(&tv, l.v, g.B, g.L, g.Hh, g.D, g.sv, kTok) ||
        !make_map_out(&tdq, l.dq, g.B, g.L, g.Hh, g.D, g.so, true) ||
        !make_map_out(&tdk, l.dk, g.B, g.L, g.Hh, g.D, g.so, true) ||
        !make_map_out(&tdv, l.dv, g.B, g.L, g.Hh, g.D, g.so, true))
        return cudaErrorInvalidValue;
    LrTcBwdArgs a;
    a.dout = l.dout;
    a.S = l.S;
    a.z = l.z;
    a.dS = nullptr;
    a.dz = nullptr;
    a.A = l.A;
    a.tab = l.tab;
    for (int e = 0; e < kMaxPairs; ++e)
        a.pair_info[e] = e < meta.npairs ? make_int2(meta.axis[e], meta.tab_off[e]) : make_int2(0, 0);
    a.dq = l.dq;
    a.dk = l.dk;
    a.dv = l.dv;
    a.ds_part = l.ds_part;
    a.dz_part = l.dz_part;
    a.da_part = l.da_part;
    a.nsplit = l.nsplit;
    a.tiles_per_split = ((g.L + kTok - 1) / kTok + l.nsplit - 1) / l.nsplit;
    a.status = l.status;
    a.timeout_ns = l.timeout_ns;
    a.accumulate = l.accumulate;
    const bool relu = g.act == 0 && !g.inside;
    const long long koff = l.key_proj_offset(g);
    switch (g.R) {
        case 16:
            return relu ? launch_lr_bwd_tc_r<16, true>(a, g, tq, tk, tv, tdq, tdk, tdv, l.dS, l.dz, koff, st)
                        : launch_lr_bwd_tc_r<16, false>(a, g, tq, tk, tv, tdq, tdk, tdv, l.dS, l.dz, koff, st);
        case 32:
            return relu ? launch_lr_bwd_tc_r<32, true>(a, g, tq, tk, tv, tdq, tdk, tdv, l.dS, l.dz, koff, st)
                        : launch_lr_bwd_tc_r<32, false>(a, g, tq, tk, tv, tdq, tdk, tdv, l.dS, l.dz, koff, st);
        case 48:
            return relu ? launch_lr_bwd_tc_r<48, true>(a, g, tq, tk, tv, tdq, tdk, tdv, l.dS, l.dz, koff, st)
                        : launch_lr_bwd_tc_r<48, false>(a, g, tq, tk, tv, tdq, tdk, tdv, l.dS, l.dz, koff, st);
        case 64:
            return relu ? launch_lr_bwd_tc_r<64, true>(a, g, tq, tk, tv, tdq, tdk, tdv, l.dS, l.dz, koff, st)
                        : launch_lr_bwd_tc_r<64, false>(a, g, tq, tk, tv, tdq, tdk, tdv, l.dS, l.dz, koff, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace slra
