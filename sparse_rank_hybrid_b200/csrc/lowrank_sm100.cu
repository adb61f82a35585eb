// Low-rank summary on the sm_100a tensor cores (head_dim 128): per head, over all L keys,
//   S = sum_j psi(k_j) v_j^T,   z = sum_j phi(k_j),   phi(k) = act(k A) (relu by default), psi = phi with its first
// r coordinates rotated by the token's 3D RoPE angles (RoLA "4.1", "4.2", "4.3", "B.1").
//
// Persistent CTAs (one per SM, 256 threads: two threads per token row, each taking half of the
// features) walk work items = (head, range of 128-token tiles).  Per tile:
//   TMA    raw k and v tiles [128 tokens][128] bf16 straight from the [B][L][Hh][D] inputs (4D tensor
//          maps, 128-B swizzle, two stages so the next tiles stream in while this one is processed);
//   MMA    phi = k A  (M = 128 tokens, N = r, K = 128; A^T staged in shared memory as the B operand:
//          once per CTA when the projection is shared, again at each change of head when it is per head);
//   threads (thread = token = TMEM lane) apply the activation (relu unless another is chosen),
//          accumulate z in registers, rotate the first r coordinates (unless the low-rank RoPE is
//          off) and write psi as bf16 hi + lo halves (psi = hi + lo to ~2^-16) into shared memory,
//          token-major;
//   MMA    S^T += v^T [psi_hi | psi_lo]  (M = 128 = D, N = 2*Rp, K = 128 tokens), accumulated in TMEM
//          over the whole work item; v is exact in bf16, so S is exact to the fp32 accumulation.
// At the end of an item its S and z partial sums go to the split-L partial buffers, which a
// fixed-order reduction sums per head.
#include "common.cuh"
#include "sm100.cuh"

namespace slra {

namespace {

constexpr int kD = 128;
constexpr int kTok = 128;                      // tokens per tile
constexpr int kTileBytes = kTok * kD * 2;      // 32 KB (two 64-column slabs of 16 KB)
// k/v stages per CTA: rank <= 48 uses one stage (about 110 KB of shared memory) and 256 TMEM columns,
// so two CTAs share an SM and hide each other's latencies; larger ranks use two stages, one CTA per SM
// (rank 64's single-stage layout, 114 KB, would not fit twice).  TMEM: phi at column 0 (R columns), S^T
// at column 128 (2 RP columns).
template <int R>
struct LrCfg {
    static constexpr int kStages = R <= 48 ? 1 : 2;
    static constexpr int kTmemCols = R <= 64 ? 256 : 512;
    static constexpr int kCtasPerSm = R <= 48 ? 2 : 1;
};
constexpr int kMaxStages = 2;

struct LrLayout {
    int rp;           // padded psi width per half (64 or 128)
    int off_k[kMaxStages], off_v[kMaxStages];
    int off_at;       // A^T [r][128] bf16, K-major swizzled
    int off_psi;      // [128 tokens][2*rp] bf16, 64-column slabs
    int off_zred;     // [8 warps][R/2] fp32
    int off_bar;
    int off_misc;
    int bytes;
};

__host__ __device__ inline LrLayout lr_layout(int R, int stages) {
    LrLayout l;
    l.rp = R <= 64 ? 64 : 128;
    int o = 0;
    for (int s = 0; s < kMaxStages; ++s) l.off_k[s] = l.off_v[s] = 0;
    for (int s = 0; s < stages; ++s) { l.off_k[s] = o; o += kTileBytes; l.off_v[s] = o; o += kTileBytes; }
    l.off_at = o;
    o += ((R * 256 + 1023) / 1024) * 1024;
    l.off_psi = o;
    o += kTok * 2 * l.rp * 2;
    // R = 128 has no psi padding to preserve, so its z slots reuse the psi buffer (free at item end)
    l.off_zred = R == 128 ? l.off_psi : o;
    if (R != 128) o += 8 * (R / 2) * 4;
    l.off_bar = o;
    o += 128;
    l.off_misc = o;
    o += 64;
    l.bytes = o;
    return l;
}

}  // namespace

struct LrArgs {
    const __nv_bfloat16* A;
    const double2* tab;
    int2 pair_info[kMaxPairs];  // per rotary pair: (axis, offset of its cos/sin table), read through the
                                // constant cache
    float* s_part;   // [BH][nsplit][R][D]
    float* z_part;   // [BH][nsplit][R]
    int nsplit;
    int tiles_per_split;
    int* status;
    unsigned long long timeout_ns;
    int debug_unsatisfied_wait;  // test hook: wait on a barrier nothing signals before any work
};

// kDefault: relu features with the RoPE (the benchmark's configuration); the activation and no-RoPE
// branches then fold away at compile time.
template <int R, bool kDefault>
__global__ void __launch_bounds__(256, LrCfg<R>::kCtasPerSm)
    lowrank_sm100_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         LrArgs a, Geom g) {
    constexpr int kStages = LrCfg<R>::kStages;
    const LrLayout lay = lr_layout(R, kStages);
    const int act = kDefault ? 0 : g.act;
    const int norope = kDefault ? 0 : g.norope;
    const int inside = kDefault ? 0 : g.inside;  // RoPE before the activation; z then sums psi
    constexpr int RP = R <= 64 ? 64 : 128;
    constexpr int RH = R / 2;           // features per thread: two threads share a token row
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + lay.off_bar);
    uint64_t* bar_kv = bars;         // [kStages]: k and v tile of a stage landed
    uint64_t* bar_phi = bars + 2;    // phi MMA done (covers every earlier MMA)
    uint64_t* bar_s = bars + 3;      // S MMA done (covers every earlier MMA)
    uint64_t* bar_debug = bars + 4;  // test hook: nothing arrives here
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + lay.off_misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + lay.off_misc + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row = tid & 127;          // token row = TMEM lane
    const int half = tid >> 7;          // features [half*RH, half*RH + RH)
    const uint64_t tmo = a.timeout_ns;

    if (tid == 0) {
        for (int i = 0; i < 5; ++i) mbar_init(bars + i, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, LrCfg<R>::kTmemCols);
        tmem_relinquish();
    }
    const int ntiles = (g.L + kTok - 1) / kTok;
    const int n_items = g.BH() * a.nsplit;
    // The sequence of (item, tile) this CTA processes, flattened, so loads can run ahead.
    auto tile_of = [&](int q, int& item, int& tile) -> bool {  // q-th tile of this CTA
        int it = blockIdx.x;
        while (it < n_items) {
            const int split = it % a.nsplit;
            const int t0 = split * a.tiles_per_split, t1 = min(ntiles, t0 + a.tiles_per_split);
            const int cnt = max(0, t1 - t0);
            if (q < cnt) { item = it; tile = t0 + q; return true; }
            q -= cnt;
            it += gridDim.x;
        }
        return false;
    };
    auto head_of_tile = [&](int q) -> int {  // head of this CTA's q-th tile (-1 past the end)
        int item, tile;
        return tile_of(q, item, tile) ? (item / a.nsplit) % g.Hh : -1;
    };
    // A^T as the K-major B operand of phi = k A: row n = feature, 128 dims in two swizzled slabs; with
    // per-head projections, the matrix of head hd.
    auto build_at = [&](int hd) {
        const __nv_bfloat16* Ah = a.A + static_cast<size_t>(hd) * g.a_stride;
        for (int e = tid; e < R * kD; e += 256) {
            const int d = e / R, c = e % R;  // coalesced read of A [D][R]
            *reinterpret_cast<uint16_t*>(smem + lay.off_at + sw128_offset(c, d, R)) =
                *reinterpret_cast<const uint16_t*>(Ah + e);
        }
    };
    int h_loaded = g.a_stride ? max(0, head_of_tile(0)) : 0;  // head whose projection is staged
    build_at(h_loaded);
    // zero the padding columns of both psi halves once; tiles only ever write the first R of each half
    for (int e = tid; e < kTok * 2 * RP; e += 256) {
        const int t = e / (2 * RP), col = e % (2 * RP);
        if ((col % RP) >= R) *reinterpret_cast<uint16_t*>(smem + lay.off_psi + sw128_offset(t, col, kTok)) = 0;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_phi = tmem;          // R columns
    const uint32_t t_s = tmem + 128;      // 2*RP columns: S^T hi | lo
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t idesc_phi = idesc_bf16_f32(128, R);
    const uint32_t idesc_s = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                             ((uint32_t(2 * RP) >> 3) << 17) | ((128u >> 4) << 24);
    const uint32_t at_addr = smem_addr(smem + lay.off_at), psi_addr = smem_addr(smem + lay.off_psi);

    // thread 0's bookkeeping of issued / observed operations (for the bounded drain on abort)
    int n_load[kMaxStages] = {0, 0}, n_wait[kMaxStages] = {0, 0};
    int n_s_issued = 0, n_s_done = 0, n_phi_issued = 0;
    int q_total = 0;  // tiles this CTA will process
    {
        int it2, t2;
        while (tile_of(q_total, it2, t2)) ++q_total;
    }
    auto issue_load = [&](int q) {
        int item, tile;
        if (!tile_of(q, item, tile)) return;
        const int s = q % kStages;
        const int bh = item / a.nsplit, b = bh / g.Hh, h = bh % g.Hh;
        mbar_expect_tx(bar_kv + s, 2 * kTileBytes);
        for (int x = 0; x < 2; ++x) {
            tma_load_4d(smem + lay.off_k[s] + x * (kTileBytes / 2), &tm_k, bar_kv + s, x * 64, h, tile * kTok, b);
            tma_load_4d(smem + lay.off_v[s] + x * (kTileBytes / 2), &tm_v, bar_kv + s, x * 64, h, tile * kTok, b);
        }
        ++n_load[s];
    };
    auto fail = [&]() {
        *abort_flag = 1;
        atomicOr(a.status, kDevTimeout);
    };
    // phi_q = k_q A for the q-th tile (thread 0): wait for its k tile, issue, commit
    auto issue_phi = [&](int q) -> bool {
        const int s = q % kStages;
        if (!mbar_wait(bar_kv + s, n_wait[s] & 1, tmo, abort_flag)) return false;
        ++n_wait[s];
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(smem_addr(smem + lay.off_k[s]) + (kk >> 2) * (kTok * 128) + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(at_addr + (kk >> 2) * (R * 128) + (kk & 3) * 32, 16, 1024);
            umma_ss(t_phi, ad, bd, idesc_phi, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar_phi);
        ++n_phi_issued;
        return true;
    };
    // Test hook: a wait on a barrier that nothing arrives at runs out, records a timeout and raises the
    // abort flag before any copy or product has been issued; every thread then leaves the item loop.
    if (a.debug_unsatisfied_wait && tid == 0 && !mbar_wait(bar_debug, 0, tmo, abort_flag)) fail();
    __syncthreads();
    if (tid == 0 && !*abort_flag) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        for (int st = 0; st < kStages; ++st) issue_load(st);
        if (q_total > 0 && !issue_phi(0)) fail();
    }

    int q = 0;      // running tile count of this CTA (same in every thread)
    int n_phi = 0;  // phi MMAs observed complete (same in every thread)
    int n_s = 0;    // S MMAs issued (same in every thread)
    bool aborted = false;
    for (int item = blockIdx.x; item < n_items && !aborted; item += gridDim.x) {
        const int bh = item / a.nsplit, split = item % a.nsplit;
        const int t0 = split * a.tiles_per_split, t1 = min(ntiles, t0 + a.tiles_per_split);
        if (t1 <= t0) {  // empty split (the host plans avoid them): contributes zeros
            float* sp0 = a.s_part + (static_cast<size_t>(bh) * a.nsplit + split) * R * kD;
            for (int e = tid; e < R * kD; e += 256) sp0[e] = 0.f;
            if (tid < R) a.z_part[(static_cast<size_t>(bh) * a.nsplit + split) * R + tid] = 0.f;
            continue;
        }
        if (g.a_stride && bh % g.Hh != h_loaded) {
            // Another head's projection.  Its first phi product was held back (below), and every earlier
            // phi product has completed (each was waited for at its tile's start), so the A^T slot is
            // free; all threads are past the previous item's closing barrier.
            h_loaded = bh % g.Hh;
            build_at(h_loaded);
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            if (tid == 0 && !*abort_flag && !issue_phi(q)) fail();
        }
        float zacc[RH];
#pragma unroll
        for (int c = 0; c < RH; ++c) zacc[c] = 0.f;
        for (int tile = t0; tile < t1; ++tile, ++q) {
            const int s = q % kStages;
            // phi_q was issued by thread 0 (at the end of the previous tile, before the loop, or after a
            // change of head's projection at the item start); its
            // completion also means every earlier S product has finished with the psi buffer
            const bool ok = mbar_wait(bar_phi, n_phi & 1, tmo, abort_flag);
            if (__syncthreads_or(!ok)) {
                if (tid == 0) fail();
                aborted = true;
                break;
            }
            ++n_phi;
            tc_fence_after();
            // ---- activation, z, rotation, psi hi/lo into shared memory (two threads per token row)
            const int n = tile * kTok + row;
            const bool real = n < g.L;
            uint32_t raw[RH];
#pragma unroll
            for (int c0 = 0; c0 < RH; c0 += 32) {
                uint32_t r32[32];  // a window past RH reads unused (in-range) TMEM columns
                tmem_ld32(t_phi + lane_base + half * RH + c0, r32);
                tmem_ld_wait(r32);
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (c0 + i < RH) raw[c0 + i] = r32[i];
            }
            const int HW = g.H * g.W;
            const int nt = real ? n : 0;  // rows past the sequence: any valid table entry (unused)
            const int pos_t = nt / HW, pos_h = (nt / g.W) % g.H, pos_w = nt % g.W;
#pragma unroll
            for (int p0 = 0; p0 < RH / 2; p0 += 8) {
                // (cos, sin) of eight pairs, every load issued before any is used
                double2 cs[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (p0 + u < RH / 2) {
                        const int2 pi = a.pair_info[half * (RH / 2) + p0 + u];
                        cs[u] = norope ? make_double2(1.0, 0.0)
                                         : __ldg(a.tab + pi.y + (pi.x == 0 ? pos_t : (pi.x == 1 ? pos_h : pos_w)));
                    }
                }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int pp = p0 + u;
                if (pp >= RH / 2) break;
                const int p = half * (RH / 2) + pp;  // global rotary pair
                const float u0 = real ? __uint_as_float(raw[2 * pp]) : 0.f;
                const float u1 = real ? __uint_as_float(raw[2 * pp + 1]) : 0.f;
                float x0 = inside ? u0 : phi_act(u0, act), x1 = inside ? u1 : phi_act(u1, act);
                const float cf = static_cast<float>(cs[u].x), sf = static_cast<float>(cs[u].y);
                float y0 = x0 * cf - x1 * sf, y1 = x0 * sf + x1 * cf;
                if (inside) {  // rotate, then the activation; the normaliser sums these features
                    y0 = phi_act(y0, act);
                    y1 = phi_act(y1, act);
                    x0 = y0;
                    x1 = y1;
                }
                zacc[2 * pp] += x0;
                zacc[2 * pp + 1] += x1;
                const __nv_bfloat162 hi = __floats2bfloat162_rn(y0, y1);
                const float2 hf = __bfloat1622float2(hi);
                const __nv_bfloat162 lo = __floats2bfloat162_rn(y0 - hf.x, y1 - hf.y);
                *reinterpret_cast<__nv_bfloat162*>(smem + lay.off_psi + sw128_offset(row, 2 * p, kTok)) = hi;
                *reinterpret_cast<__nv_bfloat162*>(smem + lay.off_psi + sw128_offset(row, RP + 2 * p, kTok)) = lo;
            }
            }
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            // ---- S^T += v^T [psi_hi | psi_lo]; then phi of the next tile; then reload stage s
            if (tid == 0 && !*abort_flag) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kTok / 16; ++kk) {
                    const uint64_t ad = sdesc_sw128(smem_addr(smem + lay.off_v[s]) + kk * 2048, kTileBytes / 2, 1024);
                    const uint64_t bd = sdesc_sw128(psi_addr + kk * 2048, kTok * 128, 1024);
                    umma_ss(t_s, ad, bd, idesc_s, (tile > t0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(bar_s);
                ++n_s_issued;
                bool good = true;
                const bool next_phi = q + 1 < q_total && (!g.a_stride || head_of_tile(q + 1) == h_loaded);
                if constexpr (kStages > 1) {
                    // the next tile's phi product goes in right behind (its k tile is already loading),
                    // unless it needs another head's projection: then it is issued once that is staged
                    if (next_phi) good = issue_phi(q + 1);
                    // stage s is free once this S product is done: refill it with the tile two ahead
                    if (good && mbar_wait(bar_s, n_s_done & 1, tmo, abort_flag)) {
                        ++n_s_done;
                        issue_load(q + kStages);
                    } else {
                        fail();
                    }
                } else {
                    // one stage: the next tile loads once this S product is done with v, then its phi
                    // product follows (the other CTA on the SM works meanwhile)
                    if (mbar_wait(bar_s, n_s_done & 1, tmo, abort_flag)) {
                        ++n_s_done;
                        issue_load(q + 1);
                        if (next_phi) good = issue_phi(q + 1);
                        if (!good) fail();
                    } else {
                        fail();
                    }
                }
            }
            ++n_s;
        }
        if (aborted) break;
        // ---- item done: S^T (lane = e, columns = c for hi and lo) and z to the partial buffers
        const bool ok = mbar_wait(bar_s, (n_s - 1) & 1, tmo, abort_flag);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) fail();
            aborted = true;
            break;
        }
        tc_fence_after();
        float* sp = a.s_part + (static_cast<size_t>(bh) * a.nsplit + split) * R * kD;
#pragma unroll
        for (int c0 = 0; c0 < RH; c0 += 16) {
            uint32_t hi[32], lo[32];
            tmem_ld32(t_s + lane_base + half * RH + c0, hi);
            tmem_ld_wait(hi);
            tmem_ld32(t_s + lane_base + RP + half * RH + c0, lo);
            tmem_ld_wait(lo);
            const int cn = min(16, RH - c0);
            for (int i = 0; i < cn; ++i)
                sp[(half * RH + c0 + i) * kD + row] = __uint_as_float(hi[i]) + __uint_as_float(lo[i]);
        }
        // z: sum the per-thread partials over the token rows (warp shuffles, then the 4 warps of a half)
#pragma unroll
        for (int c = 0; c < RH; ++c) {
            float v = zacc[c];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            zacc[c] = v;
        }
        float* zslots = reinterpret_cast<float*>(smem + lay.off_zred);  // [8 warps][RH]
        if (lane == 0) {
#pragma unroll
            for (int c = 0; c < RH; ++c) zslots[warp * RH + c] = zacc[c];
        }
        __syncthreads();
        if (tid < R) {
            const int hh = tid / RH, c = tid % RH;  // warps 4*hh .. 4*hh+3 hold half hh
            const float* zs = zslots + (4 * hh) * RH + c;
            a.z_part[(static_cast<size_t>(bh) * a.nsplit + split) * R + tid] =
                ((zs[0] + zs[RH]) + zs[2 * RH]) + zs[3 * RH];
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (aborted && tid == 0) {
        // let loads and products still in flight land before the memory is released (bounded, 10 ms each)
        volatile int no_abort = 0;
        for (int st = 0; st < kStages; ++st)
            if (n_load[st] > n_wait[st]) mbar_wait(bar_kv + st, n_wait[st] & 1, 10000000ull, &no_abort);
        if (n_phi_issued > n_phi) mbar_wait(bar_phi, n_phi & 1, 10000000ull, &no_abort);
        if (n_s_issued > n_s_done) mbar_wait(bar_s, n_s_done & 1, 10000000ull, &no_abort);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, LrCfg<R>::kTmemCols);
    }
}

}  // namespace slra

namespace slra {

int lowrank_tc_tiles_per_split(const Geom& g, int nsplit) {
    const int ntiles = (g.L + kTok - 1) / kTok;
    return (ntiles + nsplit - 1) / nsplit;
}

template <int R, bool kDefault>
static cudaError_t lr_tc_launch_v(const CUtensorMap& tk, const CUtensorMap& tv, const LrArgs& a, const Geom& g,
                                  cudaStream_t st) {
    const size_t sm = static_cast<size_t>(lr_layout(R, LrCfg<R>::kStages).bytes) + 1024;
    cudaError_t e = cudaFuncSetAttribute(lowrank_sm100_kernel<R, kDefault>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int items = g.BH() * a.nsplit;
    const int slots = sms * LrCfg<R>::kCtasPerSm;
    lowrank_sm100_kernel<R, kDefault><<<items < slots ? items : slots, 256, sm, st>>>(tk, tv, a, g);
    return cudaGetLastError();
}
template <int R>
static cudaError_t lr_tc_launch(const CUtensorMap& tk, const CUtensorMap& tv, const LrArgs& a, const Geom& g,
                                cudaStream_t st) {
    return (g.act == 0 && g.norope == 0 && g.inside == 0) ? lr_tc_launch_v<R, true>(tk, tv, a, g, st)
                                                         : lr_tc_launch_v<R, false>(tk, tv, a, g, st);
}

cudaError_t launch_lowrank_tc(const __nv_bfloat16* k, const __nv_bfloat16* v, const __nv_bfloat16* A,
                              const double2* tab, const RopeMeta& meta, const Geom& g, int nsplit, float* s_part,
                              float* z_part, int* status, unsigned long long timeout_ns, int debug_unsatisfied_wait,
                              cudaStream_t st) {
    CUtensorMap tk, tv;
    if (!make_map_tokens(&tk, k, g.B, g.L, g.Hh, g.D, g.sk, kTok) ||
        !make_map_tokens(&tv, v, g.B, g.L, g.Hh, g.D, g.sv, kTok))
        return cudaErrorInvalidValue;
    LrArgs a;
    a.A = A;
    a.tab = tab;
    for (int e = 0; e < kMaxPairs; ++e)
        a.pair_info[e] = e < meta.npairs ? make_int2(meta.axis[e], meta.tab_off[e]) : make_int2(0, 0);
    a.s_part = s_part;
    a.z_part = z_part;
    a.nsplit = nsplit;
    a.tiles_per_split = lowrank_tc_tiles_per_split(g, nsplit);
    a.status = status;
    a.timeout_ns = timeout_ns;
    a.debug_unsatisfied_wait = debug_unsatisfied_wait;
    switch (g.R) {
        case 16: return lr_tc_launch<16>(tk, tv, a, g, st);
        case 32: return lr_tc_launch<32>(tk, tv, a, g, st);
        case 48: return lr_tc_launch<48>(tk, tv, a, g, st);
        case 64: return lr_tc_launch<64>(tk, tv, a, g, st);
        case 80: return lr_tc_launch<80>(tk, tv, a, g, st);
        case 96: return lr_tc_launch<96>(tk, tv, a, g, st);
        case 112: return lr_tc_launch<112>(tk, tv, a, g, st);
        case 128: return lr_tc_launch<128>(tk, tv, a, g, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace slra
