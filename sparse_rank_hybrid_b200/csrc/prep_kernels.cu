// Preparation kernels of the hybrid attention forward (all HBM- or latency-bound, CUDA cores):
//   rope_table      cos/sin of every (rotary pair, grid position), fp64
//   rope_pool       3D RoPE of q and k, fp16 head-major copies of q^, k^ and v for the tensor-core
//                   kernel, fp64 block means of q^ and k^
//   select          fp64 block scores qbar . kbar and per-row top-k (radix select, lower index wins ties)
//   lowrank_partial phi = act(k A), rank-truncated RoPE outside the activation, split-L partial sums
//                   of S = sum_j psi(k_j) v_j^T and z = sum_j phi(k_j)
//   lowrank_reduce  fixed-order sum of the partials (deterministic)
// Method: RoLA ("3 Preliminary" 3D RoPE; "4.1" block-sparse + low-rank branches; "4.2" first r rotary
// coordinates; "4.3" RoPE outside the activation; "B.1" one query-independent sum per head).
#include "common.cuh"
#include "sm100.cuh"

namespace slra {

// ------------------------------------------------------------------------------ rope_table
__global__ void rope_table_kernel(double2* tab, int2* pairs, RopeMeta meta, int entries) {
    int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e < meta.npairs) pairs[e] = make_int2(meta.axis[e], meta.tab_off[e]);
    if (e >= entries) return;
    int j = 0;
    while (j + 1 < meta.npairs && meta.tab_off[j + 1] <= e) ++j;
    int a = meta.axis[j];
    int p = e - meta.tab_off[j];
    double da = 2.0 * static_cast<double>(meta.apairs[a]);
    double omega = pow(meta.theta, -2.0 * static_cast<double>(meta.mloc[j]) / da);
    double ang = static_cast<double>(p + meta.off[a]) * omega;
    double s, c;
    sincos(ang, &s, &c);
    tab[e] = make_double2(c, s);
}

cudaError_t launch_rope_table(double2* tab, int2* pairs, const RopeMeta& meta, int entries, cudaStream_t st) {
    const int n = entries > meta.npairs ? entries : meta.npairs;
    rope_table_kernel<<<(n + 255) / 256, 256, 0, st>>>(tab, pairs, meta, entries);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------ rope_pool
// One CTA per (query/key block, batch*head): NTH = 256 threads and two CTAs per SM when the fp16 v copy
// is made (kV), 128 threads and three CTAs per SM without it (the same shared memory then holds three
// blocks in flight).  Thread 0 brings the block's q, k (and, with kV, v) rows of this head into shared
// memory with TMA (token-major 4D maps, 64-column boxes, 128-B swizzle; tokens past L read as zero), so
// a whole block's tiles are in flight at once.  The fp16 v copy is only made for the backward kernels;
// the forward's attention kernel reads v itself.  Then thread t owns four consecutive rotary pairs (8
// elements, 16 bytes) j = 4*(t % (D/8)) .. +3 and walks the block's tokens with stride NTH/(D/8); each
// fp16 output access is one 16-byte store, and the D/8 threads of a token cover its row, so a block's
// rows go out as one contiguous stretch per tensor.  The rotation and the block sums are fp64 so the
// selection scores are exact to ~1e-15 relative (the top-k decision is made on them); the fp16 copies
// come from the same values.
template <int D, bool kV, int NTH>
__global__ void __launch_bounds__(NTH, NTH == 256 ? 2 : 3) rope_pool_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                           const __grid_constant__ CUtensorMap tm_k,
                                                           const __grid_constant__ CUtensorMap tm_v,
                                                           const double2* __restrict__ tab,
                                                           const int2* __restrict__ pairs, Geom g,
                                                           __half* __restrict__ qh, __half* __restrict__ kh,
                                                           __half* __restrict__ vh, double* __restrict__ qbar,
                                                           double* __restrict__ kbar, int* status,
                                                           unsigned long long timeout_ns) {
    constexpr int Q4 = D / 8;          // threads per token row
    constexpr int G = NTH / Q4;        // tokens in flight
    constexpr int NS = D / 64;         // 64-column slabs per row
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    const int quad = threadIdx.x % Q4, grp = threadIdx.x / Q4;
    // heads vary fastest across the grid: the CTAs in flight read all heads of the same tokens, which
    // are contiguous in the token-major inputs
    const int bh = blockIdx.x, alpha = blockIdx.y;
    const int b = bh / g.Hh, h = bh % g.Hh;
    const int blk = g.block;
    const int n0 = alpha * blk;
    const uint32_t slab = static_cast<uint32_t>(blk) * 128;  // bytes of one 64-column slab of a tile
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        tma_prefetch_desc(&tm_q);
        mbar_expect_tx(&bar, (kV ? 3 : 2) * NS * slab);
#pragma unroll
        for (int s = 0; s < NS; ++s) {
            tma_load_4d(smem + (0 * NS + s) * slab, &tm_q, &bar, 64 * s, h, n0, b);
            tma_load_4d(smem + (1 * NS + s) * slab, &tm_k, &bar, 64 * s, h, n0, b);
            if (kV) tma_load_4d(smem + (2 * NS + s) * slab, &tm_v, &bar, 64 * s, h, n0, b);
        }
    }
    int axis[4], toff[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int2 pi = pairs[4 * quad + u];
        axis[u] = pi.x;
        toff[u] = pi.y;
    }
    double sq[4][2], sk[4][2];
#pragma unroll
    for (int u = 0; u < 4; ++u) sq[u][0] = sq[u][1] = sk[u][0] = sk[u][1] = 0.0;
    bool bad = false;
    const int HW = g.H * g.W;
    const bool landed = mbar_wait(&bar, 0, timeout_ns, &abort_flag);
    if (__syncthreads_or(!landed)) {
        if (threadIdx.x == 0) {
            atomicOr(status, kDevTimeout);
            volatile int no_abort = 0;
            mbar_wait(&bar, 0, 10000000ull, &no_abort);  // let the copies land before the CTA leaves
        }
        return;
    }
    const uint32_t c16 = quad & 7, sl = quad >> 3;  // 16-byte chunk within its slab, slab
    // (cos, sin) of this thread's pairs at the last position used: a thread's tokens are G apart, so the
    // temporal position rarely changes within a block and the height one only every W tokens; only
    // the pairs whose position moved are reloaded
    double2 cs_c[4];
    int pos_c[4];
    // largest |q^|, |k^|, |v| this thread wrote: a block whose nonzero values all lie below fp16's
    // smallest normal (2^-14) has lost relative precision in the fp16 operands and is reported
    float mq = 0.f, mk = 0.f, mv = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) pos_c[u] = -1;
    for (int i = grp; i < blk; i += G) {
        const int n = n0 + i;
        const size_t dst = (static_cast<size_t>(bh) * g.Lp + n) * D + 8 * quad;
        if (n < g.L) {
            const uint32_t off = sl * slab + i * 128 + ((c16 ^ (i & 7)) << 4);
            const uint4 qr = *reinterpret_cast<const uint4*>(smem + 0 * NS * slab + off);
            const uint4 kr = *reinterpret_cast<const uint4*>(smem + 1 * NS * slab + off);
            const uint4 vr = kV ? *reinterpret_cast<const uint4*>(smem + 2 * NS * slab + off) : make_uint4(0u, 0u, 0u, 0u);
            const int pt = n / HW, ph = (n / g.W) % g.H, pw = n % g.W;
            const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&qr);
            const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kr);
            const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&vr);
            uint4 qo, ko, vo;
            uint32_t* qo2 = reinterpret_cast<uint32_t*>(&qo);
            uint32_t* ko2 = reinterpret_cast<uint32_t*>(&ko);
            uint32_t* vo2 = reinterpret_cast<uint32_t*>(&vo);
            float m = 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int pos = axis[u] == 0 ? pt : (axis[u] == 1 ? ph : pw);
                if (pos != pos_c[u]) {
                    cs_c[u] = __ldg(tab + toff[u] + pos);
                    pos_c[u] = pos;
                }
                const double2 cs = cs_c[u];
                const float2 qf = __bfloat1622float2(q2[u]);
                const float2 kf = __bfloat1622float2(k2[u]);
                const float2 vf = __bfloat1622float2(v2[u]);
                const double qy0 = static_cast<double>(qf.x) * cs.x - static_cast<double>(qf.y) * cs.y;
                const double qy1 = static_cast<double>(qf.x) * cs.y + static_cast<double>(qf.y) * cs.x;
                const double ky0 = static_cast<double>(kf.x) * cs.x - static_cast<double>(kf.y) * cs.y;
                const double ky1 = static_cast<double>(kf.x) * cs.y + static_cast<double>(kf.y) * cs.x;
                sq[u][0] += qy0; sq[u][1] += qy1; sk[u][0] += ky0; sk[u][1] += ky1;
                const float a0 = static_cast<float>(qy0), a1 = static_cast<float>(qy1);
                const float c0 = static_cast<float>(ky0), c1 = static_cast<float>(ky1);
                mq = fmaxf(mq, fmaxf(fabsf(a0), fabsf(a1)));
                mk = fmaxf(mk, fmaxf(fabsf(c0), fabsf(c1)));
                if (kV) mv = fmaxf(mv, fmaxf(fabsf(vf.x), fabsf(vf.y)));
                m = fmaxf(m, fmaxf(fmaxf(mq, mk), mv));
                const __half2 hq = __floats2half2_rn(a0, a1), hk = __floats2half2_rn(c0, c1),
                              hv = __floats2half2_rn(vf.x, vf.y);
                qo2[u] = *reinterpret_cast<const uint32_t*>(&hq);
                ko2[u] = *reinterpret_cast<const uint32_t*>(&hk);
                if (kV) vo2[u] = *reinterpret_cast<const uint32_t*>(&hv);
            }
            bad |= !(m <= 65504.0f);
            *reinterpret_cast<uint4*>(qh + dst) = qo;
            *reinterpret_cast<uint4*>(kh + dst) = ko;
            if (kV) *reinterpret_cast<uint4*>(vh + dst) = vo;
        } else {
            const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(qh + dst) = z4;
            *reinterpret_cast<uint4*>(kh + dst) = z4;
            if (kV) *reinterpret_cast<uint4*>(vh + dst) = z4;
        }
    }
    // block maxima of |q^|, |k^|, |v| (non-negative floats order like their bit patterns)
    __shared__ unsigned int blk_max[3];
    if (threadIdx.x < 3) blk_max[threadIdx.x] = 0u;
    __syncthreads();  // the tiles are consumed; the reduction reuses their space
    {
        const unsigned int wq = __reduce_max_sync(0xffffffffu, __float_as_uint(mq));
        const unsigned int wk = __reduce_max_sync(0xffffffffu, __float_as_uint(mk));
        const unsigned int wv = __reduce_max_sync(0xffffffffu, __float_as_uint(mv));
        if ((threadIdx.x & 31) == 0) {
            atomicMax(&blk_max[0], wq);
            atomicMax(&blk_max[1], wk);
            atomicMax(&blk_max[2], wv);
        }
    }
    double* red = reinterpret_cast<double*>(smem);  // [G][q0,q1,k0,k1][D/2]
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int j = 4 * quad + u;
        red[(grp * 4 + 0) * (D / 2) + j] = sq[u][0];
        red[(grp * 4 + 1) * (D / 2) + j] = sq[u][1];
        red[(grp * 4 + 2) * (D / 2) + j] = sk[u][0];
        red[(grp * 4 + 3) * (D / 2) + j] = sk[u][1];
    }
    __syncthreads();
    // thread t < D/2 finishes pair t: fixed-order sum over the token groups
    if (threadIdx.x < D / 2) {
        const int j = threadIdx.x;
        double a0 = 0.0, a1 = 0.0, c0 = 0.0, c1 = 0.0;
        for (int u = 0; u < G; ++u) {
            a0 += red[(u * 4 + 0) * (D / 2) + j]; a1 += red[(u * 4 + 1) * (D / 2) + j];
            c0 += red[(u * 4 + 2) * (D / 2) + j]; c1 += red[(u * 4 + 3) * (D / 2) + j];
        }
        const int cnt = min(g.block, g.L - n0);
        const size_t o = (static_cast<size_t>(bh) * g.nb + alpha) * D + 2 * j;
        qbar[o] = a0 / cnt; qbar[o + 1] = a1 / cnt;
        kbar[o] = c0 / cnt; kbar[o + 1] = c1 / cnt;
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(status, kDevRange);
    if (threadIdx.x == 0) {
        constexpr float kMinNormalF16 = 6.103515625e-05f;  // 2^-14
        for (int t = 0; t < 3; ++t) {
            const float mx = __uint_as_float(blk_max[t]);
            if (mx > 0.f && mx < kMinNormalF16) atomicOr(status, kDevRange);
        }
    }
}

// The q, k (and v) tiles, or the block-sum exchange that later reuses them ([threads/(D/8)][4][D/2]
// fp64 = threads/8 KB for any D), whichever is larger.
size_t rope_pool_smem_bytes(const Geom& g, bool write_v, int threads) {
    const size_t tiles = static_cast<size_t>(write_v ? 3 : 2) * g.block * g.D * 2;
    const size_t red = static_cast<size_t>(threads / (g.D / 8)) * 4 * (g.D / 2) * 8;
    return (tiles > red ? tiles : red) + 1024;
}

template <int D, bool kV>
static cudaError_t launch_rope_pool_t(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                      const double2* tab, const int2* pairs, const Geom& g, __half* qh, __half* kh,
                                      __half* vh, double* qbar, double* kbar, int* status,
                                      unsigned long long timeout_ns, cudaStream_t st) {
    // without v: three CTAs of 128 threads per SM (more blocks in flight); with v: two of 256
    constexpr int NTH = kV ? 256 : 128;
    dim3 grid(g.BH(), g.nb);
    const int sm = static_cast<int>(rope_pool_smem_bytes(g, kV, NTH));
    cudaError_t e = cudaFuncSetAttribute(rope_pool_kernel<D, kV, NTH>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e != cudaSuccess) return e;
    rope_pool_kernel<D, kV, NTH><<<grid, NTH, sm, st>>>(tm_q, tm_k, tm_v, tab, pairs, g, qh, kh, vh, qbar, kbar,
                                                        status, timeout_ns);
    return cudaGetLastError();
}

cudaError_t launch_rope_pool(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                             const double2* tab, const int2* pairs, const Geom& g, bool write_v, __half* qh,
                             __half* kh, __half* vh, double* qbar, double* kbar, int* status,
                             unsigned long long timeout_ns, cudaStream_t st) {
    if (g.D == 128)
        return write_v ? launch_rope_pool_t<128, true>(tm_q, tm_k, tm_v, tab, pairs, g, qh, kh, vh, qbar, kbar, status,
                                                       timeout_ns, st)
                       : launch_rope_pool_t<128, false>(tm_q, tm_k, tm_v, tab, pairs, g, qh, kh, vh, qbar, kbar,
                                                        status, timeout_ns, st);
    return write_v ? launch_rope_pool_t<64, true>(tm_q, tm_k, tm_v, tab, pairs, g, qh, kh, vh, qbar, kbar, status,
                                                  timeout_ns, st)
                   : launch_rope_pool_t<64, false>(tm_q, tm_k, tm_v, tab, pairs, g, qh, kh, vh, qbar, kbar, status,
                                                   timeout_ns, st);
}

// ------------------------------------------------------------------------------ select
// Order-preserving map of a double to uint64 (-0.0 folded into +0.0 first).
__device__ __forceinline__ uint64_t ordered_key(double x) {
    x = x + 0.0;
    const uint64_t u = static_cast<uint64_t>(__double_as_longlong(x));
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}
__device__ __forceinline__ double key_value(uint64_t k) {
    const uint64_t u = (k >> 63) ? (k & 0x7FFFFFFFFFFFFFFFull) : ~k;
    return __longlong_as_double(static_cast<long long>(u));
}

constexpr int kSelRows = 8;   // query blocks per CTA (one warp each in the selection phase)

// D (8x8, fp64) += A (8x4, row-major) * B (4x8, col-major) on the fp64 tensor pipe.  Fragments: lane l
// holds A[l/4][l%4], B[l%4][l/4], and D[l/4][2(l%4)], D[l/4][2(l%4)+1].
__device__ __forceinline__ void dmma_8x8x4(double& d0, double& d1, double a, double b) {
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                 : "+d"(d0), "+d"(d1)
                 : "d"(a), "d"(b));
}

// One CTA per (8 query blocks, batch*head).  Phase 1: the 8 x nb block of fp64 scores qbar kbar^T on
// the fp64 tensor pipe (m8n8k4): every warp keeps the 8 qbar rows as A fragments in registers and
// sweeps its share of 8-key tiles, streaming the kbar fragments from L2.  Phase 2: warp w selects row
// w's top-k by an 8-pass radix select on the order-preserving 64-bit keys, then writes the selected
// block indices in ascending order (ties at the threshold resolved to the lowest indices) and the tie
// flag.
template <int D>
__global__ void __launch_bounds__(256, 2) select_kernel(const double* __restrict__ qbar,
                                                     const double* __restrict__ kbar, Geom g,
                                                     int32_t* __restrict__ idx, uint8_t* __restrict__ tie) {
    extern __shared__ __align__(16) unsigned char sm_raw[];
    double* scores = reinterpret_cast<double*>(sm_raw);                 // [8][nb]
    int* hist = reinterpret_cast<int*>(scores + kSelRows * g.nb);      // [8][256]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bh = blockIdx.y;
    const int a0 = blockIdx.x * kSelRows;
    const int nb = g.nb;
    const double* qb = qbar + static_cast<size_t>(bh) * nb * D;
    const double* kb = kbar + static_cast<size_t>(bh) * nb * D;

    // The D/4 k-steps take the dims in pairs: k-steps 2m and 2m+1 give lane l dims 8m + 2(l%4) and
    // 8m + 2(l%4) + 1, so each lane loads both with one 16-byte load and the four lanes of a row read 64
    // contiguous bytes (any order of the dims gives the same dot product up to fp64 rounding).
    // A fragments: row l/4 of the 8 query blocks.
    double af[D / 4];
    {
        const int ar = a0 + (lane >> 2);
        const double2* arow = reinterpret_cast<const double2*>(qb + static_cast<size_t>(ar < nb ? ar : 0) * D) + (lane & 3);
#pragma unroll
        for (int m = 0; m < D / 8; ++m) {
            const double2 a2 = ar < nb ? __ldg(arow + 4 * m) : make_double2(0.0, 0.0);
            af[2 * m] = a2.x;
            af[2 * m + 1] = a2.y;
        }
    }
    const int ntile = (nb + 7) / 8;
    for (int t = warp; t < ntile; t += 8) {
        const int key = 8 * t + (lane >> 2);  // B fragment: key l/4 of the tile, the same dims as A
        const double2* kr =
            reinterpret_cast<const double2*>(kb + static_cast<size_t>(key < nb ? key : nb - 1) * D) + (lane & 3);
        // four independent accumulator chains over the k-steps (a single chain of D/4 dependent
        // products is latency-bound), summed at the end
        double d[4][2] = {{0.0, 0.0}, {0.0, 0.0}, {0.0, 0.0}, {0.0, 0.0}};
#pragma unroll
        for (int m = 0; m < D / 8; ++m) {
            const double2 b2 = __ldg(kr + 4 * m);
            double (&da)[2] = d[(2 * m) & 3];
            double (&db)[2] = d[(2 * m + 1) & 3];
            dmma_8x8x4(da[0], da[1], af[2 * m], b2.x);
            dmma_8x8x4(db[0], db[1], af[2 * m + 1], b2.y);
        }
        const double d0 = (d[0][0] + d[1][0]) + (d[2][0] + d[3][0]);
        const double d1 = (d[0][1] + d[1][1]) + (d[2][1] + d[3][1]);
        const int r = lane >> 2, c = 8 * t + 2 * (lane & 3);
        if (c < nb) scores[r * nb + c] = d0;
        if (c + 1 < nb) scores[r * nb + c + 1] = d1;
    }
    __syncthreads();

    const int alpha = a0 + warp;
    if (alpha >= nb) return;
    const double* srow = scores + warp * nb;
    int* hw = hist + warp * 256;
    const int keep = g.keep;
    uint64_t prefix = 0, pmask = 0;
    int rem = keep;
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = lane; i < 256; i += 32) hw[i] = 0;
        __syncwarp();
        for (int i = lane; i < nb; i += 32) {
            const uint64_t u = ordered_key(srow[i]);
            if ((u & pmask) == prefix) atomicAdd(&hw[(u >> shift) & 255], 1);
        }
        __syncwarp();
        // lane owns bins 255-8*lane .. 248-8*lane (descending)
        int cnt[8], local = 0;
#pragma unroll
        for (int t = 0; t < 8; ++t) { cnt[t] = hw[255 - (lane * 8 + t)]; local += cnt[t]; }
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int nbv = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += nbv;
        }
        const int excl = incl - local;
        const unsigned owner = __ballot_sync(0xffffffffu, excl < rem && rem <= incl);
        const int src = __ffs(owner) - 1;
        int binsel = 0, above = 0;
        if (lane == src) {
            int acc = excl;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                if (acc + cnt[t] >= rem) { binsel = 255 - (lane * 8 + t); above = acc; break; }
                acc += cnt[t];
            }
        }
        binsel = __shfl_sync(0xffffffffu, binsel, src);
        above = __shfl_sync(0xffffffffu, above, src);
        rem -= above;
        prefix |= static_cast<uint64_t>(binsel) << shift;
        pmask |= 0xFFull << shift;
        __syncwarp();
    }
    // prefix = key of the k-th largest score; take every larger key and the first `rem` equal ones.
    int32_t* out = idx + (static_cast<size_t>(bh) * nb + alpha) * keep;
    int written = 0, eq_seen = 0;
    uint64_t next_best = 0;
    bool has_next = false;
    for (int base = 0; base < nb; base += 32) {
        const int i = base + lane;
        const bool valid = i < nb;
        const uint64_t u = valid ? ordered_key(srow[i]) : 0;
        const bool gt = valid && u > prefix;
        const bool eq = valid && u == prefix;
        const unsigned eqm = __ballot_sync(0xffffffffu, eq);
        const unsigned below = (1u << lane) - 1u;
        const bool sel = gt || (eq && (eq_seen + __popc(eqm & below)) < rem);
        const unsigned selm = __ballot_sync(0xffffffffu, sel);
        if (sel) out[written + __popc(selm & below)] = i;
        written += __popc(selm);
        eq_seen += __popc(eqm);
        if (valid && !sel && (!has_next || u > next_best)) { next_best = u; has_next = true; }
    }
    // (k+1)-th largest = max over the unselected keys
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t ob = __shfl_xor_sync(0xffffffffu, next_best, o);
        const int oh = __shfl_xor_sync(0xffffffffu, has_next ? 1 : 0, o);
        if (oh && (!has_next || ob > next_best)) { next_best = ob; has_next = true; }
    }
    if (lane == 0) {
        uint8_t t = 0;
        if (keep < nb && has_next) {
            const double sk = key_value(prefix), sk1 = key_value(next_best);
            t = (sk - sk1) <= 1e-6 * fmax(1.0, fabs(sk));
        }
        tie[static_cast<size_t>(bh) * nb + alpha] = t;
    }
}

static size_t select_smem(const Geom& g) {
    return sizeof(double) * static_cast<size_t>(kSelRows) * g.nb + sizeof(int) * kSelRows * 256;
}

cudaError_t launch_select(const double* qbar, const double* kbar, const Geom& g, int32_t* idx, uint8_t* tie,
                          cudaStream_t st) {
    dim3 grid((g.nb + kSelRows - 1) / kSelRows, g.BH());
    const size_t sm = select_smem(g);
    cudaError_t e;
    if (g.D == 128) {
        e = cudaFuncSetAttribute(select_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        select_kernel<128><<<grid, 256, sm, st>>>(qbar, kbar, g, idx, tie);
    } else {
        e = cudaFuncSetAttribute(select_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        select_kernel<64><<<grid, 256, sm, st>>>(qbar, kbar, g, idx, tie);
    }
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------ low-rank summary
constexpr int kLrTile = 32;  // tokens per step

// One CTA per (split of the sequence, batch*head).  Per 32-token step: stage raw k and v (fp32) in
// shared memory, phi = act(k A) (thread per (token, feature)), rotate the first R coordinates with
// the token's 3D RoPE angles (psi), then accumulate S[c][e] += sum_t psi[t][c] v[t][e] in registers
// (thread owns one e and R/(256/D) features) and z[c] += sum_t phi[t][c].
template <int D, int R>
__global__ void __launch_bounds__(256) lowrank_partial_kernel(const __nv_bfloat16* __restrict__ k,
                                                              const __nv_bfloat16* __restrict__ v,
                                                              const __nv_bfloat16* __restrict__ A,
                                                              const double2* __restrict__ tab,
                                                              const int2* __restrict__ pairs, Geom g, int nsplit, float* __restrict__ s_part,
                                                              float* __restrict__ z_part) {
    extern __shared__ __align__(16) float smf[];
    float* As = smf;                        // [D][R]
    float* ks = As + D * R;                 // [32][D+1]
    float* vs = ks + kLrTile * (D + 1);     // [32][D]
    float* ph = vs + kLrTile * D;           // [32][R+1]
    float* ps = ph + kLrTile * (R + 1);     // [32][R]
    constexpr int G = 256 / D;              // feature groups
    constexpr int NA = R / G;               // accumulators per thread
    const int tid = threadIdx.x;
    const int split = blockIdx.x, bh = blockIdx.y;
    const int b = bh / g.Hh, h = bh % g.Hh;
    const int ntiles = (g.L + kLrTile - 1) / kLrTile;
    const int per = (ntiles + nsplit - 1) / nsplit;
    const int t0 = split * per, t1 = min(ntiles, t0 + per);

    const __nv_bfloat16* Ah = A + static_cast<size_t>(h) * g.a_stride;  // this head's key projection
    for (int e = tid; e < D * R; e += 256) As[e] = __bfloat162float(Ah[e]);
    const int e_own = tid % D, cg = tid / D;
    float acc[NA];
#pragma unroll
    for (int i = 0; i < NA; ++i) acc[i] = 0.f;
    float zacc = 0.f;

    for (int tile = t0; tile < t1; ++tile) {
        const int n0 = tile * kLrTile;
        __syncthreads();
        for (int e = tid; e < kLrTile * (D / 2); e += 256) {
            const int tt = e / (D / 2), dp = e % (D / 2);
            const int n = n0 + tt;
            float2 kf = make_float2(0.f, 0.f), vf = make_float2(0.f, 0.f);
            if (n < g.L) {
                kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(k + g.sk.row(b, n, h) + 2 * dp));
                vf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(v + g.sv.row(b, n, h) + 2 * dp));
            }
            ks[tt * (D + 1) + 2 * dp] = kf.x; ks[tt * (D + 1) + 2 * dp + 1] = kf.y;
            vs[tt * D + 2 * dp] = vf.x; vs[tt * D + 2 * dp + 1] = vf.y;
        }
        __syncthreads();
        for (int o = tid; o < kLrTile * R; o += 256) {
            const int tt = o / R, c = o % R;
            const float* kr = ks + tt * (D + 1);
            float a = 0.f;
#pragma unroll 16
            for (int d = 0; d < D; ++d) a = fmaf(kr[d], As[d * R + c], a);
            ph[tt * (R + 1) + c] = g.inside ? a : phi_act(a, g.act);  // inside: activation after the rotation
        }
        __syncthreads();
        for (int o = tid; o < kLrTile * (R / 2); o += 256) {
            const int tt = o / (R / 2), p = o % (R / 2);
            const int n = n0 + tt;
            const float x0 = ph[tt * (R + 1) + 2 * p], x1 = ph[tt * (R + 1) + 2 * p + 1];
            float c = 1.f, s = 0.f;
            if (n < g.L && !g.norope) {
                const int2 pi = pairs[p];
                const double2 cs = tab[pi.y + token_axis_pos(n, pi.x, g.H, g.W)];
                c = static_cast<float>(cs.x);
                s = static_cast<float>(cs.y);
            }
            float y0 = x0 * c - x1 * s, y1 = x0 * s + x1 * c;
            if (g.inside) {
                y0 = phi_act(y0, g.act);
                y1 = phi_act(y1, g.act);
            }
            ps[tt * R + 2 * p] = y0;
            ps[tt * R + 2 * p + 1] = y1;
        }
        __syncthreads();
#pragma unroll 4
        for (int tt = 0; tt < kLrTile; ++tt) {
            const float vv = vs[tt * D + e_own];
            const float* pr = ps + tt * R + cg;
#pragma unroll
            for (int i = 0; i < NA; ++i) acc[i] = fmaf(pr[G * i], vv, acc[i]);
        }
        if (tid < R)  // z sums the unrotated features, or psi when the RoPE is inside the activation
            for (int tt = 0; tt < kLrTile; ++tt) zacc += g.inside ? ps[tt * R + tid] : ph[tt * (R + 1) + tid];
    }
    float* sp = s_part + (static_cast<size_t>(bh) * nsplit + split) * R * D;
#pragma unroll
    for (int i = 0; i < NA; ++i) sp[(cg + G * i) * D + e_own] = acc[i];
    if (tid < R) z_part[(static_cast<size_t>(bh) * nsplit + split) * R + tid] = zacc;
}

template <int D, int R>
static cudaError_t lr_launch(const __nv_bfloat16* k, const __nv_bfloat16* v, const __nv_bfloat16* A,
                             const double2* tab, const int2* pairs, const Geom& g, int nsplit, float* s_part,
                             float* z_part, cudaStream_t st) {
    const size_t sm = sizeof(float) * (D * R + kLrTile * (D + 1) + kLrTile * D + kLrTile * (R + 1) + kLrTile * R);
    cudaError_t e = cudaFuncSetAttribute(lowrank_partial_kernel<D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sm);
    if (e != cudaSuccess) return e;
    lowrank_partial_kernel<D, R><<<dim3(nsplit, g.BH()), 256, sm, st>>>(k, v, A, tab, pairs, g, nsplit, s_part, z_part);
    return cudaGetLastError();
}

cudaError_t launch_lowrank_partial(const __nv_bfloat16* k, const __nv_bfloat16* v, const __nv_bfloat16* A,
                                   const double2* tab, const int2* pairs, const Geom& g, int nsplit,
                                   float* s_part, float* z_part, cudaStream_t st) {
    if (g.D == 128) {
        switch (g.R) {
            case 16: return lr_launch<128, 16>(k, v, A, tab, pairs, g, nsplit, s_part, z_part, st);
            case 32: return lr_launch<128, 32>(k, v, A, tab, pairs, g, nsplit, s_part, z_part, st);
            case 48: return lr_launch<128, 48>(k, v, A, tab, pairs, g, nsplit, s_part, z_part, st);
            case 64: return lr_launch<128, 64>(k, v, A, tab, pairs, g, nsplit, s_part, z_part, st);
            case 80: return lr_launch<128, 80>(k, v, A, tab, pairs, g, nsplit, s_part, z_part, st);
            case 96: return lr_launch<128, 96>(k, v, A, tab, pairs, g, nsplit, s_part, z_part, st);
            case 112: return lr_launch<128, 112>(k, v, A, tab, pairs, g, nsplit, s_part, z_part, st);
            case 128: return lr_launch<128, 128>(k, v, A, tab, pairs, g, nsplit, s_part, z_part, st);
        }
    } else if (g.D == 64) {
        switch (g.R) {
            case 16: return lr_launch<64, 16>(k, v, A, tab, pairs, g, nsplit, s_part, z_part, st);
            case 32: return lr_launch<64, 32>(k, v, A, tab, pairs, g, nsplit, s_part, z_part, st);
            case 48: return lr_launch<64, 48>(k, v, A, tab, pairs, g, nsplit, s_part, z_part, st);
            case 64: return lr_launch<64, 64>(k, v, A, tab, pairs, g, nsplit, s_part, z_part, st);
        }
    }
    return cudaErrorInvalidValue;
}

__device__ __forceinline__ uint16_t bf16_rn_bits(float x) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    return *reinterpret_cast<const uint16_t*>(&h);
}

// Fixed-order sum of the split-L partials -> S [R][D] and z [R] per head.  With images requested
// (head_dim 128) it also writes, per head and 64-feature chunk, the S operand image of the attention
// epilogue's readout product (K columns S_hi | S_lo | S_hi, bf16 split so that hi + lo = S to ~2^-16),
// and the A^T operand image of its feature product from the query projection A: one image written by
// the blocks of head 0 when A is shared (a_stride 0), else one per head, by the blocks of batch 0.
__global__ void lowrank_reduce_kernel(const float* __restrict__ s_part, const float* __restrict__ z_part, int RD,
                                      int R, int D, int nsplit, float* __restrict__ S, float* __restrict__ z,
                                      const __nv_bfloat16* __restrict__ A, uint8_t* __restrict__ at_img,
                                      uint8_t* __restrict__ sb_img, int Hh, int a_stride) {
    const int bh = blockIdx.y;
    const int o = blockIdx.x * blockDim.x + threadIdx.x;
    if (o < RD) {
        const float* p = s_part + static_cast<size_t>(bh) * nsplit * RD + o;
        float a = 0.f;
        for (int s = 0; s < nsplit; ++s) a += p[static_cast<size_t>(s) * RD];
        S[static_cast<size_t>(bh) * RD + o] = a;
        if (sb_img) {
            const int c = o / D, e = o % D;
            const int nch = (R + 63) / 64, ch = c / 64, cc = c % 64, rc = min(64, R - 64 * ch);
            const uint16_t hi = bf16_rn_bits(a);
            const uint16_t lo = bf16_rn_bits(a - __uint_as_float(static_cast<uint32_t>(hi) << 16));
            uint8_t* img = sb_img + (static_cast<size_t>(bh) * nch + ch) * kSbChunkBytes;
            *reinterpret_cast<uint16_t*>(img + sw128_offset(e, cc, D)) = hi;
            *reinterpret_cast<uint16_t*>(img + sw128_offset(e, rc + cc, D)) = lo;
            *reinterpret_cast<uint16_t*>(img + sw128_offset(e, 2 * rc + cc, D)) = hi;
        }
        if (at_img && (a_stride == 0 ? bh == 0 : bh < Hh)) {  // element (c, d) of A^T = A[d][c]
            const int c = o / D, d = o % D;
            const size_t hd = a_stride == 0 ? 0 : static_cast<size_t>(bh);  // bh = head when b = 0
            *reinterpret_cast<uint16_t*>(at_img + hd * R * 256 + sw128_offset(c, d, R)) =
                *reinterpret_cast<const uint16_t*>(A + hd * a_stride + static_cast<size_t>(d) * R + c);
        }
    } else if (o < RD + R) {
        const int c = o - RD;
        const float* p = z_part + static_cast<size_t>(bh) * nsplit * R + c;
        float a = 0.f;
        for (int s = 0; s < nsplit; ++s) a += p[static_cast<size_t>(s) * R];
        z[static_cast<size_t>(bh) * R + c] = a;
    }
}

cudaError_t launch_lowrank_reduce(const float* s_part, const float* z_part, const Geom& g, int nsplit, float* S,
                                  float* z, const __nv_bfloat16* A, uint8_t* at_img, uint8_t* sb_img,
                                  cudaStream_t st) {
    const int RD = g.R * g.D;
    dim3 grid((RD + g.R + 255) / 256, g.BH());
    lowrank_reduce_kernel<<<grid, 256, 0, st>>>(s_part, z_part, RD, g.R, g.D, nsplit, S, z, A, at_img, sb_img, g.Hh,
                                                g.a_stride);
    return cudaGetLastError();
}

}  // namespace slra
