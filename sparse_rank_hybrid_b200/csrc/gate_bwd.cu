// Backward of the gated fusion of the two branches (RoLA 4.4, in the reading the forward implements):
//   out = O_s + c O_lr,   c = g a / b,   a = sqrt(mean(O_s^2)),   b = sqrt(mean(O_lr^2) + 1e-6),
//   g = sigmoid(q . Wg + bg) on the head's raw query row.
// Per row, with t = dout . O_lr:
//   dO_s   = dout + c t / (D a^2) O_s        (the a-term is absent when a = 0)
//   dO_lr  = c dout - c t / (D b^2) O_lr
//   dlogit = t (a / b) g (1 - g),   dq += dlogit Wg,   dWg = sum dlogit q,   dbg = sum dlogit.
// The sparse gradient kernels then run on dO_s (through the fp16 copy and Delta = dO_s . O_s this prep
// writes) and the low-rank passes on dO_lr.
#include "common.cuh"

namespace slra {

namespace {

// One warp per row (b, h, n) of the padded head-major grid: O_s and O_lr head-major fp32, dout and
// dO_lr token-major fp32, the fp16 copy of dO_s head-major (rows past L zero).
template <int D>
__global__ void __launch_bounds__(256) bwd_gate_prep_kernel(const float* __restrict__ dout, const float* __restrict__ os,
                                     const float* __restrict__ olr, const __nv_bfloat16* __restrict__ q,
                                     const float* __restrict__ gate_w, float gate_b, Geom g,
                                     __half* __restrict__ doh, float* __restrict__ delta, float* __restrict__ dolr,
                                     float* __restrict__ dlogit, int* status) {
    const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const long long rows = static_cast<long long>(g.BH()) * g.Lp;
    if (warp >= rows) return;
    const int bh = static_cast<int>(warp / g.Lp), n = static_cast<int>(warp % g.Lp);
    const int b = bh / g.Hh, h = bh % g.Hh;
    constexpr int per = D / 32;  // elements per lane: 2 or 4
    __half* dst = doh + static_cast<size_t>(warp) * D + lane * per;
    if (n >= g.L) {
        for (int e = 0; e < per; e += 2) *reinterpret_cast<__half2*>(dst + e) = __floats2half2_rn(0.f, 0.f);
        if (lane == 0) {
            delta[warp] = 0.f;
            dlogit[warp] = 0.f;
        }
        return;
    }
    float x[per], s[per], l[per], qf[per];
    float ss_s = 0.f, ss_l = 0.f, t = 0.f, qw = 0.f;
    const float* src = dout + g.so.row(b, n, h) + lane * per;
    const float* so = os + static_cast<size_t>(warp) * D + lane * per;
    const float* sl = olr + static_cast<size_t>(warp) * D + lane * per;
    const __nv_bfloat16* sq = q + g.sq.row(b, n, h) + lane * per;
#pragma unroll
    for (int e = 0; e < per; e += 2) {  // 8-byte loads (the rows are 16-byte aligned)
        const float2 x2 = *reinterpret_cast<const float2*>(src + e), s2 = *reinterpret_cast<const float2*>(so + e),
                     l2 = *reinterpret_cast<const float2*>(sl + e);
        const float2 q2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(sq + e));
        x[e] = x2.x; x[e + 1] = x2.y;
        s[e] = s2.x; s[e + 1] = s2.y;
        l[e] = l2.x; l[e + 1] = l2.y;
        qf[e] = q2.x; qf[e + 1] = q2.y;
    }
#pragma unroll
    for (int e = 0; e < per; ++e) {
        ss_s = fmaf(s[e], s[e], ss_s);
        ss_l = fmaf(l[e], l[e], ss_l);
        t = fmaf(x[e], l[e], t);
        qw = fmaf(qf[e], __ldg(gate_w + lane * per + e), qw);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ss_s += __shfl_xor_sync(0xffffffffu, ss_s, o);
        ss_l += __shfl_xor_sync(0xffffffffu, ss_l, o);
        t += __shfl_xor_sync(0xffffffffu, t, o);
        qw += __shfl_xor_sync(0xffffffffu, qw, o);
    }
    const float inv_d = 1.f / static_cast<float>(D);
    const float a = sqrtf(ss_s * inv_d), bb = sqrtf(ss_l * inv_d + 1e-6f);
    const float gg = 1.f / (1.f + expf(-(qw + gate_b)));
    const float c = gg * a / bb;
    const float ks = a > 0.f ? c * t * inv_d / (a * a) : 0.f;
    const float kl = c * t * inv_d / (bb * bb);
    float dsum = 0.f;
    bool bad = false;
    float* dl = dolr + g.so.row(b, n, h) + lane * per;
#pragma unroll
    for (int e = 0; e < per; e += 2) {
        const float d0 = fmaf(ks, s[e], x[e]), d1 = fmaf(ks, s[e + 1], x[e + 1]);
        dsum = fmaf(d0, s[e], fmaf(d1, s[e + 1], dsum));
        bad |= !(fmaxf(fabsf(d0), fabsf(d1)) < 65504.f);
        *reinterpret_cast<__half2*>(dst + e) = __floats2half2_rn(d0, d1);
        *reinterpret_cast<float2*>(dl + e) = make_float2(c * x[e] - kl * l[e], c * x[e + 1] - kl * l[e + 1]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
    if (lane == 0) {
        delta[warp] = dsum;
        dlogit[warp] = t * (a / bb) * gg * (1.f - gg);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(status, kDevRange);
}

// dq += dlogit Wg on every row, and per-CTA partial sums of dWg = sum dlogit q and dbg = sum dlogit
// over a fixed range of rows, in a fixed order.  A warp takes a row (each lane D/32 consecutive
// columns, vector loads and stores), the CTA's 8 warps 8 rows at a time, four such steps in flight.
template <int D>
__global__ void __launch_bounds__(256) bwd_gate_final_kernel(const __nv_bfloat16* __restrict__ q,
                                                             const float* __restrict__ dlogit,
                                                             const float* __restrict__ gate_w, Geom g,
                                                             long long rows_per_cta, float* __restrict__ dq,
                                                             float* __restrict__ part) {
    constexpr int P = D / 32, U = 4, NW = 8;
    __shared__ float red[NW][D + 1];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const long long rows = static_cast<long long>(g.BH()) * g.L;
    const long long r0 = blockIdx.x * rows_per_cta;
    const long long r1 = r0 + rows_per_cta < rows ? r0 + rows_per_cta : rows;
    float wg[P], acc[P];
#pragma unroll
    for (int e = 0; e < P; ++e) {
        wg[e] = __ldg(gate_w + lane * P + e);
        acc[e] = 0.f;
    }
    float accb = 0.f;
    // (head, token) of this warp's next row, advanced incrementally (no 64-bit division in the loop)
    long long r = r0 + wid;
    int bh = static_cast<int>(r / g.L), n = static_cast<int>(r % g.L);
    while (r < r1) {
        float dl[U], qv[U][P], pv[U][P];
        float* dst[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            dst[u] = nullptr;
            dl[u] = 0.f;
            if (r < r1) {
                const int b = bh / g.Hh, h = bh % g.Hh;
                dl[u] = dlogit[static_cast<size_t>(bh) * g.Lp + n];
                const __nv_bfloat16* qs = q + g.sq.row(b, n, h) + lane * P;
                dst[u] = dq + g.so.row(b, n, h) + lane * P;
                if constexpr (P == 4) {
                    const uint2 raw = *reinterpret_cast<const uint2*>(qs);
                    const float2 a0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
                    const float2 a1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
                    qv[u][0] = a0.x; qv[u][1] = a0.y; qv[u][2] = a1.x; qv[u][3] = a1.y;
                    const float4 o = *reinterpret_cast<const float4*>(dst[u]);
                    pv[u][0] = o.x; pv[u][1] = o.y; pv[u][2] = o.z; pv[u][3] = o.w;
                } else {
                    const float2 a0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(qs));
                    qv[u][0] = a0.x; qv[u][1] = a0.y;
                    const float2 o = *reinterpret_cast<const float2*>(dst[u]);
                    pv[u][0] = o.x; pv[u][1] = o.y;
                }
            }
            r += NW;
            n += NW;
            while (n >= g.L) {
                n -= g.L;
                ++bh;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (dst[u] == nullptr) continue;
#pragma unroll
            for (int e = 0; e < P; ++e) {
                acc[e] = fmaf(dl[u], qv[u][e], acc[e]);
                pv[u][e] = fmaf(dl[u], wg[e], pv[u][e]);
            }
            accb += dl[u];
            if constexpr (P == 4)
                *reinterpret_cast<float4*>(dst[u]) = make_float4(pv[u][0], pv[u][1], pv[u][2], pv[u][3]);
            else
                *reinterpret_cast<float2*>(dst[u]) = make_float2(pv[u][0], pv[u][1]);
        }
    }
#pragma unroll
    for (int e = 0; e < P; ++e) red[wid][lane * P + e] = acc[e];
    if (lane == 0) red[wid][D] = accb;  // every lane of a warp sums the same dlogit values
    __syncthreads();
    float* mine = part + static_cast<size_t>(blockIdx.x) * (D + 1);
    for (int c = threadIdx.x; c <= D; c += blockDim.x) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) t += red[w][c];
        mine[c] = t;
    }
}

// dWg, dbg from the kGateParts partials: a CTA takes 32 consecutive outputs, its 8 warps each sum
// every 8th partial, and the 8 sums are added in warp order (deterministic).
__global__ void __launch_bounds__(256) bwd_gate_reduce_kernel(const float* __restrict__ part, int nparts, int D,
                                                              float* __restrict__ dgw, float* __restrict__ dgb) {
    __shared__ float red[8][32];
    const int lo = threadIdx.x & 31, sl = threadIdx.x >> 5;
    const int o = blockIdx.x * 32 + lo;
    float s = 0.f;
    if (o <= D)
        for (int i = sl; i < nparts; i += 8) s += part[static_cast<size_t>(i) * (D + 1) + o];
    red[sl][lo] = s;
    __syncthreads();
    if (sl == 0 && o <= D) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) t += red[w][lo];
        if (o < D) dgw[o] = t;
        else *dgb = t;
    }
}

}  // namespace

cudaError_t launch_gate_prep(const float* dout, const float* os, const float* olr, const __nv_bfloat16* q,
                             const float* gate_w, float gate_b, const Geom& g, __half* doh, float* delta, float* dolr,
                             float* dlogit, int* status, cudaStream_t st) {
    const long long rows = static_cast<long long>(g.BH()) * g.Lp;
    const long long blocks = (rows * 32 + 255) / 256;
    if (g.D == 128)
        bwd_gate_prep_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, st>>>(dout, os, olr, q, gate_w, gate_b, g,
                                                                                 doh, delta, dolr, dlogit, status);
    else
        bwd_gate_prep_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, st>>>(dout, os, olr, q, gate_w, gate_b, g,
                                                                                doh, delta, dolr, dlogit, status);
    return cudaGetLastError();
}

cudaError_t launch_gate_final(const __nv_bfloat16* q, const float* dlogit, const float* gate_w, const Geom& g,
                              float* dq, float* part, float* dgw, float* dgb, cudaStream_t st) {
    const long long rows = static_cast<long long>(g.BH()) * g.L;
    const long long per = (rows + kGateParts - 1) / kGateParts;
    if (g.D == 128) bwd_gate_final_kernel<128><<<kGateParts, 256, 0, st>>>(q, dlogit, gate_w, g, per, dq, part);
    else bwd_gate_final_kernel<64><<<kGateParts, 256, 0, st>>>(q, dlogit, gate_w, g, per, dq, part);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bwd_gate_reduce_kernel<<<(g.D + 1 + 31) / 32, 256, 0, st>>>(part, kGateParts, g.D, dgw, dgb);
    return cudaGetLastError();
}

}  // namespace slra
