// Internal parameter blocks shared by the kernels and the C-ABI layer of libslra.so.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace slra {

constexpr int kMaxPairs = 64;  // head_dim <= 128

// Bits of the device status word.
constexpr int kDevTimeout = 1;
constexpr int kDevRange = 2;

// Element strides (batch, token, head) of a [B][L][Hh][D] tensor whose D elements are contiguous.
struct Strides {
    long long b, l, h;
    __host__ __device__ long long row(int bi, int n, int hi) const { return bi * b + n * l + hi * h; }
};

// Sizes of one call.  L = T*H*W; Lp = nb*block (rows of the padded head-major buffers).
struct Geom {
    int B, Hh, D, T, H, W, L, block, nb, keep, R, Lp;
    int act;     // SLRA_ACT_* of the low-rank feature map
    int norope;  // 1: no rotation in the low-rank branch (psi = phi)
    int a_stride;  // elements between consecutive heads' projections (D * R when per head, else 0)
    int inside;    // 1: the low-rank RoPE before the activation (psi = act(R x A), normaliser on psi)
    Strides sq, sk, sv, so;  // element strides of q, k, v and out
    __host__ __device__ int BH() const { return B * Hh; }
};

// Strides of a head-major [B][Hh][Lp][D] buffer addressed as [B][L][Hh][D] rows.
inline Strides headmajor_strides(const Geom& g) {
    return Strides{static_cast<long long>(g.Hh) * g.Lp * g.D, g.D, static_cast<long long>(g.Lp) * g.D};
}

// phi = act(u) for the low-rank feature map: relu (0), SiLU u / (1 + e^-u) (1), identity (2), tanh (3).
// relu stays inline; the other maps go through one out-of-line function, so the fully unrolled feature
// loops do not carry inlined copies of expf / tanhf (the choice is uniform over a launch).
static __device__ __noinline__ float phi_act_other(float u, int act) {
    switch (act) {
        case 1: return u / (1.0f + expf(-u));
        case 2: return u;
        default: return tanhf(u);
    }
}
__device__ __forceinline__ float phi_act(float u, int act) {
    return act == 0 ? fmaxf(u, 0.f) : phi_act_other(u, act);
}

// phi = act(u) and d phi / d u (the backward's feature maps; relu inline, the others out of line).
static __device__ __noinline__ void phi_act_grad_other(float u, int act, float& y, float& dy) {
    switch (act) {
        case 1: {
            const float sg = 1.0f / (1.0f + expf(-u));
            y = u * sg;
            dy = sg * (1.0f + u * (1.0f - sg));
            return;
        }
        case 2: y = u; dy = 1.0f; return;
        default: {
            // 1 - tanh^2 = 4 e / (1 + e)^2 with e = exp(-2|u|): no cancellation where tanh saturates
            // (1 - t * t in fp32 loses all digits of a derivative below ~1e-6)
            const float e = expf(-2.0f * fabsf(u));
            y = tanhf(u);
            dy = 4.0f * e / ((1.0f + e) * (1.0f + e));
            return;
        }
    }
}
__device__ __forceinline__ void phi_act_grad(float u, int act, float& y, float& dy) {
    if (act == 0) {
        y = fmaxf(u, 0.f);
        dy = u > 0.f ? 1.f : 0.f;
    } else {
        phi_act_grad_other(u, act, y, dy);
    }
}

// One rotation pair (features 2p, 2p+1) of the low-rank branch, forward and backward, for every
// ordering of the RoPE and the activation.  (c, s) is the pair's rotation ((1, 0) without the
// low-rank RoPE).  RoPE outside the activation: phi = act(u), psi = R phi, normaliser feature nf = phi;
// inside: r = R u, psi = act(r), nf = psi.  a0, a1: the activation's derivative at its input.
struct LrPair {
    float psi0, psi1, nf0, nf1, a0, a1;
};
__device__ __forceinline__ LrPair lr_pair_fwd(float u0, float u1, float c, float s, int act, int inside) {
    LrPair p;
    if (inside) {
        phi_act_grad(u0 * c - u1 * s, act, p.psi0, p.a0);
        phi_act_grad(u0 * s + u1 * c, act, p.psi1, p.a1);
        p.nf0 = p.psi0;
        p.nf1 = p.psi1;
    } else {
        phi_act_grad(u0, act, p.nf0, p.a0);
        phi_act_grad(u1, act, p.nf1, p.a1);
        p.psi0 = p.nf0 * c - p.nf1 * s;
        p.psi1 = p.nf0 * s + p.nf1 * c;
    }
    return p;
}
// du = d loss / d u of the pair, from the gradients reaching psi (dpsi) and the normaliser feature (dnf).
__device__ __forceinline__ void lr_pair_bwd(const LrPair& p, float dpsi0, float dpsi1, float dnf0, float dnf1,
                                            float c, float s, int inside, float& du0, float& du1) {
    if (inside) {  // d r = (dpsi + dnf) act'(r), du = R^T d r
        const float dr0 = (dpsi0 + dnf0) * p.a0, dr1 = (dpsi1 + dnf1) * p.a1;
        du0 = c * dr0 + s * dr1;
        du1 = -s * dr0 + c * dr1;
    } else {  // d phi = R^T dpsi + dnf, du = d phi act'(u)
        du0 = (c * dpsi0 + s * dpsi1 + dnf0) * p.a0;
        du1 = (-s * dpsi0 + c * dpsi1 + dnf1) * p.a1;
    }
}

// 3D RoPE schedule: pair j rotates with the position along axis[j]; its cos/sin for position p
// (0-based grid coordinate; the constant offset is folded into the table) is tab[tab_off[j] + p].
struct RopeMeta {
    int npairs;
    int axis[kMaxPairs];
    int mloc[kMaxPairs];   // index of the pair within its axis
    int apairs[3];         // pairs per axis
    int tab_off[kMaxPairs];
    int axis_len[3];       // T, H, W
    long long off[3];      // position offsets
    double theta;
};

__host__ __device__ inline int token_axis_pos(int n, int axis, int H, int W) {
    return axis == 0 ? n / (H * W) : (axis == 1 ? (n / W) % H : n % W);
}

// ---- launchers (defined in prep_kernels.cu and attn_sm100.cu) --------------------------------
cudaError_t launch_rope_table(double2* tab, int2* pairs, const RopeMeta& meta, int entries, cudaStream_t st);
// write_v: also the fp16 head-major v copy (for the backward kernels; the forward reads v itself).
cudaError_t launch_rope_pool(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                             const double2* tab, const int2* pairs, const Geom& g, bool write_v, __half* qh,
                             __half* kh, __half* vh, double* qbar, double* kbar, int* status,
                             unsigned long long timeout_ns, cudaStream_t st);
cudaError_t launch_select(const double* qbar, const double* kbar, const Geom& g, int32_t* idx, uint8_t* tie,
                          cudaStream_t st);
cudaError_t launch_lowrank_partial(const __nv_bfloat16* k, const __nv_bfloat16* v, const __nv_bfloat16* A,
                                   const double2* tab, const int2* pairs, const Geom& g, int nsplit,
                                   float* s_part, float* z_part, cudaStream_t st);
// Tensor-core low-rank partial sums (head_dim 128), see lowrank_sm100.cu.
cudaError_t launch_lowrank_tc(const __nv_bfloat16* k, const __nv_bfloat16* v, const __nv_bfloat16* A,
                              const double2* tab, const RopeMeta& meta, const Geom& g, int nsplit, float* s_part,
                              float* z_part, int* status, unsigned long long timeout_ns, int debug_unsatisfied_wait,
                              cudaStream_t st);
int lowrank_nsplit(const Geom& g);
bool make_map_headmajor(CUtensorMap* m, const void* base, uint64_t rows, int D, int box_rows);
bool make_map_tokens(CUtensorMap* m, const void* base, int B, int L, int Hh, int D, const Strides& st, int box_tokens);
bool make_map_out(CUtensorMap* m, void* base, int B, int L, int Hh, int D, const Strides& st, bool f32);
cudaError_t launch_lowrank_reduce(const float* s_part, const float* z_part, const Geom& g, int nsplit, float* S,
                                  float* z, const __nv_bfloat16* A, uint8_t* at_img, uint8_t* sb_img, cudaStream_t st);

// fp16 head-major [BH*Lp][D] tensor maps; q box 64 x 128 rows, k/v box 64 x `block` rows, 128-B swizzle.
struct AttnMaps {
    CUtensorMap q, k, v;
    CUtensorMap q_raw;  // 4D map over the raw bf16 queries [B][L][Hh][D], box 64 x 1 x 128 x 1
    CUtensorMap out;    // 4D map over out [B][L][Hh][D] (fp32: box 32 x 1 x 64 x 1; bf16: 64 x 1 x 64 x 1)
    CUtensorMap os;     // with AttnArgs::os_save: fp32 map over the saved sparse output (head-major)
};

// Operand images for the tensor-core low-rank readout (head_dim 128), built by the reduction:
//   A^T image: [R rows][128] bf16 K-major, 128-B swizzled (R*256 bytes);
//   S image per (batch*head, 64-feature chunk): [D rows][3*rc] bf16 K-major swizzled, the K columns
//   holding (S_hi, S_lo, S_hi) of the chunk's rc features (kSbChunkBytes apart).
constexpr int kSbChunkBytes = 3 * 128 * 128;

struct AttnArgs {
    const __half* qh;   // head-major fp16 q^, k^ rows [B*Hh][Lp][D] (read through the TMA maps; v tiles come
    const __half* kh;   // from the caller's token-major v)
    const int32_t* idx;
    int keep;  // 0: no sparse branch
    const __nv_bfloat16* q_raw;
    const __nv_bfloat16* A;
    const float* S;
    const float* z;
    const double2* tab;
    const int2* pairs;  // per rotary pair: (axis, offset of its cos/sin table)
    int2 pair_info[kMaxPairs];  // the same, as a launch parameter (read through the constant cache)
    const uint8_t* at_img;  // A^T operand image (head_dim 128)
    const uint8_t* sb_img;  // S operand images (head_dim 128)
    int lowrank;  // add the low-rank readout
    int gated;    // gated fusion of the branches instead of their sum (both branches on)
    float gate_b;
    const float* gate_w;  // [D]
    void* out;
    int out_bf16;
    int* status;
    unsigned long long timeout_ns;
    int debug_unsatisfied_wait;  // test hook: wait on a barrier nothing signals before any work
    float* lse;  // optional fp32 [B*Hh][Lp]: per query row m + log2(l) of the sparse softmax in the kernel's
                 // log2 units (P_ij = 2^(s_ij log2(e) / sqrt(D) - lse_i)); +inf for rows past L
    float* os_save;  // optional: the sparse branch's own output O_s = O / l, stored through AttnMaps::os
                     // before the low-rank readout joins O (for a backward pass)
};
cudaError_t launch_attn(const AttnMaps& m, const AttnArgs& a, const Geom& g, cudaStream_t st);
size_t attn_smem_bytes(const Geom& g);

// ---- backward pass (bwd_sm100.cu) --------------------------------------------------------------
struct BwdArgs {
    const int32_t* idx;      // [BH][nb][keep] kept key blocks per query block, ascending
    int keep;
    const int32_t* inv;      // [BH][nb][nb] query blocks that kept each key block, ascending
    const int32_t* inv_cnt;  // [BH][nb]
    const float* lse;        // [BH][Lp] (log2 units; +inf for rows past L)
    const float* delta;      // [BH][Lp] dO . O_sparse per row
    const double2* tab;      // rotary cos/sin table
    int2 pair_info[kMaxPairs];
    float* dq;  // token-major fp32 [B][L][Hh][D] (strides g.so)
    float* dk;
    float* dv;
    int accumulate;  // 1: add to the rows (the low-rank part is already there); 0: store them
    int* status;
    unsigned long long timeout_ns;
};
// fp16 head-major maps (128-B swizzle): 128-row boxes for the tiles that are an MMA's M side, block-row
// boxes for the others; `between` (optional) is recorded between the dQ and the dK/dV kernels.
struct BwdMaps {
    CUtensorMap q128, do128, kb, vb;  // dQ kernel
    CUtensorMap k128, v128, qb, dob;  // dK/dV kernel
    cudaEvent_t between;
};
struct LrBwdArgs {
    // A: the projections as the forward takes them, [1 + proj_separate][proj_per_head ? Hh : 1][D][R]
    // (per head: head h at A + h * g.a_stride; the key projection after the query projection(s))
    const __nv_bfloat16 *q, *k, *v, *A;
    int proj_separate, proj_per_head;
    const float* dout;
    const float *S, *z;
    const double2* tab;
    const int2* pairs;
    float *dq, *dk, *dv, *dA;
    float *ds_part, *dz_part, *da_part, *dS, *dz;
    int nsplit;
    const RopeMeta* meta;  // rotary schedule (tensor-core passes)
    int* status;
    unsigned long long timeout_ns;
    int accumulate;  // 1 adds dq, dk, dv to the rows (the sparse part is there); 0 stores them
    // dA: [1 + proj_separate][proj_per_head ? Hh : 1][D][R], the partials reduced in a fixed order
    long long key_proj_offset(const Geom& g) const {
        return proj_separate ? static_cast<long long>(proj_per_head ? g.Hh : 1) * g.D * g.R : 0;
    }
};
cudaError_t launch_bwd_prep(const float* dout, const float* os, const Geom& g, __half* doh, float* delta, int* status,
                            cudaStream_t st);
cudaError_t launch_bwd_invert(const int32_t* idx, const Geom& g, int32_t* inv, int32_t* inv_cnt, cudaStream_t st);
cudaError_t launch_bwd_sparse(const BwdMaps& m, const BwdArgs& a, const Geom& g, cudaStream_t st);
cudaError_t launch_lr_bwd(const LrBwdArgs& l, const Geom& g, cudaStream_t st);
// Tensor-core low-rank gradient passes (head_dim 128, rank <= 64), see lr_bwd_sm100.cu.
cudaError_t launch_lr_bwd_tc(const LrBwdArgs& l, const Geom& g, cudaStream_t st);
inline bool lr_bwd_on_tensor_cores(const Geom& g) { return g.D == 128 && g.R <= 64; }
int lr_bwd_nsplit(const Geom& g);

// ---- backward of the gated fusion (gate_bwd.cu) -------------------------------------------------
constexpr int kGateParts = 148 * 8;  // CTAs (and partial sums) of the gate-parameter reduction
// dO_s (fp16 head-major copy and Delta), dO_lr (fp32 token-major) and dlogit per row from dout, O_s and
// O_lr (head-major fp32) and the raw queries.
cudaError_t launch_gate_prep(const float* dout, const float* os, const float* olr, const __nv_bfloat16* q,
                             const float* gate_w, float gate_b, const Geom& g, __half* doh, float* delta, float* dolr,
                             float* dlogit, int* status, cudaStream_t st);
// dq += dlogit Wg; dWg, dbg (part: kGateParts x (D + 1) floats of scratch).
cudaError_t launch_gate_final(const __nv_bfloat16* q, const float* dlogit, const float* gate_w, const Geom& g,
                              float* dq, float* part, float* dgw, float* dgb, cudaStream_t st);

}  // namespace slra
