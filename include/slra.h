/*
 * slra.h - C ABI of libslra.so: the forward pass of 3D-RoPE sparse + low-rank hybrid attention for
 * video diffusion transformers, as hand-written CUDA for NVIDIA B200 (sm_100a).
 *
 * What it computes (page titles and sections of the method's sources):
 *   RoLA: Rotary-Positioned Low-Rank Linear Attention for Efficient Diffusion Transformers
 *     - "3 Preliminary": a video latent T x H x W is flattened to L = T*H*W tokens (row-major t,h,w);
 *       3D RoPE splits each head across the t, h, w axes and makes q.k depend on relative offsets
 *       (eq. (1)).
 *     - "4.1": a block-sparse softmax branch for the high-energy "spikes" plus a low-rank branch whose
 *       global context is computed once per head at O(L r d_h) cost.
 *     - "4.2": the low-rank branch reuses the first r rotary coordinates (r/2 complete pairs) of the
 *       backbone's own schedule; "4.3": that rotation is applied OUTSIDE the nonlinearity, so the
 *       summary stays query-independent ("B.1").
 *   RoPeSLR: 3D RoPE-driven Sparse-LowRank Attention for Efficient Diffusion Transformers
 *     - appendix on 3D RoPE: rotary base 10000, head dimension partitioned over (t, x, y).
 *
 *   qh, kh      = 3D RoPE of q, k (pairs (2j, 2j+1); pairs split t/h/w = c-2*floor(c/3), floor(c/3),
 *                 floor(c/3) with c = D/2, i.e. 44/42/42 dims at D = 128; omega = theta^(-2m/d_axis))
 *   qbar, kbar  = mean of qh, kh over each block of `block` tokens (last block: its real tokens)
 *   K(alpha)    = the k = clamp(round(keep_frac * nb), 1, nb) key blocks with the largest
 *                 qbar_alpha . kbar_beta, ties to the lower block index
 *   O_sparse_i  = softmax_j(qh_i . kh_j / sqrt(D)) v_j over the keys of K(alpha(i))
 *   phi(x)      = relu(x P) on raw q, k (or SiLU / identity / tanh, slra_problem.activation), with
 *                 P = Pq for queries and Pk for keys (one shared matrix A by default; separate and
 *                 per-head projections are options, see slra_problem.proj_separate / proj_per_head);
 *               psi = phi with its first r coordinates rotated like RoPE (unless lowrank_norope)
 *   S = sum_j psi(k_j) v_j^T (r x D),  z = sum_j phi(k_j)   (all L keys, per head)
 *   O_lowrank_i = psi(q_i)^T S / (phi(q_i) . z + 1e-6)
 *   out         = O_sparse + O_lowrank   (or, with slra_problem.fusion = SLRA_FUSION_GATED, RoLA "4.4"'s
 *                 token-wise gate: out_i = O_sparse,i + g_i O_lowrank,i rms(O_sparse,i) /
 *                 sqrt(mean(O_lowrank,i^2) + 1e-6), g_i = sigmoid(q_i . Wg + bg) on the raw query; the
 *                 pages print no formula, this is the library's reading of their description)
 *
 * Conventions for every entry point:
 *   - Device pointers unless stated otherwise.  The caller owns every buffer; nothing the caller
 *     passes is retained after a call returns (the library itself keeps, per device, the two copy
 *     streams and a few events slra_attn_fwd_host creates on first use, the side stream and its two
 *     events the forward uses to overlap the two branches' preparation, and the fixed scratch array
 *     of slra_lowrank_summary_noalloc).  Calls are asynchronous on `stream` (NULL = the legacy default
 *     stream) and never synchronize, except slra_device_status and slra_attn_fwd_host.
 *   - All arguments are validated before anything is launched; an invalid call returns a status and
 *     launches nothing.  Launch failures return SLRA_ERR_CUDA.
 *   - Problems detected on the device (an input too large for the fp16 operands, a bounded wait that
 *     ran out) are recorded in a status word inside the workspace and reported by
 *     slra_device_status.
 *   - A workspace may be used by one call at a time (calls on one stream are ordered; calls on
 *     different streams need different workspaces).  Where an entry point takes a workspace, NULL
 *     means the library allocates one with cudaMallocAsync on `stream` (the current device's memory
 *     pool) and frees it with cudaFreeAsync after its launches, both stream-ordered; the call's device
 *     status then goes to slra_get_device_status instead.  Raising the release threshold of the
 *     device's default pool (cudaMemPoolAttrReleaseThreshold) keeps that memory between calls.
 *   - q, k, v and out are [B][L][Hh][D] with the D elements of a row contiguous; their batch, token and
 *     head strides (in elements) are free (e.g. q, k, v as views of one fused QKV buffer), contiguous
 *     token-major by default.  Input strides must be positive multiples of 8 elements (16 bytes of
 *     bf16), output strides multiples of 16 bytes of the output type, all below 2^36, and distinct
 *     output rows may not overlap.
 */
#ifndef SLRA_H
#define SLRA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SLRA_ABI_VERSION 8

/* Exported symbols (the library is built with hidden visibility for everything else). */
#if defined(__GNUC__)
#define SLRA_API __attribute__((visibility("default")))
#else
#define SLRA_API
#endif

/* cudaStream_t without including the CUDA headers. */
typedef struct CUstream_st* slra_stream_t;

typedef enum slra_status {
    SLRA_OK = 0,
    SLRA_ERR_INVALID_ARG = 1,     /* NULL pointer, non-positive size, L overflow, keep_frac outside (0,1] */
    SLRA_ERR_UNSUPPORTED = 2,     /* valid but not implemented: head_dim, block, rank, more than 2048
                                     blocks, more than 65535 batch x heads                               */
    SLRA_ERR_ALIGNMENT = 3,       /* a pointer is not 16-byte aligned                                   */
    SLRA_ERR_WORKSPACE = 4,       /* workspace NULL, misaligned (256 B) or smaller than required         */
    SLRA_ERR_CUDA = 5,            /* a CUDA runtime/driver call or a kernel launch failed                */
    SLRA_ERR_DEVICE_TIMEOUT = 6,  /* (device status) a bounded wait inside a kernel ran out              */
    SLRA_ERR_RANGE = 7,           /* (device status) a value does not fit the fp16 operands: |value| >=
                                     65504 after RoPE, or a block of q^, k^ or (where an fp16 copy of v
                                     is made) v whose nonzero values all lie below fp16's smallest
                                     normal 2^-14 (relative precision lost)                              */
    SLRA_ERR_NO_DEVICE = 8,       /* no sm_100 device is current                                         */
    SLRA_ERR_SCRATCH_LIMIT = 9    /* slra_lowrank_summary_noalloc: problem exceeds its fixed scratch area */
} slra_status;

typedef enum slra_out_dtype { SLRA_OUT_F32 = 0, SLRA_OUT_BF16 = 1 } slra_out_dtype;

/* Element type of a tensor descriptor. */
typedef enum slra_dtype { SLRA_DTYPE_BF16 = 0, SLRA_DTYPE_F32 = 1 } slra_dtype;

/*
 * A [B][L][Hh][D] device tensor (batch, token, head, head dimension): `data` points at element
 * (0, 0, 0, 0); element (b, n, h, d) sits at data + b*sB + n*sL + h*sH + d (strides in elements; all
 * three zero = contiguous, i.e. sH = D, sL = Hh*D, sB = L*Hh*D).  The library only reads the inputs.
 */
typedef struct slra_tensor {
    void* data;
    int32_t dtype;  /* slra_dtype */
    int64_t B, L, Hh, D;
    int64_t sB, sL, sH;
} slra_tensor;

/* A [D][R] row-major device matrix: the low-rank projection A shared by queries, keys and heads. */
typedef struct slra_mat {
    const void* data;
    int32_t dtype;  /* slra_dtype: bf16 */
    int64_t D, R;
} slra_mat;

/* Which branches contribute to `out` (default both). */
enum { SLRA_BRANCH_SPARSE = 1, SLRA_BRANCH_LOWRANK = 2, SLRA_BRANCH_BOTH = 3 };

/* Test hooks (slra_problem.debug_flags).  SLRA_DEBUG_UNSATISFIED_WAIT makes every CTA of the attention
 * kernel and of the tensor-core low-rank summary kernel (head_dim 128) first wait on a barrier that
 * nothing signals, so the bounded-wait path (timeout recorded in the status word, the CTA returns
 * without issuing work) can be exercised without faulting or hanging the GPU.  Use a small
 * wait_timeout_ns with it. */
enum { SLRA_DEBUG_UNSATISFIED_WAIT = 1, SLRA_DEBUG_SERIAL_BRANCHES = 2 };
/* SLRA_DEBUG_SERIAL_BRANCHES: run the two branches' preparation one after the other on the calling
 * stream instead of overlapping them (see slra_attn_fwd_ex), so stage_events time each kernel alone. */

/* Nonlinearity of the low-rank feature map phi = act(x A) (slra_problem.activation).  RELU is the
 * benchmark's map; SILU (u / (1 + e^-u)), IDENTITY and TANH are the alternatives RoLA's ablation
 * compares ("5.3", Table 6).  With IDENTITY or TANH the normaliser phi(q) . sum_j phi(k_j) + 1e-6 can
 * come close to zero; the library computes it as defined and does not guard it. */
/* How the two branches are combined (slra_problem.fusion). */
typedef enum slra_fusion { SLRA_FUSION_SUM = 0, SLRA_FUSION_GATED = 1 } slra_fusion;

typedef enum slra_activation {
    SLRA_ACT_RELU = 0,
    SLRA_ACT_SILU = 1,
    SLRA_ACT_IDENTITY = 2,
    SLRA_ACT_TANH = 3
} slra_activation;

/*
 * Problem description.  Fill it with slra_problem_init, then adjust optional fields.
 *   batch, heads, head_dim  B, Hh, D.  D in {64, 128}.
 *   T, H, W                 latent grid; L = T*H*W tokens (row-major t, h, w).
 *   block                   tokens per block for both queries and keys; 64 or 128.
 *   keep_frac               kept fraction of key blocks per query block, in (0, 1].
 *   rank                    r: multiple of 16 with 16 <= r <= D.
 *   theta                   rotary base (default 10000).
 *   out_dtype               SLRA_OUT_F32 (default) or SLRA_OUT_BF16.
 *   branches                SLRA_BRANCH_* mask (default both).
 *   pos_offset              constant added to every (t, h, w) position (default 0; RoPE makes the
 *                           result independent of it, which the tests use).
 *   rope_split              rotary pairs per (t, h, w); all zero = default split described above.
 *   wait_timeout_ns         bound of every wait inside the kernels (default 2e9 ns = 2 s).
 *   debug_flags             SLRA_DEBUG_* test hooks (default 0).
 *   stage_events            optional cudaEvent_t handles (NULL entries are skipped), recorded
 *                           between the library's launches so a caller can time each stage: [0]
 *                           before the first launch, [1] after the rotary tables, [2] after RoPE +
 *                           pooling, [3] after block selection, [4] after the low-rank partial sums,
 *                           [5] after their reduction, [6] after the attention kernel (the branch
 *                           entry points record the boundaries of the stages they run).  With both
 *                           branches on, the low-rank preparation runs on the library's side stream
 *                           concurrently with RoPE + pooling and selection: [4] is recorded there and
 *                           [5] on `stream` once both are done, so [5] -> [6] is the attention kernel
 *                           alone (SLRA_DEBUG_SERIAL_BRANCHES serialises them for per-kernel times).
 *                           The caller creates and owns them.
 *   activation              SLRA_ACT_* map of the low-rank features (default SLRA_ACT_RELU).
 *   lowrank_norope          0 (default): the low-rank branch rotates the first r feature coordinates
 *                           with the truncated 3D RoPE after the activation (RoLA "4.2", "4.3");
 *                           1: no rotation, psi = phi (the no-RoPE setting of RoLA "5.3").
 *   proj_separate           0 (default): one projection serves queries and keys; 1: separate query and
 *                           key projections Pq, Pk (the parameters RoLA "E.2" lists).
 *   proj_per_head           0 (default): one projection (or pair) for all heads; 1: one per head (the
 *                           head-wise low-rank parameterization of RoPeSLR's abstract).
 *                           Both flags only change how the A argument is laid out:
 *                           bf16 [1 + proj_separate][proj_per_head ? heads : 1][D][rank], the query
 *                           projection(s) first; slra_projection_elems gives its element count.
 *   fusion                  SLRA_FUSION_SUM (default): out = sparse + low-rank output;
 *                           SLRA_FUSION_GATED: the gated fusion above (needs both branches).
 *   gate_bias               bg of the gated fusion (a negative value starts near the sparse output).
 *   gate_w                  Wg of the gated fusion: DEVICE pointer to fp32 [D], 16-B aligned, shared by
 *                           all heads (also for slra_attn_fwd_host); NULL unless fusion is GATED.
 *   lowrank_rope_inside     0 (default); 1: the truncated RoPE is applied to the projected features
 *                           BEFORE the activation, psi = act(R_r(p) x P), and the normaliser uses psi
 *                           too: the ordering RoLA's ablation compares against ("5.1" Table 2, "5.3",
 *                           "B.3"); the summary stays linear but loses the relative property.  Not
 *                           with lowrank_norope.
 *   q_strides, k_strides,   (sB, sL, sH) element strides of q, k, v and out (see the conventions at the
 *   v_strides, out_strides  top); all zero (default) = contiguous [B][L][Hh][D].  slra_attn_fwd_host
 *                           takes contiguous host buffers only.
 */
typedef struct slra_problem {
    int64_t batch, heads, head_dim;
    int64_t T, H, W;
    int64_t block;
    double keep_frac;
    int64_t rank;
    double theta;
    int32_t out_dtype;
    int32_t branches;
    int64_t pos_offset[3];
    int64_t rope_split[3];
    uint64_t wait_timeout_ns;
    uint32_t debug_flags;
    void* stage_events[7];
    int32_t activation;
    int32_t lowrank_norope;
    int32_t proj_separate;
    int32_t proj_per_head;
    int32_t fusion;
    float gate_bias;
    const void* gate_w;
    int32_t lowrank_rope_inside;
    int64_t q_strides[3], k_strides[3], v_strides[3], out_strides[3];
    void* dgate_w;  /* backward, gated fusion: output fp32 [head_dim], d loss / d Wg (16-B aligned) */
    void* dgate_b;  /* backward, gated fusion: output fp32 [1], d loss / d bg (4-B aligned) */
} slra_problem;

/*
 * Where the intermediates live inside a workspace (byte offsets from its start; all 256-B aligned).
 * They are valid after a forward call and may be read for inspection:
 *   qh, kh, vh   fp16 [B*Hh][nb*block][D]  rotated q, k and fp16 copy of v, head-major, zero padded
 *                                          (vh: written by slra_select_blocks, the training forward and
 *                                          the backward; the inference forward reads v itself)
 *   qbar, kbar   fp64 [B*Hh][nb][D]        block means of qh, kh (computed in fp64)
 *   idx          int32 [B*Hh][nb][keep]    kept key blocks per query block, ascending
 *   tie          uint8 [B*Hh][nb]          1 where the k-th and (k+1)-th block scores are within
 *                                          1e-6 * max(1, |s_k|) (a numerically fragile selection)
 *   S            fp32 [B*Hh][rank][D]      low-rank summary
 *   z            fp32 [B*Hh][rank]         sum of the unrotated key features
 *   status       int32                     device status word (see slra_device_status)
 */
typedef struct slra_ws_layout {
    size_t total_bytes;
    int64_t L, nb, keep, nsplit;
    size_t status, rope_table, qh, kh, vh, qbar, kbar, idx, tie, s_part, z_part, S, z;
} slra_ws_layout;

/* ABI version (SLRA_ABI_VERSION).  Never fails. */
SLRA_API int slra_abi_version(void);

/* Static, human-readable name of a status code.  Never returns NULL. */
SLRA_API const char* slra_status_string(int status);

/* Fill *p with the given sizes and the defaults above.  Returns SLRA_ERR_INVALID_ARG if p is NULL. */
SLRA_API slra_status slra_problem_init(slra_problem* p, int64_t batch, int64_t heads, int64_t head_dim, int64_t T,
                              int64_t H, int64_t W, int64_t block, double keep_frac, int64_t rank);

/* Check a problem description without touching the GPU.  SLRA_OK or the reason it is rejected. */
SLRA_API slra_status slra_validate(const slra_problem* p);

/* Kept key blocks per query block, k = clamp(floor(keep_frac * nb + 0.5), 1, nb); -1 if invalid. */
SLRA_API int64_t slra_keep_count(const slra_problem* p);

/* Number of bf16 elements the projection argument A holds:
 * (1 + proj_separate) * (proj_per_head ? heads : 1) * head_dim * rank; -1 if the problem is invalid. */
SLRA_API int64_t slra_projection_elems(const slra_problem* p);

/* Workspace size and the offsets of the intermediates in it.  No GPU access. */
SLRA_API slra_status slra_workspace_layout(const slra_problem* p, slra_ws_layout* layout);

/*
 * Workspace bytes of a forward call with these sizes (the same value slra_workspace_layout gives for a
 * problem with the default options); 0 if the sizes are invalid.  No GPU access.
 */
SLRA_API size_t slra_workspace_bytes(int64_t batch, int64_t heads, int64_t head_dim, int64_t T, int64_t H,
                                     int64_t W, int64_t block, float keep_frac, int64_t rank);

/*
 * Full forward pass, all steps listed at the top of this file (RoLA "4.1": block-sparse softmax
 * branch over the top-k key blocks by block-mean-pooled post-RoPE scores, plus the low-rank branch
 * with the rank-truncated RoPE outside the relu feature map, "4.2", "4.3"; the two outputs summed).
 *   q, k, v    bf16 descriptors of equal shape [B][L][Hh][D], L = T*H*W; any strides per the
 *              conventions above (e.g. three views of one fused QKV projection output).
 *   A          bf16 [D][rank] projection shared by queries, keys and heads.
 *   T, H, W    latent grid (row-major t, h, w); block in {64, 128}; keep_frac in (0, 1] (widened to
 *              double: k = clamp(floor(keep_frac * nb + 0.5), 1, nb)); rank a multiple of 16, <= D.
 *   out        fp32 or bf16 descriptor of the same shape; may not overlap q, k, v or A.
 * The library allocates its workspace on `stream` (see the conventions) and leaves the device status
 * to slra_get_device_status.  Asynchronous; the default options of slra_problem apply.
 */
SLRA_API slra_status slra_attn_fwd(const slra_tensor* q, const slra_tensor* k, const slra_tensor* v,
                                   const slra_mat* A, int T, int H, int W, int block, float keep_frac, int rank,
                                   slra_tensor* out, slra_stream_t stream);

/*
 * The forward pass with every option of the problem struct: feature map, RoPE ordering, projection layouts,
 * gated fusion, branches, strides, timing events, test hooks.
 *   q, k, v    bf16 [B][L][Hh][D] device tensors, 16-B aligned, strides from p (contiguous by default).
 *   A          bf16 projection(s), contiguous, 16-B aligned: [D][rank] shared by q, k and all heads by
 *              default; [1 + proj_separate][proj_per_head ? Hh : 1][D][rank] in general (query
 *              projections first, then key projections).  May be NULL when the low-rank branch is off.
 *   out        [B][L][Hh][D], fp32 or bf16 as p->out_dtype, strides from p; must not overlap the
 *              inputs or the workspace.
 *   workspace  device buffer of at least layout.total_bytes bytes, 256-B aligned, or NULL (allocated
 *              by the library, see the conventions).
 * Launches 6 kernels on `stream` (tables, RoPE + pooling, selection, low-rank partial sums and their
 * reduction, attention with the fused low-rank readout) and returns without synchronizing.
 */
SLRA_API slra_status slra_attn_fwd_ex(const slra_problem* p, const void* q, const void* k, const void* v,
                                      const void* A, void* out, void* workspace, size_t workspace_bytes,
                                      slra_stream_t stream);

/*
 * The sparse branch alone (RoLA "4.1": softmax attention of each query block over its top-k key blocks,
 * selected by block-mean-pooled post-RoPE scores): out = O_sparse.  Arguments as slra_attn_fwd; the
 * workspace holds slra_workspace_bytes(B, Hh, D, T, H, W, block, keep_frac, 16) bytes (the branch has no
 * rank; 16 sizes the unused low-rank sections) or is NULL.
 */
SLRA_API slra_status slra_sparse_fwd(const slra_tensor* q, const slra_tensor* k, const slra_tensor* v, int T,
                                     int H, int W, int block, float keep_frac, slra_tensor* out, void* workspace,
                                     size_t workspace_bytes, slra_stream_t stream);

/*
 * The low-rank branch alone (RoLA "4.1", "4.2", "4.3", "B.1"): out = psi(q)^T S / (phi(q) . z + 1e-6)
 * with S = sum_j psi(k_j) v_j^T and z = sum_j phi(k_j) over all L keys.  Arguments as slra_attn_fwd;
 * S (fp32 [B*Hh][rank][D]) and z (fp32 [B*Hh][rank]) receive the summary when not NULL (16-B aligned).
 * The workspace holds slra_workspace_bytes(B, Hh, D, T, H, W, 128, 1e-4f, rank) bytes (the branch does
 * not select blocks; these values size the unused sections) or is NULL.
 */
SLRA_API slra_status slra_lowrank_fwd(const slra_tensor* q, const slra_tensor* k, const slra_tensor* v,
                                      const slra_mat* A, int T, int H, int W, int rank, slra_tensor* out, float* S,
                                      float* z, void* workspace, size_t workspace_bytes, slra_stream_t stream);

/*
 * Workspace bytes of slra_attn_bwd, slra_attn_bwd_saved and slra_attn_fwd_train for p (the forward's
 * layout followed by the backward's sections: the sparse output and its per-row log-sum-exp, an fp16
 * copy of dout, the inverted kept-block lists and the low-rank gradient partial sums; with the gated
 * fusion also the low-rank output, its gradient and the gate's per-row terms and partial sums); 0 if p
 * is invalid or has output strides (the backward's gradients are contiguous).  No GPU access.
 */
SLRA_API size_t slra_bwd_workspace_bytes(const slra_problem* p);

/*
 * Backward pass: the gradients of sum(dout * out) with respect to q, k, v and A, where out is the
 * forward pass of slra_attn_fwd_ex on the same arguments (RoLA "4.5", "E.1", "E.2": the branch's
 * parameters are trained jointly with the backbone).  The block selection is held at the forward's (it
 * is piecewise constant in q and k).  Every option of the forward is covered: the feature maps, the
 * RoPE orderings, separate and per-head projections (dA then has A's layout), any branches mask, and
 * the gated fusion, whose parameter gradients go to p->dgate_w (fp32 [head_dim], 16-B aligned) and
 * p->dgate_b (one fp32), both required then and disjoint from every other argument.
 *   q, k, v, A   as for slra_attn_fwd_ex (q, k, v may be strided per p).
 *   dout         fp32 [B][L][Hh][D] contiguous: the gradient of the loss with respect to out.
 *   dq, dk, dv   fp32 [B][L][Hh][D] contiguous outputs (p->out_strides must be zero).
 *   dA           fp32 output in the projection argument's layout, slra_projection_elems(p) elements
 *                (zero when the low-rank branch is off).
 *   workspace    at least slra_bwd_workspace_bytes(p) bytes, 256-B aligned (the forward's sections are
 *                refilled by the recompute and can be inspected afterwards).
 * The sparse branch's gradients run on the tensor cores: a dQ kernel per query block (S = q^ k^T and
 * dP = dO v^T in TMEM, dS = P (dP - rowsum(dO O_sparse)), dQ^ += dS k^) and a dK/dV kernel per key block
 * over the query blocks that kept it (dV += P^T dO, dK^ += dS^T q^), with fp16 operands (dout must stay
 * below 65504 in magnitude, else SLRA_ERR_RANGE is recorded) and fp32 accumulation; the low-rank chain
 * follows as a pass over the queries and one over the keys (on the tensor cores for head_dim 128 and
 * rank <= 64, fp32 otherwise) that add their parts to dq, dk, dv and produce dA.  With the gated fusion
 * the low-rank branch's output is recomputed too, one pass per row splits dout into the two branches'
 * gradients and the gate's, and a last pass adds the gate's part to dq and reduces dWg, dbg.
 * Deterministic.
 * stage_events are recorded at: [0] start, [1] after the recomputed forward, [2] after the dO copy and
 * the inverted lists, [3] after the dQ kernel, [4] after the dK/dV kernel, [5] and [6] after the
 * low-rank (and gate) gradients.  Device problems go to the workspace's status word (slra_device_status).
 */
SLRA_API slra_status slra_attn_bwd(const slra_problem* p, const void* q, const void* k, const void* v,
                                   const void* A, const float* dout, float* dq, float* dk, float* dv, float* dA,
                                   void* workspace, size_t workspace_bytes, slra_stream_t stream);

/*
 * Forward pass for training: slra_attn_fwd_ex with out contiguous (same arguments), which also keeps
 * in `workspace` what the backward would recompute: the tables, the block selection, the low-rank
 * summary and readout operands, the fp16 operand copies, each query row's log-sum-exp and the sparse
 * branch's own output (stored by the attention kernel before the low-rank readout joins it).  out is
 * bit for bit that of slra_attn_fwd_ex.  (With the gated fusion the backward still recomputes the
 * low-rank branch's output alone, a pass without the sparse loop.)
 *   workspace    at least slra_bwd_workspace_bytes(p) bytes, 256-B aligned (NULL is rejected:
 *                SLRA_ERR_WORKSPACE); its status word starts cleared, as for slra_attn_fwd_ex.
 * Pass the same workspace, untouched, to slra_attn_bwd_saved.
 */
SLRA_API slra_status slra_attn_fwd_train(const slra_problem* p, const void* q, const void* k, const void* v,
                                         const void* A, void* out, void* workspace, size_t workspace_bytes,
                                         slra_stream_t stream);

/*
 * Backward pass from a forward kept by slra_attn_fwd_train: slra_attn_bwd without the recompute (the
 * same problem and the same q, k, v, A as that forward; the workspace as it left it).  The gradients
 * are bit for bit those of slra_attn_bwd.  The workspace's status word is not cleared: it holds what
 * the forward and the backward recorded.  stage_events as for slra_attn_bwd, [1] right after [0].
 * The library cannot tell a workspace of another problem or of other inputs: the gradients are then
 * meaningless.
 */
SLRA_API slra_status slra_attn_bwd_saved(const slra_problem* p, const void* q, const void* k, const void* v,
                                         const void* A, const float* dout, float* dq, float* dk, float* dv,
                                         float* dA, void* workspace, size_t workspace_bytes,
                                         slra_stream_t stream);

/*
 * Device status of the calls whose workspace the library allocated (slra_attn_fwd, and the others when
 * given a NULL workspace) on the current device: synchronize `stream`, then read and clear the word
 * their status words were ORed into.  *status receives SLRA_OK, SLRA_ERR_DEVICE_TIMEOUT or SLRA_ERR_RANGE.
 */
SLRA_API slra_status slra_get_device_status(slra_stream_t stream, int32_t* status);

/*
 * The same forward pass on HOST buffers: copies q, k, v and A (slra_projection_elems(p) elements)
 * from host memory into `io` (a device buffer of at least slra_host_io_bytes(p) bytes), computes, and
 * copies `out` back to host memory, then synchronizes `stream`.  Host buffers should be pinned.
 * Heads are independent, so the call splits the problem into groups of heads (about sixteen per batch
 * element) and pipelines them: the upload of one group, the compute of the previous one (on `stream`)
 * and the download of the one before that overlap, on two copy streams of the library's own (created
 * on first use, one pair per device) and two device slots carved from `io` and the workspace.  When
 * two slots do not fit (or there is a single group) it copies everything in, computes and copies
 * out, all on `stream`.  The device status word of `workspace` holds the OR of all groups' status.
 * Calls on the same device are serialized inside the library; stage_events are not recorded.
 */
SLRA_API size_t slra_host_io_bytes(const slra_problem* p);
/* Number of head groups slra_attn_fwd_host will pipeline for p with the given buffer sizes (1: no
 * pipelining), or -1 if p is invalid.  No GPU access. */
SLRA_API int64_t slra_host_pipeline_groups(const slra_problem* p, size_t io_bytes, size_t workspace_bytes);
SLRA_API slra_status slra_attn_fwd_host(const slra_problem* p, const void* q_host, const void* k_host,
                               const void* v_host, const void* A_host, void* out_host, void* io,
                               size_t io_bytes, void* workspace, size_t workspace_bytes, slra_stream_t stream);

/*
 * Block selection only (3D RoPE, block means, scores, top-k): fills the qh/kh/vh, qbar/kbar, idx and
 * tie sections of the workspace.  Same argument rules as slra_attn_fwd_ex (the workspace is required).
 */
SLRA_API slra_status slra_select_blocks(const slra_problem* p, const void* q, const void* k, const void* v,
                               void* workspace, size_t workspace_bytes, slra_stream_t stream);

/*
 * Low-rank summary only (RoLA "4.1", "B.1"): fills the S and z sections of the workspace from raw k,
 * v and A.  Same argument rules as slra_attn_fwd_ex (the workspace is required).
 */
SLRA_API slra_status slra_lowrank_summary(const slra_problem* p, const void* k, const void* v, const void* A,
                                 void* workspace, size_t workspace_bytes, slra_stream_t stream);

/*
 * Synchronize `stream`, then read and clear the device status word of `workspace`.  *status receives
 * SLRA_OK, SLRA_ERR_DEVICE_TIMEOUT or SLRA_ERR_RANGE.  Every compute entry point clears the word when it
 * starts, so this reports the calls made since the last compute call began (a timeout wins over a
 * range problem).
 */
SLRA_API slra_status slra_device_status(void* workspace, slra_stream_t stream, int32_t* status);

/*
 * Low-rank summary without any allocation: S = sum_j psi(k_j) v_j^T and z = sum_j phi(k_j), the same
 * result as slra_lowrank_summary (up to the order of the fp32 partial sums), written straight into
 * caller buffers and using no workspace.  The method's sources have no counterpart to this entry
 * point; it exists for callers that cannot allocate device memory at the point of the call: code
 * running inside a framework that hands out device memory only through its own pool and forbids side
 * allocations, plugin-style execute hooks that must not allocate, and latency-critical serving loops
 * where cudaMalloc/cudaFree would synchronize the device and stall other streams.
 *
 *   k, v     bf16 [B][L][Hh][D], 16-B aligned (device), strides from p (contiguous by default).
 *   A        bf16 projection(s) laid out as for slra_attn_fwd_ex, 16-B aligned (device); the summary
 *            uses the key projection(s).
 *   S        fp32 [B*Hh][rank][D] output (device, 16-B aligned).
 *   z        fp32 [B*Hh][rank]    output (device, 16-B aligned).
 *
 * Scratch (the rotary tables and the split-L partial sums) lives in one fixed array of
 * SLRA_NOALLOC_SCRATCH_BYTES (16 MiB) compiled into the library: every GPU that loads the library
 * holds that array until the process exits.  The number of sequence splits is reduced until the
 * partial sums fit; a problem whose partial sums do not fit even unsplit
 * (B*Hh*rank*(D+1)*4 bytes plus the tables over the limit) is rejected with SLRA_ERR_SCRATCH_LIMIT
 * before anything is launched.  The call performs no cudaMalloc, cudaFree or other allocation.
 *
 * The first call on each device looks up the array's device address (cudaGetSymbolAddress, with
 * that device current) and caches it for the life of the process; make that first call before any
 * stream capture, and do not keep using the entry point after a cudaDeviceReset of that device (the
 * cached address would then be stale).  All calls share the one array, which keeps the last call's
 * contents.  Each call first clears the array's status word (an asynchronous memset on `stream`);
 * every other scratch byte a call reads it has first written itself, so nothing left by an earlier
 * call is used.  Calls that overlap on the GPU (on different streams, or from different host threads
 * without ordering) race on the array and must be serialized by the caller.
 *
 * Problems detected on the device (a bounded wait inside the summary kernel that ran out) are
 * recorded in the array's status word: read them with slra_noalloc_device_status.  After a timeout
 * S and z are unspecified.
 */
#define SLRA_NOALLOC_SCRATCH_BYTES (16u << 20)
SLRA_API slra_status slra_lowrank_summary_noalloc(const slra_problem* p, const void* k, const void* v,
                                                  const void* A, float* S, float* z, slra_stream_t stream);

/*
 * Device status of slra_lowrank_summary_noalloc on the current device: synchronize `stream`, then
 * read and clear the status word of the fixed scratch array.  *status receives SLRA_OK or
 * SLRA_ERR_DEVICE_TIMEOUT (the calls since the last no-allocation call began).  Allocates nothing.
 * Like the entry point itself, this has no counterpart in the method's sources.
 */
SLRA_API slra_status slra_noalloc_device_status(slra_stream_t stream, int32_t* status);

#ifdef __cplusplus
}
#endif

#endif /* SLRA_H */
