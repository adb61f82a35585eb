// C ABI of libslra.so (declared in include/slra.h): argument validation, workspace layout, TMA
// descriptors and the launch sequence of the hybrid attention forward.
#include <cudaTypedefs.h>

#include <algorithm>
#include <utility>
#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/slra.h"
#include "common.cuh"

using namespace slra;

namespace slra {
// The pipelined host call's device status: each group's status word ORed into the caller's.
__global__ void status_or_kernel(int* acc, const int* src) {
    const int v = *src;
    if (v) atomicOr(acc, v);
}

// Device status of the calls whose workspace the library allocated (and freed) itself: their status
// words are ORed here before the workspace goes back to the pool (slra_get_device_status reads it).
__device__ int g_call_status;
__global__ void status_or_global_kernel(const int* src) {
    const int v = *src;
    if (v) atomicOr(&g_call_status, v);
}
}  // namespace slra

namespace {

constexpr int64_t kMaxBlocks = 2048;  // selection keeps a row of scores in shared memory
// The branch entry points size their workspace with the parameters the branch does not use set to these.
constexpr int kSparseOnlyRank = 16;
constexpr int kLowrankOnlyBlock = 128;
constexpr float kLowrankOnlyKeep = 1e-4f;  // one kept block per query block (up to 2048 blocks)

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool default_split(int64_t D, const int64_t* s, int64_t out[3]) {
    const int64_t c = D / 2;
    if (s[0] == 0 && s[1] == 0 && s[2] == 0) {
        out[1] = c / 3;
        out[2] = c / 3;
        out[0] = c - 2 * (c / 3);
        return true;
    }
    if (s[0] < 0 || s[1] < 0 || s[2] < 0 || s[0] + s[1] + s[2] != c) return false;
    out[0] = s[0]; out[1] = s[1]; out[2] = s[2];
    return true;
}

// Element strides (batch, token, head) of a [B][L][Hh][D] tensor: all zero means contiguous
// (token-major); otherwise positive multiples of `align` elements (16-byte TMA strides), below 2^36.
bool strides_of(const int64_t s[3], int64_t L, int64_t Hh, int64_t D, int64_t align, Strides* out) {
    if (s[0] == 0 && s[1] == 0 && s[2] == 0) {
        out->h = D;
        out->l = Hh * D;
        out->b = L * Hh * D;
        return true;
    }
    for (int i = 0; i < 3; ++i)
        if (s[i] <= 0 || s[i] % align != 0 || s[i] >= (int64_t(1) << 36)) return false;
    out->b = s[0];
    out->l = s[1];
    out->h = s[2];
    return true;
}

// Elements from a tensor's first element to one past its last.
int64_t extent_elems(const Strides& st, int64_t B, int64_t L, int64_t Hh, int64_t D) {
    return (B - 1) * st.b + (L - 1) * st.l + (Hh - 1) * st.h + D;
}

// True when distinct (batch, token, head) rows of D elements never share an element: taking the
// dimensions by increasing stride, each stride clears everything the smaller ones span.
bool rows_disjoint(const Strides& st, int64_t B, int64_t L, int64_t Hh, int64_t D) {
    int64_t s[3] = {st.b, st.l, st.h}, n[3] = {B, L, Hh};
    for (int i = 0; i < 3; ++i)
        for (int j = i + 1; j < 3; ++j)
            if (s[j] < s[i]) { std::swap(s[i], s[j]); std::swap(n[i], n[j]); }
    int64_t span = D;
    for (int i = 0; i < 3; ++i) {
        if (n[i] == 1) continue;
        if (s[i] < span) return false;
        span += s[i] * (n[i] - 1);
    }
    return true;
}

struct Derived {
    Geom g;
    RopeMeta meta;
    int table_entries;
    int nsplit;
    slra_ws_layout lay;
    size_t at_img, sb_img;  // operand images of the tensor-core readout (offsets; head_dim 128 only)
    size_t a_elems;         // bf16 elements of the projection argument
    size_t ak_off;          // elements from its start to the key projection(s)
    bool gated;             // gated fusion of the branches
};

slra_status derive(const slra_problem* p, Derived* d) {
    if (!p) return SLRA_ERR_INVALID_ARG;
    if (p->batch < 1 || p->heads < 1 || p->T < 1 || p->H < 1 || p->W < 1) return SLRA_ERR_INVALID_ARG;
    if (!(p->keep_frac > 0.0 && p->keep_frac <= 1.0)) return SLRA_ERR_INVALID_ARG;
    if (p->theta < 0.0 || std::isnan(p->theta)) return SLRA_ERR_INVALID_ARG;
    if (p->out_dtype != SLRA_OUT_F32 && p->out_dtype != SLRA_OUT_BF16) return SLRA_ERR_INVALID_ARG;
    if (p->branches < 0 || p->branches > 3) return SLRA_ERR_INVALID_ARG;
    if (p->activation < SLRA_ACT_RELU || p->activation > SLRA_ACT_TANH) return SLRA_ERR_INVALID_ARG;
    if (p->lowrank_norope != 0 && p->lowrank_norope != 1) return SLRA_ERR_INVALID_ARG;
    if (p->lowrank_rope_inside != 0 && p->lowrank_rope_inside != 1) return SLRA_ERR_INVALID_ARG;
    if (p->lowrank_rope_inside && p->lowrank_norope) return SLRA_ERR_INVALID_ARG;
    if (p->proj_separate != 0 && p->proj_separate != 1) return SLRA_ERR_INVALID_ARG;
    if (p->proj_per_head != 0 && p->proj_per_head != 1) return SLRA_ERR_INVALID_ARG;
    if (p->fusion != SLRA_FUSION_SUM && p->fusion != SLRA_FUSION_GATED) return SLRA_ERR_INVALID_ARG;
    if (p->fusion == SLRA_FUSION_GATED) {  // gate parameters given, both branches on
        if (!p->gate_w || !std::isfinite(p->gate_bias)) return SLRA_ERR_INVALID_ARG;
        if (p->branches != 0 && p->branches != SLRA_BRANCH_BOTH) return SLRA_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(p->gate_w) & 15u) != 0) return SLRA_ERR_ALIGNMENT;
    }
    if (p->head_dim != 64 && p->head_dim != 128) return SLRA_ERR_UNSUPPORTED;
    if (p->block != 64 && p->block != 128) return SLRA_ERR_UNSUPPORTED;
    if (p->rank < 16 || p->rank > p->head_dim || p->rank % 16 != 0) return SLRA_ERR_UNSUPPORTED;
    const int64_t L = p->T * p->H * p->W;
    if (p->T > (1 << 20) || p->H > (1 << 20) || p->W > (1 << 20) || L > (int64_t(1) << 28))
        return SLRA_ERR_INVALID_ARG;
    const int64_t nb = (L + p->block - 1) / p->block;
    if (nb > kMaxBlocks) return SLRA_ERR_UNSUPPORTED;
    const int64_t BH = p->batch * p->heads;
    if (BH > 65535) return SLRA_ERR_UNSUPPORTED;  // a launch grid dimension
    if (BH * nb * p->block >= (int64_t(1) << 31)) return SLRA_ERR_UNSUPPORTED;  // TMA row coordinate
    int64_t split[3];
    if (!default_split(p->head_dim, p->rope_split, split)) return SLRA_ERR_INVALID_ARG;
    int64_t keep = static_cast<int64_t>(std::floor(p->keep_frac * static_cast<double>(nb) + 0.5));
    keep = keep < 1 ? 1 : (keep > nb ? nb : keep);

    Geom& g = d->g;
    g.B = static_cast<int>(p->batch);
    g.Hh = static_cast<int>(p->heads);
    g.D = static_cast<int>(p->head_dim);
    g.T = static_cast<int>(p->T);
    g.H = static_cast<int>(p->H);
    g.W = static_cast<int>(p->W);
    g.L = static_cast<int>(L);
    g.block = static_cast<int>(p->block);
    g.nb = static_cast<int>(nb);
    g.keep = static_cast<int>(keep);
    g.R = static_cast<int>(p->rank);
    g.Lp = static_cast<int>(nb * p->block);
    g.act = static_cast<int>(p->activation);
    g.norope = static_cast<int>(p->lowrank_norope);
    g.a_stride = p->proj_per_head ? g.D * g.R : 0;
    g.inside = static_cast<int>(p->lowrank_rope_inside);
    // element strides: inputs in 16-byte units of bf16; out in 16-byte units of its type, rows disjoint
    const int64_t out_align = p->out_dtype == SLRA_OUT_F32 ? 4 : 8;
    if (!strides_of(p->q_strides, L, p->heads, p->head_dim, 8, &g.sq) ||
        !strides_of(p->k_strides, L, p->heads, p->head_dim, 8, &g.sk) ||
        !strides_of(p->v_strides, L, p->heads, p->head_dim, 8, &g.sv) ||
        !strides_of(p->out_strides, L, p->heads, p->head_dim, out_align, &g.so) ||
        !rows_disjoint(g.so, p->batch, L, p->heads, p->head_dim))
        return SLRA_ERR_INVALID_ARG;
    // projection argument: [1 + separate][per_head ? Hh : 1][D][R], query projection(s) first
    const size_t one_side = static_cast<size_t>(p->proj_per_head ? p->heads : 1) * p->head_dim * p->rank;
    d->a_elems = one_side * (p->proj_separate ? 2 : 1);
    d->ak_off = p->proj_separate ? one_side : 0;
    d->gated = p->fusion == SLRA_FUSION_GATED;

    RopeMeta& m = d->meta;
    std::memset(&m, 0, sizeof m);
    m.npairs = g.D / 2;
    m.theta = p->theta > 0.0 ? p->theta : 10000.0;
    const int lens[3] = {g.T, g.H, g.W};
    int j = 0, off = 0;
    for (int a = 0; a < 3; ++a) {
        m.apairs[a] = static_cast<int>(split[a]);
        m.axis_len[a] = lens[a];
        m.off[a] = p->pos_offset[a];
        for (int mm = 0; mm < split[a]; ++mm, ++j) {
            m.axis[j] = a;
            m.mloc[j] = mm;
            m.tab_off[j] = off;
            off += lens[a];
        }
    }
    d->table_entries = off;
    const int64_t ns = lowrank_nsplit(g);
    d->nsplit = static_cast<int>(ns);

    slra_ws_layout& w = d->lay;
    std::memset(&w, 0, sizeof w);
    w.L = L;
    w.nb = nb;
    w.keep = keep;
    w.nsplit = ns;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t at = o;
        o = align_up(o + bytes, 256);
        return at;
    };
    const size_t rows = static_cast<size_t>(BH) * nb * p->block;
    w.status = take(256);
    w.rope_table = take(sizeof(double2) * static_cast<size_t>(off) + sizeof(int2) * kMaxPairs);
    w.qh = take(rows * p->head_dim * 2);
    w.kh = take(rows * p->head_dim * 2);
    w.vh = take(rows * p->head_dim * 2);
    w.qbar = take(static_cast<size_t>(BH) * nb * p->head_dim * 8);
    w.kbar = take(static_cast<size_t>(BH) * nb * p->head_dim * 8);
    w.idx = take(static_cast<size_t>(BH) * nb * keep * 4);
    w.tie = take(static_cast<size_t>(BH) * nb);
    w.s_part = take(static_cast<size_t>(BH) * ns * p->rank * p->head_dim * 4);
    w.z_part = take(static_cast<size_t>(BH) * ns * p->rank * 4);
    w.S = take(static_cast<size_t>(BH) * p->rank * p->head_dim * 4);
    w.z = take(static_cast<size_t>(BH) * p->rank * 4);
    if (p->head_dim == 128) {
        d->at_img = take(static_cast<size_t>(p->proj_per_head ? p->heads : 1) * p->rank * 256);
        d->sb_img = take(static_cast<size_t>(BH) * ((p->rank + 63) / 64) * kSbChunkBytes);
    } else {
        d->at_img = d->sb_img = 0;
    }
    w.total_bytes = o;
    return SLRA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

// The current device must be an sm_100 part (the kernels are built for sm_100a only).
slra_status check_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return SLRA_ERR_NO_DEVICE; }
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return SLRA_ERR_NO_DEVICE;
    }
    return (major == 10 && minor == 0) ? SLRA_OK : SLRA_ERR_NO_DEVICE;
}

struct Ptrs {
    uint8_t* base;
    int* status;
    double2* tab;
    int2* pairs;
    __half *qh, *kh, *vh;
    double *qbar, *kbar;
    int32_t* idx;
    uint8_t* tie;
    float *s_part, *z_part, *S, *z;
    uint8_t *at_img, *sb_img;  // nullptr unless head_dim 128
};

Ptrs carve(void* ws, const Derived& d) {
    Ptrs p;
    uint8_t* b = static_cast<uint8_t*>(ws);
    const slra_ws_layout& w = d.lay;
    p.base = b;
    p.status = reinterpret_cast<int*>(b + w.status);
    p.tab = reinterpret_cast<double2*>(b + w.rope_table);
    p.pairs = reinterpret_cast<int2*>(b + w.rope_table + sizeof(double2) * d.table_entries);
    p.qh = reinterpret_cast<__half*>(b + w.qh);
    p.kh = reinterpret_cast<__half*>(b + w.kh);
    p.vh = reinterpret_cast<__half*>(b + w.vh);
    p.qbar = reinterpret_cast<double*>(b + w.qbar);
    p.kbar = reinterpret_cast<double*>(b + w.kbar);
    p.idx = reinterpret_cast<int32_t*>(b + w.idx);
    p.tie = b + w.tie;
    p.s_part = reinterpret_cast<float*>(b + w.s_part);
    p.z_part = reinterpret_cast<float*>(b + w.z_part);
    p.S = reinterpret_cast<float*>(b + w.S);
    p.z = reinterpret_cast<float*>(b + w.z);
    p.at_img = d.at_img ? b + d.at_img : nullptr;
    p.sb_img = d.sb_img ? b + d.sb_img : nullptr;
    return p;
}

slra_status check_ws(const Derived& d, void* ws, size_t bytes) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || bytes < d.lay.total_bytes) return SLRA_ERR_WORKSPACE;
    return SLRA_OK;
}

slra_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SLRA_OK : SLRA_ERR_CUDA; }

// Record the caller's timing event for stage boundary i, if one was given.
slra_status mark(const slra_problem* p, int i, cudaStream_t st) {
    void* e = p->stage_events[i];
    if (e && cudaEventRecord(static_cast<cudaEvent_t>(e), st) != cudaSuccess) return SLRA_ERR_CUDA;
    return SLRA_OK;
}

unsigned long long timeout_of(const slra_problem* p) {
    return p->wait_timeout_ns ? p->wait_timeout_ns : 2000000000ull;
}

int debug_wait_of(const slra_problem* p) { return (p->debug_flags & SLRA_DEBUG_UNSATISFIED_WAIT) ? 1 : 0; }


// Tables + RoPE/pooling + selection; write_v: also the fp16 v copy the backward kernels read.
slra_status run_select(const slra_problem* p, const Derived& d, const Ptrs& w, const void* q, const void* k,
                       const void* v, bool write_v, cudaStream_t st) {
    const Geom& g = d.g;
    CUtensorMap mq, mk, mv;  // token-major inputs, boxes of 64 columns x one key block of tokens
    if (!make_map_tokens(&mq, q, g.B, g.L, g.Hh, g.D, g.sq, g.block) ||
        !make_map_tokens(&mk, k, g.B, g.L, g.Hh, g.D, g.sk, g.block) ||
        !make_map_tokens(&mv, v, g.B, g.L, g.Hh, g.D, g.sv, g.block))
        return SLRA_ERR_CUDA;
    cudaError_t e = launch_rope_pool(mq, mk, mv, w.tab, w.pairs, g, write_v, w.qh, w.kh, w.vh, w.qbar, w.kbar,
                                     w.status, timeout_of(p), st);
    if (e != cudaSuccess) return SLRA_ERR_CUDA;
    slra_status s = mark(p, 2, st);
    if (s != SLRA_OK) return s;
    if ((s = cuda_status(launch_select(w.qbar, w.kbar, g, w.idx, w.tie, st))) != SLRA_OK) return s;
    return mark(p, 3, st);
}

// Low-rank partial sums: tensor-core kernel for head_dim 128, CUDA-core kernel otherwise.  A is the
// whole projection argument; the kernels get the key projection(s).
cudaError_t lowrank_partial(const Derived& d, const void* k, const void* v, const void* A, const double2* tab,
                            const int2* pairs, int nsplit, float* s_part, float* z_part, int* status,
                            unsigned long long timeout_ns, int debug_wait, cudaStream_t st) {
    const auto* kb = static_cast<const __nv_bfloat16*>(k);
    const auto* vb = static_cast<const __nv_bfloat16*>(v);
    const auto* Ab = static_cast<const __nv_bfloat16*>(A) + d.ak_off;  // the key projection(s)
    if (d.g.D == 128)
        return launch_lowrank_tc(kb, vb, Ab, tab, d.meta, d.g, nsplit, s_part, z_part, status, timeout_ns, debug_wait,
                                 st);
    return launch_lowrank_partial(kb, vb, Ab, tab, pairs, d.g, nsplit, s_part, z_part, st);
}

slra_status run_lowrank(const slra_problem* p, const Derived& d, const Ptrs& w, const void* k, const void* v,
                        const void* A, cudaStream_t st) {
    const Geom& g = d.g;
    cudaError_t e = lowrank_partial(d, k, v, A, w.tab, w.pairs, d.nsplit, w.s_part, w.z_part, w.status,
                                    timeout_of(p), debug_wait_of(p), st);
    if (e != cudaSuccess) return SLRA_ERR_CUDA;
    slra_status s = mark(p, 4, st);
    if (s != SLRA_OK) return s;
    // the readout's A^T image comes from the query projection(s), at the start of A
    if ((s = cuda_status(launch_lowrank_reduce(w.s_part, w.z_part, g, d.nsplit, w.S, w.z,
                                               static_cast<const __nv_bfloat16*>(A), w.at_img, w.sb_img, st))) !=
        SLRA_OK)
        return s;
    return mark(p, 5, st);
}

slra_status begin(const slra_problem* p, const Derived& d, const Ptrs& w, cudaStream_t st) {
    slra_status s = mark(p, 0, st);
    if (s != SLRA_OK) return s;
    if (cudaMemsetAsync(w.status, 0, sizeof(int), st) != cudaSuccess) return SLRA_ERR_CUDA;
    if ((s = cuda_status(launch_rope_table(w.tab, w.pairs, d.meta, d.table_entries, st))) != SLRA_OK) return s;
    return mark(p, 1, st);
}

size_t qkv_bytes(const Derived& d) {
    return static_cast<size_t>(d.g.B) * d.g.L * d.g.Hh * d.g.D * 2;
}

// Bytes a [B][L][Hh][D] tensor with strides st spans (es bytes per element).
size_t span_bytes(const Geom& g, const Strides& st, size_t es) {
    return static_cast<size_t>(extent_elems(st, g.B, g.L, g.Hh, g.D)) * es;
}

bool contiguous_io(const slra_problem* p) {
    for (int i = 0; i < 3; ++i)
        if (p->q_strides[i] || p->k_strides[i] || p->v_strides[i] || p->out_strides[i]) return false;
    return true;
}

// The forward pass on a caller's (or the library's) workspace; arguments already validated by derive.
// `lse` and `os` (both NULL, or both set): also keep each row's lse and the sparse branch's own output
// for a backward pass (head-major fp32, the backward workspace's sections).
slra_status fwd_impl(const slra_problem* p, const Derived& d, const void* q, const void* k, const void* v,
                     const void* A, void* out, void* workspace, cudaStream_t st, float* lse = nullptr,
                     float* os = nullptr);

// Runs body(workspace) on the caller's workspace, or, when that is NULL, on one the library allocates
// with cudaMallocAsync on `st` (the device's current memory pool) and frees with cudaFreeAsync after the
// launches, both stream-ordered; that call's device status word is ORed into g_call_status first.
template <class Body>
slra_status with_workspace(const Derived& d, void* workspace, size_t workspace_bytes, cudaStream_t st, Body&& body) {
    if (workspace) {
        slra_status s = check_ws(d, workspace, workspace_bytes);
        return s != SLRA_OK ? s : body(workspace);
    }
    void* raw = nullptr;
    if (cudaMallocAsync(&raw, d.lay.total_bytes + 256, st) != cudaSuccess) {
        cudaGetLastError();
        return SLRA_ERR_CUDA;
    }
    void* ws = reinterpret_cast<void*>(align_up(reinterpret_cast<uintptr_t>(raw), 256));
    slra_status s = body(ws);
    if (s == SLRA_OK) {
        slra::status_or_global_kernel<<<1, 1, 0, st>>>(reinterpret_cast<const int*>(static_cast<uint8_t*>(ws) +
                                                                                    d.lay.status));
        if (cudaGetLastError() != cudaSuccess) s = SLRA_ERR_CUDA;
    }
    if (cudaFreeAsync(raw, st) != cudaSuccess) {
        cudaGetLastError();
        if (s == SLRA_OK) s = SLRA_ERR_CUDA;
    }
    return s;
}

// Shared validation of the device entry points' tensor arguments.  A may be NULL when the low-rank
// branch is off.
slra_status check_fwd_args(const slra_problem* p, const Derived& d, const void* q, const void* k, const void* v,
                           const void* A, const void* out, const void* workspace, size_t workspace_bytes) {
    const int branches = p->branches == 0 ? SLRA_BRANCH_BOTH : p->branches;
    if (!q || !k || !v || !out || ((branches & SLRA_BRANCH_LOWRANK) && !A)) return SLRA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || (A && !aligned16(A)) || !aligned16(out))
        return SLRA_ERR_ALIGNMENT;
    const Geom& g = d.g;
    const size_t out_b = span_bytes(g, g.so, p->out_dtype == SLRA_OUT_F32 ? 4 : 2);
    if (overlaps(out, out_b, q, span_bytes(g, g.sq, 2)) || overlaps(out, out_b, k, span_bytes(g, g.sk, 2)) ||
        overlaps(out, out_b, v, span_bytes(g, g.sv, 2)) || (A && overlaps(out, out_b, A, d.a_elems * 2)) ||
        (workspace && overlaps(out, out_b, workspace, workspace_bytes)))
        return SLRA_ERR_INVALID_ARG;
    return SLRA_OK;
}

// ------------------------------------------------------------------ host entry point, pipelined
// Over PCIe the host entry point's copies (q, k, v in, out back) take several times the compute.
// Heads are independent, so the call runs groups of heads as independent sub-problems, with the
// upload of one group, the compute of the previous one and the download of the one before that in
// flight together: two device slots used in turn, copies on two streams of their own (one per
// direction), compute on the caller's stream, ordered by events.
constexpr int kMaxPipeDevices = 64;
struct HostPipe {
    std::mutex mu;  // one pipelined call per device at a time: the streams and events are shared
    bool ready = false;
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr, in[2] = {}, done[2] = {}, out[2] = {};
};
HostPipe g_pipes[kMaxPipeDevices];

// The low-rank branch's preparation (partial sums and their reduction, on raw k and v) does not depend
// on the sparse branch's (RoPE + pooling, selection), so it runs on a side stream of the library's own
// (one per device, with a fork and a join event, created on first use) while the calling stream runs
// the other; the calling stream waits for it before the attention kernel.
struct SideStream {
    std::mutex mu;  // the fork/join events are shared by the calls on this device
    bool ready = false;
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
SideStream g_side[kMaxPipeDevices];

slra_status side_init(SideStream& ss) {
    if (ss.ready) return SLRA_OK;
    const unsigned ef = cudaEventDisableTiming;
    if (cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.fork, ef) != cudaSuccess || cudaEventCreateWithFlags(&ss.join, ef) != cudaSuccess) {
        cudaGetLastError();
        return SLRA_ERR_CUDA;
    }
    ss.ready = true;
    return SLRA_OK;
}

slra_status pipe_init(HostPipe& hp) {
    if (hp.ready) return SLRA_OK;
    const unsigned ef = cudaEventDisableTiming;
    if (cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&hp.start, ef) != cudaSuccess)
        return SLRA_ERR_CUDA;
    for (int i = 0; i < 2; ++i)
        if (cudaEventCreateWithFlags(&hp.in[i], ef) != cudaSuccess ||
            cudaEventCreateWithFlags(&hp.done[i], ef) != cudaSuccess ||
            cudaEventCreateWithFlags(&hp.out[i], ef) != cudaSuccess)
            return SLRA_ERR_CUDA;
    hp.ready = true;
    return SLRA_OK;
}

// Heads per group: about sixteen groups per batch element (at Wan2.1-14B, 14 groups of 3 heads: 47.6 ms
// per call, against 49.8 with 8 groups and 58.3 with 4; the first upload and the last download are
// what smaller groups shorten).
int pipe_group_heads(int Hh) { return (Hh + 15) / 16; }

// How the host entry point splits a problem: groups of hg heads (the last of a batch element may be
// smaller), each a sub-problem with batch 1, run through two device slots.
struct PipePlan {
    int hg, per_b, G;      // heads per group, groups per batch element, groups
    slra_problem sub;      // a full group's sub-problem (stage events cleared)
    size_t row_in, row_out;  // bytes of one head row of the inputs / of the output
    size_t in_g, out_g;    // bytes of one input tensor / of the output of a group in a slot
    size_t a_full, a_g;    // the whole projection argument; a group's per-head projections (or 0)
    size_t side;           // elements of one head's projection
    size_t slot_io, slot_ws;  // one slot in the io buffer and in the workspace
};

// Fills *pl; returns the number of groups (1: no pipelining, because there is a single group or two
// slots do not fit the buffers).
int plan_pipeline(const slra_problem* p, const Derived& d, size_t io_bytes, size_t ws_bytes, PipePlan* pl) {
    const Geom& g = d.g;
    pl->hg = pipe_group_heads(g.Hh);
    pl->per_b = (g.Hh + pl->hg - 1) / pl->hg;
    pl->G = g.B * pl->per_b;
    if (pl->G < 2) return 1;
    pl->sub = *p;
    pl->sub.batch = 1;
    pl->sub.heads = pl->hg;
    for (auto& e : pl->sub.stage_events) e = nullptr;  // the sub-calls time nothing
    Derived dg;
    if (derive(&pl->sub, &dg) != SLRA_OK) return 1;
    const size_t osz = p->out_dtype == SLRA_OUT_F32 ? 4 : 2;
    pl->row_in = static_cast<size_t>(g.D) * 2;
    pl->row_out = static_cast<size_t>(g.D) * osz;
    pl->in_g = align_up(static_cast<size_t>(g.L) * pl->hg * pl->row_in, 256);
    pl->out_g = align_up(static_cast<size_t>(g.L) * pl->hg * pl->row_out, 256);
    pl->a_full = align_up(d.a_elems * 2, 256);
    pl->side = static_cast<size_t>(g.D) * g.R;
    pl->a_g = p->proj_per_head ? align_up((p->proj_separate ? 2 : 1) * pl->hg * pl->side * 2, 256) : 0;
    pl->slot_io = 3 * pl->in_g + pl->out_g + pl->a_g;
    pl->slot_ws = align_up(dg.lay.total_bytes, 256);
    if (pl->a_full + 2 * pl->slot_io > io_bytes || 256 + 2 * pl->slot_ws > ws_bytes) return 1;
    return pl->G;
}

// Runs the host entry point as pipelined head groups.  *used = false (nothing launched) when the plan
// has a single group.
slra_status host_fwd_pipelined(const slra_problem* p, const Derived& d, const void* q_host, const void* k_host,
                               const void* v_host, const void* A_host, void* out_host, uint8_t* io, size_t io_bytes,
                               uint8_t* ws, size_t ws_bytes, cudaStream_t st, bool* used) {
    *used = false;
    const Geom& g = d.g;
    PipePlan pl;
    if (plan_pipeline(p, d, io_bytes, ws_bytes, &pl) < 2) return SLRA_OK;

    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxPipeDevices) return SLRA_ERR_NO_DEVICE;
    HostPipe& hp = g_pipes[dev];
    std::lock_guard<std::mutex> lock(hp.mu);
    slra_status s = pipe_init(hp);
    if (s != SLRA_OK) return s;
    *used = true;
    auto fail = [&](slra_status why) {  // let nothing in flight outlive the call
        cudaStreamSynchronize(hp.h2d);
        cudaStreamSynchronize(hp.d2h);
        cudaStreamSynchronize(st);
        cudaGetLastError();
        return why;
    };
    uint8_t* dA = io;
    const int hg = pl.hg, per_b = pl.per_b, G = pl.G;
    const size_t row_in = pl.row_in, row_out = pl.row_out, in_g = pl.in_g, out_g = pl.out_g, side = pl.side;
    const size_t slot_io = pl.slot_io, slot_ws = pl.slot_ws;
    int* acc = reinterpret_cast<int*>(ws);  // the caller's status word (offset 0, as for slra_attn_fwd)
    if (cudaEventRecord(hp.start, st) != cudaSuccess || cudaStreamWaitEvent(hp.h2d, hp.start, 0) != cudaSuccess ||
        cudaMemsetAsync(acc, 0, sizeof(int), st) != cudaSuccess ||
        cudaMemcpyAsync(dA, A_host, d.a_elems * 2, cudaMemcpyHostToDevice, hp.h2d) != cudaSuccess)
        return fail(SLRA_ERR_CUDA);
    for (int gi = 0; gi < G; ++gi) {
        const int sl = gi & 1;
        const int b = gi / per_b, h0 = (gi % per_b) * hg, hn = std::min(hg, g.Hh - h0);
        uint8_t* base = io + pl.a_full + sl * slot_io;
        uint8_t *sq = base, *sk = base + in_g, *sv = base + 2 * in_g, *so = base + 3 * in_g, *sa = so + out_g;
        uint8_t* sws = ws + 256 + sl * slot_ws;
        const size_t off = (static_cast<size_t>(b) * g.L * g.Hh + h0);  // first row element offset / D
        // upload, once the slot's previous group has finished reading its inputs
        if (gi >= 2 && cudaStreamWaitEvent(hp.h2d, hp.done[sl], 0) != cudaSuccess) return fail(SLRA_ERR_CUDA);
        const void* srcs[3] = {q_host, k_host, v_host};
        uint8_t* dsts[3] = {sq, sk, sv};
        for (int t = 0; t < 3; ++t)
            if (cudaMemcpy2DAsync(dsts[t], hn * row_in, static_cast<const uint8_t*>(srcs[t]) + off * row_in,
                                  g.Hh * row_in, hn * row_in, g.L, cudaMemcpyHostToDevice, hp.h2d) != cudaSuccess)
                return fail(SLRA_ERR_CUDA);
        if (cudaEventRecord(hp.in[sl], hp.h2d) != cudaSuccess) return fail(SLRA_ERR_CUDA);
        // compute, once the inputs are in and the slot's previous output has been downloaded
        if (cudaStreamWaitEvent(st, hp.in[sl], 0) != cudaSuccess ||
            (gi >= 2 && cudaStreamWaitEvent(st, hp.out[sl], 0) != cudaSuccess))
            return fail(SLRA_ERR_CUDA);
        const void* Ag = dA;
        if (p->proj_per_head) {  // this group's heads of each side, contiguous
            for (int sd = 0; sd < (p->proj_separate ? 2 : 1); ++sd)
                if (cudaMemcpyAsync(sa + sd * hn * side * 2, dA + (sd * g.Hh + h0) * side * 2, hn * side * 2,
                                    cudaMemcpyDeviceToDevice, st) != cudaSuccess)
                    return fail(SLRA_ERR_CUDA);
            Ag = sa;
        }
        slra_problem pgi = pl.sub;
        pgi.heads = hn;
        s = slra_attn_fwd_ex(&pgi, sq, sk, sv, Ag, so, sws, slot_ws, reinterpret_cast<slra_stream_t>(st));
        if (s != SLRA_OK) return fail(s);
        slra::status_or_kernel<<<1, 1, 0, st>>>(acc, reinterpret_cast<const int*>(sws));
        if (cudaGetLastError() != cudaSuccess || cudaEventRecord(hp.done[sl], st) != cudaSuccess)
            return fail(SLRA_ERR_CUDA);
        // download into the group's strided place in the host output
        if (cudaStreamWaitEvent(hp.d2h, hp.done[sl], 0) != cudaSuccess ||
            cudaMemcpy2DAsync(static_cast<uint8_t*>(out_host) + off * row_out, g.Hh * row_out, so, hn * row_out,
                              hn * row_out, g.L, cudaMemcpyDeviceToHost, hp.d2h) != cudaSuccess ||
            cudaEventRecord(hp.out[sl], hp.d2h) != cudaSuccess)
            return fail(SLRA_ERR_CUDA);
    }
    if (cudaStreamWaitEvent(st, hp.out[(G - 1) & 1], 0) != cudaSuccess) return fail(SLRA_ERR_CUDA);
    return cuda_status(cudaStreamSynchronize(st));
}

slra_status fwd_impl(const slra_problem* p, const Derived& d, const void* q, const void* k, const void* v,
                     const void* A, void* out, void* workspace, cudaStream_t st, float* lse, float* os) {
    slra_status s;
    const Ptrs w = carve(workspace, d);
    const int branches = p->branches == 0 ? SLRA_BRANCH_BOTH : p->branches;
    const Geom& g = d.g;

    AttnMaps maps;
    const uint64_t rows = static_cast<uint64_t>(g.BH()) * g.Lp;
    if (!make_map_headmajor(&maps.q, w.qh, rows, g.D, 128) || !make_map_headmajor(&maps.k, w.kh, rows, g.D, g.block) ||
        !make_map_tokens(&maps.v, v, g.B, g.L, g.Hh, g.D, g.sv, g.block) ||
        !make_map_tokens(&maps.q_raw, q, g.B, g.L, g.Hh, g.D, g.sq, 128) ||
        !make_map_out(&maps.out, out, g.B, g.L, g.Hh, g.D, g.so, p->out_dtype == SLRA_OUT_F32))
        return SLRA_ERR_CUDA;
    std::memset(&maps.os, 0, sizeof maps.os);
    if (os && !make_map_out(&maps.os, os, g.B, g.L, g.Hh, g.D, headmajor_strides(g), true)) return SLRA_ERR_CUDA;

    if ((s = begin(p, d, w, st)) != SLRA_OK) return s;
    const bool overlap = branches == SLRA_BRANCH_BOTH && !(p->debug_flags & SLRA_DEBUG_SERIAL_BRANCHES);
    if (overlap) {
        int dev = -1;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxPipeDevices) {
            cudaGetLastError();
            return SLRA_ERR_NO_DEVICE;
        }
        SideStream& ss = g_side[dev];
        std::lock_guard<std::mutex> lock(ss.mu);
        if ((s = side_init(ss)) != SLRA_OK) return s;
        if (cudaEventRecord(ss.fork, st) != cudaSuccess || cudaStreamWaitEvent(ss.s, ss.fork, 0) != cudaSuccess)
            return SLRA_ERR_CUDA;
        // the low-rank preparation on the side stream (stage events [4], [5] recorded there), the
        // sparse one on the calling stream; the join is enqueued whatever happened, so nothing of this
        // call is left running unordered
        const slra_status s_lr = run_lowrank(p, d, w, k, v, A, ss.s);
        const bool rec = cudaEventRecord(ss.join, ss.s) == cudaSuccess;
        const slra_status s_sel = run_select(p, d, w, q, k, v, lse != nullptr, st);
        const bool joined = rec && cudaStreamWaitEvent(st, ss.join, 0) == cudaSuccess;
        if (!joined) {
            cudaGetLastError();
            cudaStreamSynchronize(ss.s);
            return SLRA_ERR_CUDA;
        }
        if (s_lr != SLRA_OK) return s_lr;
        if (s_sel != SLRA_OK) return s_sel;
        // [5] again, on the calling stream: both preparations are done and the attention kernel starts
        if ((s = mark(p, 5, st)) != SLRA_OK) return s;
    } else {
        // a branch that is off still records its stage boundaries, so its stages time as zero
        if (branches & SLRA_BRANCH_SPARSE) {
            if ((s = run_select(p, d, w, q, k, v, lse != nullptr, st)) != SLRA_OK) return s;
        } else if ((s = mark(p, 2, st)) != SLRA_OK || (s = mark(p, 3, st)) != SLRA_OK) {
            return s;
        }
        if (branches & SLRA_BRANCH_LOWRANK) {
            if ((s = run_lowrank(p, d, w, k, v, A, st)) != SLRA_OK) return s;
        } else if ((s = mark(p, 4, st)) != SLRA_OK || (s = mark(p, 5, st)) != SLRA_OK) {
            return s;
        }
    }

    AttnArgs a;
    a.qh = w.qh;
    a.kh = w.kh;
    a.idx = w.idx;
    a.keep = (branches & SLRA_BRANCH_SPARSE) ? g.keep : 0;
    a.q_raw = static_cast<const __nv_bfloat16*>(q);
    a.A = static_cast<const __nv_bfloat16*>(A);  // query projection(s); NULL when the low-rank branch is off
    a.S = w.S;
    a.z = w.z;
    a.tab = w.tab;
    a.pairs = w.pairs;
    for (int e = 0; e < kMaxPairs; ++e)
        a.pair_info[e] = e < d.meta.npairs ? make_int2(d.meta.axis[e], d.meta.tab_off[e]) : make_int2(0, 0);
    a.at_img = w.at_img;
    a.sb_img = w.sb_img;
    a.lowrank = (branches & SLRA_BRANCH_LOWRANK) ? 1 : 0;
    a.gated = p->fusion == SLRA_FUSION_GATED ? 1 : 0;
    a.gate_b = p->gate_bias;
    a.gate_w = static_cast<const float*>(p->gate_w);
    a.out = out;
    a.out_bf16 = p->out_dtype == SLRA_OUT_BF16 ? 1 : 0;
    a.status = w.status;
    a.timeout_ns = timeout_of(p);
    a.debug_unsatisfied_wait = debug_wait_of(p);
    a.lse = lse;
    a.os_save = os;
    if ((s = cuda_status(launch_attn(maps, a, g, st))) != SLRA_OK) return s;
    return mark(p, 6, st);
}

// ---------------------------------------------------------------- backward pass
// Sections the backward adds after the forward's workspace layout (256-B aligned byte offsets).
struct BwdLayout {
    size_t lse, delta, os, doh, inv_cnt, inv, ds_part, dz_part, dS, dz, da_part;
    size_t olr, dolr, dlogit, gpart;  // gated fusion only (empty otherwise)
    size_t total;
    int ns;  // splits of the low-rank gradient passes
};

BwdLayout bwd_layout(const Derived& d) {
    const Geom& g = d.g;
    BwdLayout b;
    size_t o = d.lay.total_bytes;
    auto take = [&](size_t bytes) {
        size_t at = o;
        o = align_up(o + bytes, 256);
        return at;
    };
    const size_t rows = static_cast<size_t>(g.BH()) * g.Lp;
    b.ns = lr_bwd_nsplit(g);
    b.lse = take(rows * 4);
    b.delta = take(rows * 4);
    b.os = take(rows * g.D * 4);
    b.doh = take(rows * g.D * 2);
    b.inv_cnt = take(static_cast<size_t>(g.BH()) * g.nb * 4);
    b.inv = take(static_cast<size_t>(g.BH()) * g.nb * g.nb * 4);
    b.ds_part = take(static_cast<size_t>(g.BH()) * b.ns * g.R * g.D * 4);
    b.dz_part = take(static_cast<size_t>(g.BH()) * b.ns * g.R * 4);
    b.dS = take(static_cast<size_t>(g.BH()) * g.R * g.D * 4);
    b.dz = take(static_cast<size_t>(g.BH()) * g.R * 4);
    b.da_part = take(2 * static_cast<size_t>(g.BH()) * b.ns * g.D * g.R * 4);
    const bool gated = d.gated;
    b.olr = take(gated ? rows * g.D * 4 : 0);
    b.dolr = take(gated ? static_cast<size_t>(g.B) * g.L * g.Hh * g.D * 4 : 0);
    b.dlogit = take(gated ? rows * 4 : 0);
    b.gpart = take(gated ? static_cast<size_t>(kGateParts) * (g.D + 1) * 4 : 0);
    b.total = o;
    return b;
}

// The backward covers every option of the forward; gradients are contiguous fp32 [B][L][Hh][D].
slra_status check_bwd_problem(const slra_problem* p, Derived* d) {
    slra_status s = derive(p, d);
    if (s != SLRA_OK) return s;
    for (int i = 0; i < 3; ++i)
        if (p->out_strides[i]) return SLRA_ERR_INVALID_ARG;
    return SLRA_OK;
}

// A problem description from the tensor descriptors of the descriptor-style entry points.
slra_status problem_from(const slra_tensor* q, const slra_tensor* k, const slra_tensor* v, const slra_tensor* out,
                         int T, int H, int W, int block, float keep_frac, int rank, slra_problem* p) {
    if (!q || !k || !v || !out) return SLRA_ERR_INVALID_ARG;
    for (const slra_tensor* t : {q, k, v})
        if (t->dtype != SLRA_DTYPE_BF16 || t->B != q->B || t->L != q->L || t->Hh != q->Hh || t->D != q->D)
            return SLRA_ERR_INVALID_ARG;
    if (out->dtype != SLRA_DTYPE_F32 && out->dtype != SLRA_DTYPE_BF16) return SLRA_ERR_INVALID_ARG;
    if (out->B != q->B || out->L != q->L || out->Hh != q->Hh || out->D != q->D) return SLRA_ERR_INVALID_ARG;
    if (static_cast<int64_t>(T) * H * W != q->L) return SLRA_ERR_INVALID_ARG;
    slra_status s = slra_problem_init(p, q->B, q->Hh, q->D, T, H, W, block, static_cast<double>(keep_frac), rank);
    if (s != SLRA_OK) return s;
    p->out_dtype = out->dtype == SLRA_DTYPE_F32 ? SLRA_OUT_F32 : SLRA_OUT_BF16;
    const slra_tensor* ts[4] = {q, k, v, out};
    int64_t* dst[4] = {p->q_strides, p->k_strides, p->v_strides, p->out_strides};
    for (int i = 0; i < 4; ++i) {
        dst[i][0] = ts[i]->sB;
        dst[i][1] = ts[i]->sL;
        dst[i][2] = ts[i]->sH;
    }
    return SLRA_OK;
}

}  // namespace

extern "C" {

int slra_abi_version(void) { return SLRA_ABI_VERSION; }

const char* slra_status_string(int s) {
    switch (s) {
        case SLRA_OK: return "ok";
        case SLRA_ERR_INVALID_ARG: return "invalid argument";
        case SLRA_ERR_UNSUPPORTED: return "unsupported size or option";
        case SLRA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case SLRA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case SLRA_ERR_CUDA: return "CUDA call or kernel launch failed";
        case SLRA_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel ran out";
        case SLRA_ERR_RANGE: return "input values outside the fp16 operands' range after RoPE (overflow, or a block below 2^-14)";
        case SLRA_ERR_NO_DEVICE: return "no sm_100 device is current";
        case SLRA_ERR_SCRATCH_LIMIT: return "problem needs more scratch than the fixed no-allocation area holds";
        default: return "unknown status";
    }
}

slra_status slra_problem_init(slra_problem* p, int64_t batch, int64_t heads, int64_t head_dim, int64_t T, int64_t H,
                              int64_t W, int64_t block, double keep_frac, int64_t rank) {
    if (!p) return SLRA_ERR_INVALID_ARG;
    std::memset(p, 0, sizeof *p);
    p->batch = batch;
    p->heads = heads;
    p->head_dim = head_dim;
    p->T = T;
    p->H = H;
    p->W = W;
    p->block = block;
    p->keep_frac = keep_frac;
    p->rank = rank;
    p->theta = 10000.0;
    p->out_dtype = SLRA_OUT_F32;
    p->branches = SLRA_BRANCH_BOTH;
    p->wait_timeout_ns = 2000000000ull;
    p->activation = SLRA_ACT_RELU;
    p->lowrank_norope = 0;
    p->proj_separate = 0;
    p->proj_per_head = 0;
    p->fusion = SLRA_FUSION_SUM;
    p->gate_bias = 0.0f;
    p->gate_w = nullptr;
    p->lowrank_rope_inside = 0;
    p->dgate_w = nullptr;
    p->dgate_b = nullptr;
    return SLRA_OK;
}

slra_status slra_validate(const slra_problem* p) {
    Derived d;
    return derive(p, &d);
}

int64_t slra_keep_count(const slra_problem* p) {
    Derived d;
    return derive(p, &d) == SLRA_OK ? d.g.keep : -1;
}

int64_t slra_projection_elems(const slra_problem* p) {
    Derived d;
    return derive(p, &d) == SLRA_OK ? static_cast<int64_t>(d.a_elems) : -1;
}

slra_status slra_workspace_layout(const slra_problem* p, slra_ws_layout* layout) {
    if (!layout) return SLRA_ERR_INVALID_ARG;
    Derived d;
    slra_status s = derive(p, &d);
    if (s != SLRA_OK) return s;
    *layout = d.lay;
    return SLRA_OK;
}

slra_status slra_attn_fwd_ex(const slra_problem* p, const void* q, const void* k, const void* v, const void* A,
                             void* out, void* workspace, size_t workspace_bytes, slra_stream_t stream) {
    Derived d;
    slra_status s = derive(p, &d);
    if (s != SLRA_OK) return s;
    if ((s = check_fwd_args(p, d, q, k, v, A, out, workspace, workspace_bytes)) != SLRA_OK) return s;
    if (workspace && (s = check_ws(d, workspace, workspace_bytes)) != SLRA_OK) return s;  // before the device
    if ((s = check_device()) != SLRA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    return with_workspace(d, workspace, workspace_bytes, st,
                          [&](void* ws) { return fwd_impl(p, d, q, k, v, A, out, ws, st); });
}

size_t slra_host_io_bytes(const slra_problem* p) {
    Derived d;
    if (derive(p, &d) != SLRA_OK) return 0;
    const size_t in_b = align_up(qkv_bytes(d), 256);
    const size_t a_b = align_up(d.a_elems * 2, 256);
    const size_t out_b = align_up(qkv_bytes(d) / 2 * (p->out_dtype == SLRA_OUT_F32 ? 4 : 2), 256);
    return 3 * in_b + a_b + out_b;
}

int64_t slra_host_pipeline_groups(const slra_problem* p, size_t io_bytes, size_t workspace_bytes) {
    Derived d;
    if (derive(p, &d) != SLRA_OK) return -1;
    PipePlan pl;
    return plan_pipeline(p, d, io_bytes, workspace_bytes, &pl);
}

slra_status slra_attn_fwd_host(const slra_problem* p, const void* q_host, const void* k_host, const void* v_host,
                               const void* A_host, void* out_host, void* io, size_t io_bytes, void* workspace,
                               size_t workspace_bytes, slra_stream_t stream) {
    Derived d;
    slra_status s = derive(p, &d);
    if (s != SLRA_OK) return s;
    if (!q_host || !k_host || !v_host || !A_host || !out_host || !io) return SLRA_ERR_INVALID_ARG;
    if (!contiguous_io(p)) return SLRA_ERR_INVALID_ARG;  // host buffers are contiguous [B][L][Hh][D]
    if ((reinterpret_cast<uintptr_t>(io) & 255u) != 0 || io_bytes < slra_host_io_bytes(p)) return SLRA_ERR_WORKSPACE;
    if ((s = check_ws(d, workspace, workspace_bytes)) != SLRA_OK) return s;
    if ((s = check_device()) != SLRA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    bool used = false;
    s = host_fwd_pipelined(p, d, q_host, k_host, v_host, A_host, out_host, static_cast<uint8_t*>(io), io_bytes,
                           static_cast<uint8_t*>(workspace), workspace_bytes, st, &used);
    if (used || s != SLRA_OK) return s;
    // one group (or too little room for two slots): copy in, compute, copy out
    const size_t raw = qkv_bytes(d);
    const size_t in_b = align_up(raw, 256);
    const size_t a_raw = d.a_elems * 2;
    const size_t out_raw = raw / 2 * (p->out_dtype == SLRA_OUT_F32 ? 4 : 2);
    uint8_t* b = static_cast<uint8_t*>(io);
    void *dq = b, *dk = b + in_b, *dv = b + 2 * in_b, *dA = b + 3 * in_b;
    void* dout = b + 3 * in_b + align_up(a_raw, 256);
    if (cudaMemcpyAsync(dq, q_host, raw, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(dk, k_host, raw, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(dv, v_host, raw, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(dA, A_host, a_raw, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return SLRA_ERR_CUDA;
    s = slra_attn_fwd_ex(p, dq, dk, dv, dA, dout, workspace, workspace_bytes, stream);
    if (s != SLRA_OK) return s;
    if (cudaMemcpyAsync(out_host, dout, out_raw, cudaMemcpyDeviceToHost, st) != cudaSuccess) return SLRA_ERR_CUDA;
    return cuda_status(cudaStreamSynchronize(st));
}

slra_status slra_select_blocks(const slra_problem* p, const void* q, const void* k, const void* v, void* workspace,
                               size_t workspace_bytes, slra_stream_t stream) {
    Derived d;
    slra_status s = derive(p, &d);
    if (s != SLRA_OK) return s;
    if (!q || !k || !v) return SLRA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return SLRA_ERR_ALIGNMENT;
    if ((s = check_ws(d, workspace, workspace_bytes)) != SLRA_OK) return s;
    if ((s = check_device()) != SLRA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const Ptrs w = carve(workspace, d);
    if ((s = begin(p, d, w, st)) != SLRA_OK) return s;
    return run_select(p, d, w, q, k, v, true, st);
}

slra_status slra_lowrank_summary(const slra_problem* p, const void* k, const void* v, const void* A, void* workspace,
                                 size_t workspace_bytes, slra_stream_t stream) {
    Derived d;
    slra_status s = derive(p, &d);
    if (s != SLRA_OK) return s;
    if (!k || !v || !A) return SLRA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(A)) return SLRA_ERR_ALIGNMENT;
    if ((s = check_ws(d, workspace, workspace_bytes)) != SLRA_OK) return s;
    if ((s = check_device()) != SLRA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const Ptrs w = carve(workspace, d);
    if ((s = begin(p, d, w, st)) != SLRA_OK) return s;
    return run_lowrank(p, d, w, k, v, A, st);
}

slra_status slra_device_status(void* workspace, slra_stream_t stream, int32_t* status) {
    if (!workspace || !status) return SLRA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int v = 0;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SLRA_ERR_CUDA;
    if (cudaMemcpy(&v, workspace, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return SLRA_ERR_CUDA;
    if (cudaMemset(workspace, 0, sizeof v) != cudaSuccess) return SLRA_ERR_CUDA;
    *status = (v & kDevTimeout) ? SLRA_ERR_DEVICE_TIMEOUT : ((v & kDevRange) ? SLRA_ERR_RANGE : SLRA_OK);
    return SLRA_OK;
}

size_t slra_workspace_bytes(int64_t batch, int64_t heads, int64_t head_dim, int64_t T, int64_t H, int64_t W,
                            int64_t block, float keep_frac, int64_t rank) {
    slra_problem p;
    if (slra_problem_init(&p, batch, heads, head_dim, T, H, W, block, static_cast<double>(keep_frac), rank) != SLRA_OK)
        return 0;
    Derived d;
    return derive(&p, &d) == SLRA_OK ? d.lay.total_bytes : 0;
}

slra_status slra_attn_fwd(const slra_tensor* q, const slra_tensor* k, const slra_tensor* v, const slra_mat* A,
                          int T, int H, int W, int block, float keep_frac, int rank, slra_tensor* out,
                          slra_stream_t stream) {
    slra_problem p;
    slra_status s = problem_from(q, k, v, out, T, H, W, block, keep_frac, rank, &p);
    if (s != SLRA_OK) return s;
    if (!A || !A->data || A->dtype != SLRA_DTYPE_BF16 || A->D != q->D || A->R != rank) return SLRA_ERR_INVALID_ARG;
    return slra_attn_fwd_ex(&p, q->data, k->data, v->data, A->data, out->data, nullptr, 0, stream);
}

slra_status slra_sparse_fwd(const slra_tensor* q, const slra_tensor* k, const slra_tensor* v, int T, int H, int W,
                            int block, float keep_frac, slra_tensor* out, void* workspace, size_t workspace_bytes,
                            slra_stream_t stream) {
    slra_problem p;
    slra_status s = problem_from(q, k, v, out, T, H, W, block, keep_frac, kSparseOnlyRank, &p);
    if (s != SLRA_OK) return s;
    p.branches = SLRA_BRANCH_SPARSE;
    return slra_attn_fwd_ex(&p, q->data, k->data, v->data, nullptr, out->data, workspace, workspace_bytes, stream);
}

slra_status slra_lowrank_fwd(const slra_tensor* q, const slra_tensor* k, const slra_tensor* v, const slra_mat* A,
                             int T, int H, int W, int rank, slra_tensor* out, float* S, float* z, void* workspace,
                             size_t workspace_bytes, slra_stream_t stream) {
    slra_problem p;
    slra_status s = problem_from(q, k, v, out, T, H, W, kLowrankOnlyBlock, kLowrankOnlyKeep, rank, &p);
    if (s != SLRA_OK) return s;
    if (!A || !A->data || A->dtype != SLRA_DTYPE_BF16 || A->D != q->D || A->R != rank) return SLRA_ERR_INVALID_ARG;
    if ((S && !aligned16(S)) || (z && !aligned16(z))) return SLRA_ERR_ALIGNMENT;
    p.branches = SLRA_BRANCH_LOWRANK;
    Derived d;
    if ((s = derive(&p, &d)) != SLRA_OK) return s;
    if ((s = check_fwd_args(&p, d, q->data, k->data, v->data, A->data, out->data, workspace, workspace_bytes)) !=
        SLRA_OK)
        return s;
    if (workspace && (s = check_ws(d, workspace, workspace_bytes)) != SLRA_OK) return s;
    if ((s = check_device()) != SLRA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t s_bytes = static_cast<size_t>(d.g.BH()) * d.g.R * d.g.D * 4, z_bytes = static_cast<size_t>(d.g.BH()) * d.g.R * 4;
    return with_workspace(d, workspace, workspace_bytes, st, [&](void* ws) {
        slra_status r = fwd_impl(&p, d, q->data, k->data, v->data, A->data, out->data, ws, st);
        if (r != SLRA_OK) return r;
        const uint8_t* b = static_cast<const uint8_t*>(ws);
        if ((S && cudaMemcpyAsync(S, b + d.lay.S, s_bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess) ||
            (z && cudaMemcpyAsync(z, b + d.lay.z, z_bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess))
            return SLRA_ERR_CUDA;
        return SLRA_OK;
    });
}

size_t slra_bwd_workspace_bytes(const slra_problem* p) {
    Derived d;
    return check_bwd_problem(p, &d) == SLRA_OK ? bwd_layout(d).total : 0;
}

namespace {
// The backward pass.  saved: the workspace holds the state slra_attn_fwd_train left for this problem
// and these inputs (tables, selection, summary, fp16 copies, lse, O_s), so nothing is recomputed.
slra_status bwd_impl(const slra_problem* p, const void* q, const void* k, const void* v, const void* A,
                     const float* dout, float* dq, float* dk, float* dv, float* dA, void* workspace,
                     size_t workspace_bytes, slra_stream_t stream, bool saved) {
    Derived d;
    slra_status s = check_bwd_problem(p, &d);
    if (s != SLRA_OK) return s;
    const int branches = p->branches == 0 ? SLRA_BRANCH_BOTH : p->branches;
    const bool lowrank = (branches & SLRA_BRANCH_LOWRANK) != 0, sparse = (branches & SLRA_BRANCH_SPARSE) != 0;
    if (!q || !k || !v || !dout || !dq || !dk || !dv || !dA || (lowrank && !A)) return SLRA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || (A && !aligned16(A)) || !aligned16(dout) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(dA))
        return SLRA_ERR_ALIGNMENT;
    const Geom& g = d.g;
    const BwdLayout bl = bwd_layout(d);
    const size_t gb = qkv_bytes(d) * 2, ab = d.a_elems * 4;  // fp32 gradient bytes
    const void* outs[4] = {dq, dk, dv, dA};
    const size_t out_n[4] = {gb, gb, gb, ab};
    const void* ins[5] = {q, k, v, A, dout};
    const size_t in_n[5] = {span_bytes(g, g.sq, 2), span_bytes(g, g.sk, 2), span_bytes(g, g.sv, 2), d.a_elems * 2, gb};
    for (int i = 0; i < 4; ++i) {
        for (int j = 0; j < 5; ++j)
            if (ins[j] && overlaps(outs[i], out_n[i], ins[j], in_n[j])) return SLRA_ERR_INVALID_ARG;
        for (int j = i + 1; j < 4; ++j)
            if (overlaps(outs[i], out_n[i], outs[j], out_n[j])) return SLRA_ERR_INVALID_ARG;
        if (workspace && overlaps(outs[i], out_n[i], workspace, workspace_bytes)) return SLRA_ERR_INVALID_ARG;
    }
    // the gated fusion's parameter gradients: disjoint from every other argument
    float* dgw = static_cast<float*>(p->dgate_w);
    float* dgb = static_cast<float*>(p->dgate_b);
    if (d.gated) {
        if (!dgw || !dgb) return SLRA_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(dgw) & 15u) != 0 || (reinterpret_cast<uintptr_t>(dgb) & 3u) != 0)
            return SLRA_ERR_ALIGNMENT;
        const size_t gwb = static_cast<size_t>(g.D) * 4;
        if (overlaps(dgw, gwb, dgb, 4)) return SLRA_ERR_INVALID_ARG;
        for (const auto& [ptr, n] : {std::pair<const void*, size_t>{dgw, gwb}, {dgb, 4}}) {
            for (int j = 0; j < 5; ++j)
                if (ins[j] && overlaps(ptr, n, ins[j], in_n[j])) return SLRA_ERR_INVALID_ARG;
            for (int j = 0; j < 4; ++j)
                if (overlaps(ptr, n, outs[j], out_n[j])) return SLRA_ERR_INVALID_ARG;
            if (overlaps(ptr, n, p->gate_w, gwb) || (workspace && overlaps(ptr, n, workspace, workspace_bytes)))
                return SLRA_ERR_INVALID_ARG;
        }
    }
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < bl.total)
        return SLRA_ERR_WORKSPACE;
    if ((s = check_device()) != SLRA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const Ptrs w = carve(workspace, d);
    uint8_t* base = static_cast<uint8_t*>(workspace);
    float* lse = reinterpret_cast<float*>(base + bl.lse);
    float* delta = reinterpret_cast<float*>(base + bl.delta);
    float* os = reinterpret_cast<float*>(base + bl.os);
    __half* doh = reinterpret_cast<__half*>(base + bl.doh);
    int32_t* inv_cnt = reinterpret_cast<int32_t*>(base + bl.inv_cnt);
    int32_t* inv = reinterpret_cast<int32_t*>(base + bl.inv);
    // the recompute runs the forward's stages without recording the caller's events
    slra_problem pr = *p;
    for (auto& e : pr.stage_events) e = nullptr;

    if ((s = mark(p, 0, st)) != SLRA_OK) return s;
    // the saved forward's status word keeps whatever it recorded; a recompute starts a fresh one
    if (!saved && cudaMemsetAsync(w.status, 0, sizeof(int), st) != cudaSuccess) return SLRA_ERR_CUDA;
    if (!saved && (s = cuda_status(launch_rope_table(w.tab, w.pairs, d.meta, d.table_entries, st))) != SLRA_OK)
        return s;
    if (!saved && sparse && (s = run_select(&pr, d, w, q, k, v, true, st)) != SLRA_OK) return s;
    if (!saved && lowrank && (s = run_lowrank(&pr, d, w, k, v, A, st)) != SLRA_OK) return s;
    if (!saved && sparse) {
        // the sparse forward again, writing its output O_s (head-major fp32) and each row's lse
        AttnMaps maps;
        const uint64_t rows = static_cast<uint64_t>(g.BH()) * g.Lp;
        if (!make_map_headmajor(&maps.q, w.qh, rows, g.D, 128) ||
            !make_map_headmajor(&maps.k, w.kh, rows, g.D, g.block) ||
            !make_map_tokens(&maps.v, v, g.B, g.L, g.Hh, g.D, g.sv, g.block) ||
            !make_map_tokens(&maps.q_raw, q, g.B, g.L, g.Hh, g.D, g.sq, 128) ||
            !make_map_out(&maps.out, os, g.B, g.L, g.Hh, g.D, headmajor_strides(g), true))
            return SLRA_ERR_CUDA;
        std::memset(&maps.os, 0, sizeof maps.os);
        AttnArgs a;
        std::memset(&a, 0, sizeof a);
        a.qh = w.qh;
        a.kh = w.kh;
        a.idx = w.idx;
        a.keep = g.keep;
        a.q_raw = static_cast<const __nv_bfloat16*>(q);
        a.tab = w.tab;
        a.pairs = w.pairs;
        a.lowrank = 0;
        a.out = os;
        a.status = w.status;
        a.timeout_ns = timeout_of(p);
        a.lse = lse;
        a.os_save = nullptr;
        if ((s = cuda_status(launch_attn(maps, a, g, st))) != SLRA_OK) return s;
    }
    float* olr = reinterpret_cast<float*>(base + bl.olr);
    float* dolr = reinterpret_cast<float*>(base + bl.dolr);
    float* dlogit = reinterpret_cast<float*>(base + bl.dlogit);
    if (d.gated) {
        // the low-rank branch's own output O_lr (head-major fp32): the attention kernel with the sparse
        // branch off, the readout alone (both in the recompute and after a training forward)
        AttnMaps maps;
        const uint64_t rows = static_cast<uint64_t>(g.BH()) * g.Lp;
        if (!make_map_headmajor(&maps.q, w.qh, rows, g.D, 128) ||
            !make_map_headmajor(&maps.k, w.kh, rows, g.D, g.block) ||
            !make_map_tokens(&maps.v, v, g.B, g.L, g.Hh, g.D, g.sv, g.block) ||
            !make_map_tokens(&maps.q_raw, q, g.B, g.L, g.Hh, g.D, g.sq, 128) ||
            !make_map_out(&maps.out, olr, g.B, g.L, g.Hh, g.D, headmajor_strides(g), true))
            return SLRA_ERR_CUDA;
        std::memset(&maps.os, 0, sizeof maps.os);
        AttnArgs a;
        std::memset(&a, 0, sizeof a);
        a.qh = w.qh;
        a.kh = w.kh;
        a.idx = w.idx;
        a.keep = 0;
        a.q_raw = static_cast<const __nv_bfloat16*>(q);
        a.A = static_cast<const __nv_bfloat16*>(A);
        a.S = w.S;
        a.z = w.z;
        a.tab = w.tab;
        a.pairs = w.pairs;
        for (int e = 0; e < kMaxPairs; ++e)
            a.pair_info[e] = e < d.meta.npairs ? make_int2(d.meta.axis[e], d.meta.tab_off[e]) : make_int2(0, 0);
        a.at_img = w.at_img;
        a.sb_img = w.sb_img;
        a.lowrank = 1;
        a.out = olr;
        a.status = w.status;
        a.timeout_ns = timeout_of(p);
        if ((s = cuda_status(launch_attn(maps, a, g, st))) != SLRA_OK) return s;
    }
    if ((s = mark(p, 1, st)) != SLRA_OK) return s;
    // The sparse kernels store dq, dk, dv; the low-rank gradients then add their parts (or store them
    // when the sparse branch is off).
    if (sparse) {
        // dO_s as the sparse branch sees it: dout itself, or through the gate (with dO_lr and dlogit)
        if (d.gated)
            s = cuda_status(launch_gate_prep(dout, os, olr, static_cast<const __nv_bfloat16*>(q),
                                             static_cast<const float*>(p->gate_w), p->gate_bias, g, doh, delta, dolr,
                                             dlogit, w.status, st));
        else
            s = cuda_status(launch_bwd_prep(dout, os, g, doh, delta, w.status, st));
        if (s != SLRA_OK) return s;
        if ((s = cuda_status(launch_bwd_invert(w.idx, g, inv, inv_cnt, st))) != SLRA_OK) return s;
        if ((s = mark(p, 2, st)) != SLRA_OK) return s;
        BwdMaps m;
        const uint64_t rows = static_cast<uint64_t>(g.BH()) * g.Lp;
        if (!make_map_headmajor(&m.q128, w.qh, rows, g.D, 128) || !make_map_headmajor(&m.do128, doh, rows, g.D, 128) ||
            !make_map_headmajor(&m.kb, w.kh, rows, g.D, g.block) || !make_map_headmajor(&m.vb, w.vh, rows, g.D, g.block) ||
            !make_map_headmajor(&m.k128, w.kh, rows, g.D, 128) || !make_map_headmajor(&m.v128, w.vh, rows, g.D, 128) ||
            !make_map_headmajor(&m.qb, w.qh, rows, g.D, g.block) || !make_map_headmajor(&m.dob, doh, rows, g.D, g.block))
            return SLRA_ERR_CUDA;
        m.between = static_cast<cudaEvent_t>(p->stage_events[3]);
        BwdArgs ba;
        ba.idx = w.idx;
        ba.keep = g.keep;
        ba.inv = inv;
        ba.inv_cnt = inv_cnt;
        ba.lse = lse;
        ba.delta = delta;
        ba.tab = w.tab;
        for (int e = 0; e < kMaxPairs; ++e)
            ba.pair_info[e] = e < d.meta.npairs ? make_int2(d.meta.axis[e], d.meta.tab_off[e]) : make_int2(0, 0);
        ba.dq = dq;
        ba.dk = dk;
        ba.dv = dv;
        ba.accumulate = 0;
        ba.status = w.status;
        ba.timeout_ns = timeout_of(p);
        if ((s = cuda_status(launch_bwd_sparse(m, ba, g, st))) != SLRA_OK) return s;
    } else if ((s = mark(p, 2, st)) != SLRA_OK || (s = mark(p, 3, st)) != SLRA_OK) {
        return s;
    }
    if ((s = mark(p, 4, st)) != SLRA_OK) return s;
    if (lowrank) {
        LrBwdArgs l;
        l.q = static_cast<const __nv_bfloat16*>(q);
        l.k = static_cast<const __nv_bfloat16*>(k);
        l.v = static_cast<const __nv_bfloat16*>(v);
        l.A = static_cast<const __nv_bfloat16*>(A);
        l.proj_separate = p->proj_separate ? 1 : 0;
        l.proj_per_head = p->proj_per_head ? 1 : 0;
        l.dout = d.gated ? dolr : dout;
        l.S = w.S;
        l.z = w.z;
        l.tab = w.tab;
        l.pairs = w.pairs;
        l.dq = dq;
        l.dk = dk;
        l.dv = dv;
        l.dA = dA;
        l.ds_part = reinterpret_cast<float*>(base + bl.ds_part);
        l.dz_part = reinterpret_cast<float*>(base + bl.dz_part);
        l.da_part = reinterpret_cast<float*>(base + bl.da_part);
        l.dS = reinterpret_cast<float*>(base + bl.dS);
        l.dz = reinterpret_cast<float*>(base + bl.dz);
        l.nsplit = bl.ns;
        l.meta = &d.meta;
        l.status = w.status;
        l.timeout_ns = timeout_of(p);
        l.accumulate = sparse ? 1 : 0;
        if ((s = cuda_status(launch_lr_bwd(l, g, st))) != SLRA_OK) return s;
    } else if (cudaMemsetAsync(dA, 0, ab, st) != cudaSuccess) {
        return SLRA_ERR_CUDA;
    }
    if (d.gated &&
        (s = cuda_status(launch_gate_final(static_cast<const __nv_bfloat16*>(q), dlogit,
                                           static_cast<const float*>(p->gate_w), g, dq,
                                           reinterpret_cast<float*>(base + bl.gpart), dgw, dgb, st))) != SLRA_OK)
        return s;
    if ((s = mark(p, 5, st)) != SLRA_OK) return s;
    return mark(p, 6, st);
}
}  // namespace

slra_status slra_attn_bwd(const slra_problem* p, const void* q, const void* k, const void* v, const void* A,
                          const float* dout, float* dq, float* dk, float* dv, float* dA, void* workspace,
                          size_t workspace_bytes, slra_stream_t stream) {
    return bwd_impl(p, q, k, v, A, dout, dq, dk, dv, dA, workspace, workspace_bytes, stream, false);
}

slra_status slra_attn_bwd_saved(const slra_problem* p, const void* q, const void* k, const void* v, const void* A,
                                const float* dout, float* dq, float* dk, float* dv, float* dA, void* workspace,
                                size_t workspace_bytes, slra_stream_t stream) {
    return bwd_impl(p, q, k, v, A, dout, dq, dk, dv, dA, workspace, workspace_bytes, stream, true);
}

slra_status slra_attn_fwd_train(const slra_problem* p, const void* q, const void* k, const void* v, const void* A,
                                void* out, void* workspace, size_t workspace_bytes, slra_stream_t stream) {
    Derived d;
    slra_status s = check_bwd_problem(p, &d);
    if (s != SLRA_OK) return s;
    if ((s = check_fwd_args(p, d, q, k, v, A, out, workspace, workspace_bytes)) != SLRA_OK) return s;
    const BwdLayout bl = bwd_layout(d);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < bl.total)
        return SLRA_ERR_WORKSPACE;
    if ((s = check_device()) != SLRA_OK) return s;
    uint8_t* base = static_cast<uint8_t*>(workspace);
    const int branches = p->branches == 0 ? SLRA_BRANCH_BOTH : p->branches;
    const bool sparse = (branches & SLRA_BRANCH_SPARSE) != 0;
    return fwd_impl(p, d, q, k, v, A, out, workspace, reinterpret_cast<cudaStream_t>(stream),
                    sparse ? reinterpret_cast<float*>(base + bl.lse) : nullptr,
                    sparse ? reinterpret_cast<float*>(base + bl.os) : nullptr);
}

slra_status slra_get_device_status(slra_stream_t stream, int32_t* status) {
    if (!status) return SLRA_ERR_INVALID_ARG;
    slra_status s = check_device();
    if (s != SLRA_OK) return s;
    int v = 0;
    const int zero = 0;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess ||
        cudaMemcpyFromSymbol(&v, slra::g_call_status, sizeof v) != cudaSuccess ||
        cudaMemcpyToSymbol(slra::g_call_status, &zero, sizeof zero) != cudaSuccess) {
        cudaGetLastError();
        return SLRA_ERR_CUDA;
    }
    *status = (v & kDevTimeout) ? SLRA_ERR_DEVICE_TIMEOUT : ((v & kDevRange) ? SLRA_ERR_RANGE : SLRA_OK);
    return SLRA_OK;
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------
// Allocation-free low-rank summary.  Its scratch (status word, rotary tables, split-L partial sums) is
// this file-scope device array; host code must not pass the array's name to a kernel (on the host it
// is only a stand-in), so its device address is looked up once per device and cached.
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[SLRA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
constexpr size_t kNoallocStatusBytes = 256;  // the status word, at the start of the scratch
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up on first use).
slra_status scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return SLRA_ERR_NO_DEVICE;
    }
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return SLRA_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return SLRA_OK;
}

// Tokens per step of the partial-sum kernel: 128-token tiles on the tensor cores (head_dim 128), 32 on
// the CUDA cores; a split covers ceil(tiles / nsplit) consecutive steps.
int64_t lowrank_steps(const Geom& g) { return g.D == 128 ? (g.L + 127) / 128 : (g.L + 31) / 32; }

}  // namespace

extern "C" slra_status slra_lowrank_summary_noalloc(const slra_problem* p, const void* k, const void* v,
                                                    const void* A, float* S, float* z, slra_stream_t stream) {
    Derived d;
    slra_status s = derive(p, &d);
    if (s != SLRA_OK) return s;
    if (!k || !v || !A || !S || !z) return SLRA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(A) || !aligned16(S) || !aligned16(z)) return SLRA_ERR_ALIGNMENT;
    const Geom& g = d.g;
    // scratch: [status word] [cos/sin table | pair info] [partial S] [partial z], each 256-B aligned
    const size_t tab_bytes = align_up(sizeof(double2) * static_cast<size_t>(d.table_entries) + sizeof(int2) * kMaxPairs, 256);
    const size_t fixed = kNoallocStatusBytes + tab_bytes;
    const size_t per_split = static_cast<size_t>(g.BH()) * g.R * (g.D + 1) * sizeof(float) + 512;
    if (fixed + per_split > SLRA_NOALLOC_SCRATCH_BYTES) return SLRA_ERR_SCRATCH_LIMIT;
    int64_t nsplit = d.nsplit;
    const int64_t fit = static_cast<int64_t>((SLRA_NOALLOC_SCRATCH_BYTES - fixed) / per_split);
    if (nsplit > fit) nsplit = fit;
    // with fewer splits, re-balance so that no split is left without a step: ceil(steps / per split)
    const int64_t steps = lowrank_steps(g);
    const int64_t per = (steps + nsplit - 1) / nsplit;
    nsplit = (steps + per - 1) / per;
    if ((s = check_device()) != SLRA_OK) return s;
    void* scratch = nullptr;
    if ((s = scratch_address(&scratch)) != SLRA_OK) return s;
    uint8_t* base = static_cast<uint8_t*>(scratch);
    int* status = reinterpret_cast<int*>(base);
    double2* tab = reinterpret_cast<double2*>(base + kNoallocStatusBytes);
    int2* pairs = reinterpret_cast<int2*>(base + kNoallocStatusBytes + sizeof(double2) * d.table_entries);
    float* s_part = reinterpret_cast<float*>(base + fixed);
    float* z_part = reinterpret_cast<float*>(
        base + fixed + align_up(static_cast<size_t>(g.BH()) * nsplit * g.R * g.D * sizeof(float), 256));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // The status word starts each call at zero (an async memset allocates nothing).  The kernels below
    // write all the other scratch they later read (the whole table, every partial slot of every split),
    // unless a bounded wait runs out: the status word then reports the timeout and S, z are unspecified.
    if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return SLRA_ERR_CUDA;
    if (launch_rope_table(tab, pairs, d.meta, d.table_entries, st) != cudaSuccess) return SLRA_ERR_CUDA;
    if (lowrank_partial(d, k, v, A, tab, pairs, static_cast<int>(nsplit), s_part, z_part, status, timeout_of(p),
                        debug_wait_of(p), st) != cudaSuccess)
        return SLRA_ERR_CUDA;
    return cuda_status(launch_lowrank_reduce(s_part, z_part, g, static_cast<int>(nsplit), S, z, nullptr, nullptr,
                                             nullptr, st));
}

extern "C" slra_status slra_noalloc_device_status(slra_stream_t stream, int32_t* status) {
    if (!status) return SLRA_ERR_INVALID_ARG;
    slra_status s = check_device();
    if (s != SLRA_OK) return s;
    void* scratch = nullptr;
    if ((s = scratch_address(&scratch)) != SLRA_OK) return s;
    int v = 0;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return SLRA_ERR_CUDA;
    if (cudaMemcpy(&v, scratch, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return SLRA_ERR_CUDA;
    if (cudaMemset(scratch, 0, sizeof v) != cudaSuccess) return SLRA_ERR_CUDA;
    *status = (v & kDevTimeout) ? SLRA_ERR_DEVICE_TIMEOUT : ((v & kDevRange) ? SLRA_ERR_RANGE : SLRA_OK);
    return SLRA_OK;
}
