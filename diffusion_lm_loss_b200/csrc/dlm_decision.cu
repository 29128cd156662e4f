// dlm_decision.cu -- typed-decision losses at label slots, forward + backward.
//
// "Native diffusion language-model training", Typed-decision training: the
// decision loss combines candidate-restricted CE, full-vocabulary CE and a
// 0.1 Brier term; Labels: hard / dist / set labels, labels.label_softmax
// (restricted, full or both) and hard_label_smoothing (spread over the
// question's answer tokens; Brier targets unchanged); Adapters, merging and
// inference: the restricted-label and Brier terms are computed over the
// allowed answers, the full-vocabulary CE over the whole vocabulary.
//
// Each label slot is one bf16 logits row z (the final read computes logits
// at label slots only) and the K <= 128 answer tokens of its question.  With
// r = softmax of the K candidate logits, P = softmax over the vocabulary, q
// the CE target and y the Brier target over the K answers (Q = sum q):
//   CE_res = -sum q_k log r_k,  CE_full = -sum q_k log P(a_k),
//   Brier  = sum (r_k - y_k)^2,  loss = mean over slots of the chosen terms;
//   dz_v   = g w [full] (Q P_v - q(v))                       every v
//          + g w ([res] (Q r_k - q_k) + b 2 r_k ((r_k - y_k) - sum_j r_j (r_j - y_j)))
//                                                           at v = a_k.
//
// The work is a streaming pass over n_slots rows of V bf16 values, read
// twice (the second time from L2) and written once: HBM-bound, a few tens
// of MB per call.  A handful of rows cannot fill 148 SMs, so each row is
// split over several CTAs by columns.  Fast path (16-byte aligned rows):
//   1. k_dec_cluster (one cluster of 1-8 CTAs per slot): each CTA's
//      (max, sum exp) of its split, exchanged through distributed shared
//      memory, then the gradient of its split and the answer entries;
//   2. k_dec_reduce  (1 CTA): the mean over slots in a fixed order, double,
//      and the status word.
// General path (any row stride or alignment): k_dec_partial (per-split
// partials to the workspace), k_dec_grad (every CTA of a row merges them and
// writes its split), k_dec_reduce.
// Invalid slots (a row or answer offsets outside the given arrays, an answer
// id outside [0, V), repeated answer ids, K outside 1..128, a malformed
// label) set a status bit and contribute a zero loss and a zero gradient row.
#include "dlm_device.cuh"
#include "dlm_host.h"

namespace dlm {

constexpr int kDecThreads = 256;
constexpr int kDecUnroll = 4;          // 16-byte loads in flight per thread
constexpr float kDecLog2e = 1.4426950408889634f;

struct DecParams {
    const uint16_t* logits;
    int64_t ld;
    int vocab;
    const int64_t* slot_rows;          // logits row of each slot, or null (row = slot)
    int64_t n_rows;                    // rows of the logits tensor
    const int32_t* cand_off;           // [n_slots + 1]
    int64_t n_cands;                   // entries of cand_ids and val
    const int32_t* cand_ids;           // answer token ids
    const int32_t* kind;               // [n_slots] DLM_LABEL_*
    const float* val;                  // one value per answer (see dlm.h)
    int n_slots;
    int n_split;
    int chunk;                         // columns per split, a multiple of 8
    int use_res, use_full;
    float brier_w, smoothing, grad_scale, w;
    float2* partial;                   // [n_slots][n_split] (max, sum exp)
    float* slot_loss;                  // [n_slots]
    float* loss;                       // [1]
    uint16_t* dlogits;
    int64_t ld_out;
    uint32_t* status;
    uint32_t* err;                     // cluster path: [n_slots][n_split] error words, or null
    int vec;                           // 16-byte loads and stores allowed
};

// (m, s) pairs stand for s * exp(m); merging keeps the larger max.  An
// all -inf part (s = 0) merges as the identity.
__device__ __forceinline__ void lse_merge(float& m, float& s, float m2, float s2) {
    if (s2 == 0.f) return;
    if (s == 0.f) { m = m2; s = s2; return; }
    const float M = fmaxf(m, m2);
    s = s * ex2((m - M) * kDecLog2e) + s2 * ex2((m2 - M) * kDecLog2e);
    m = M;
}

__device__ __forceinline__ void acc_value(float x, float& m, float& s) {
    if (x == -INFINITY) return;
    if (x > m) { s = s * ex2((m - x) * kDecLog2e); m = x; }   // s = 0 while m = -inf
    s += ex2((x - m) * kDecLog2e);
}

__device__ __forceinline__ void acc_vec(uint4 r, float& m, float& s) {
    const float mx = bf16x8_max(r);
    if (mx == -INFINITY) return;
    if (mx > m) { s = s * ex2((m - mx) * kDecLog2e); m = mx; }
    const uint32_t w4[4] = {r.x, r.y, r.z, r.w};
    #pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float lo = bf16lo(w4[k]), hi = bf16hi(w4[k]);
        s += (lo == -INFINITY ? 0.f : ex2((lo - m) * kDecLog2e));
        s += (hi == -INFINITY ? 0.f : ex2((hi - m) * kDecLog2e));
    }
}

// The logits row of `slot` and whether it lies inside the logits tensor
// (slot_rows is device data the host cannot check); an invalid row reads
// row 0 instead, harmlessly, and the slot is refused.
__device__ __forceinline__ bool slot_row_ok(const DecParams& P, int slot, int64_t& row) {
    row = P.slot_rows ? P.slot_rows[slot] : int64_t(slot);
    const bool ok = row >= 0 && row < P.n_rows;
    if (!ok) row = 0;
    return ok;
}

__global__ void __launch_bounds__(kDecThreads) k_dec_partial(DecParams P) {
    __shared__ float sm_m[kDecThreads / 32], sm_s[kDecThreads / 32];
    const int split = blockIdx.x, slot = blockIdx.y, tid = threadIdx.x;
    pdl_wait();                        // the previous call may still read the workspace
    pdl_launch_dependents();
    if (split == 0 && slot == 0 && tid == 0) *P.status = 0u;
    int64_t row;
    slot_row_ok(P, slot, row);
    const uint16_t* x = P.logits + row * P.ld;
    const int c0 = split * P.chunk;
    const int c1 = min(c0 + P.chunk, P.vocab);
    float m = -INFINITY, s = 0.f;
    int cv = c0;                       // first column left for the scalar loop
    if (P.vec) {
        const int nv = (c1 - c0) / 8;  // whole 8-column vectors of this split
        const uint4* xv = reinterpret_cast<const uint4*>(x + c0);
        int i = tid;
        for (; i + (kDecUnroll - 1) * kDecThreads < nv; i += kDecUnroll * kDecThreads) {
            uint4 r[kDecUnroll];
            #pragma unroll
            for (int u = 0; u < kDecUnroll; ++u) r[u] = __ldg(xv + i + u * kDecThreads);
            #pragma unroll
            for (int u = 0; u < kDecUnroll; ++u) acc_vec(r[u], m, s);
        }
        for (; i < nv; i += kDecThreads) acc_vec(__ldg(xv + i), m, s);
        cv = c0 + nv * 8;
    }
    for (int c = cv + tid; c < c1; c += kDecThreads) acc_value(bf16_bits_to_float(x[c]), m, s);
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
        lse_merge(m, s, m2, s2);
    }
    if ((tid & 31) == 0) { sm_m[tid >> 5] = m; sm_s[tid >> 5] = s; }
    __syncthreads();
    if (tid == 0) {
        float M = sm_m[0], S = sm_s[0];
        for (int k = 1; k < kDecThreads / 32; ++k) lse_merge(M, S, sm_m[k], sm_s[k]);
        P.partial[int64_t(slot) * P.n_split + split] = make_float2(M, S);
    }
}

__device__ __forceinline__ float warp_sum(float v) {
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Per-slot state in shared memory: what one warp works out about the
// slot's answers and label.
struct DecSlot {
    int id[DLM_DECISION_MAX_ANSWERS];     // answer token ids
    float z[DLM_DECISION_MAX_ANSWERS];    // their logits
    float q[DLM_DECISION_MAX_ANSWERS];    // CE target
    float gr[DLM_DECISION_MAX_ANSWERS];   // restricted-CE + Brier part of d loss / dz (no g w)
    float g[DLM_DECISION_MAX_ANSWERS];    // the full gradient value written at each answer token
    float Q, qz, ce_res, brier, coef;     // sum q, sum q z, CE_res, Brier; dense coefficient g w [full] Q
    int K;                                // answer entries to write (0 for an invalid slot)
    uint32_t bad;                         // status bits the slot raises (0 when valid)
};

// One warp, before the row's lse is known: the K answer tokens and the
// label -- validity, the restricted softmax, the targets, CE_res, Brier and
// the restricted + Brier part of each answer's gradient.  Needs only the K
// answer logits, so it runs while the row itself is still being loaded.
__device__ __forceinline__ void dec_slot_prepare(const DecParams& P, int slot, const uint16_t* x, bool row_ok,
                                                 int lane, DecSlot& S) {
    const int o0 = P.cand_off[slot], o1 = P.cand_off[slot + 1];
    const int K = o1 - o0;
    const int kind = P.kind[slot];
    // 3: the slot's row or its answer offsets lie outside the given arrays;
    // 2: a malformed label; 1: an answer id outside the vocabulary
    int bad = (!row_ok || o0 < 0 || o1 < o0 || int64_t(o1) > P.n_cands) ? 3 : 0;
    if (!bad) bad = (K < 1 || K > DLM_DECISION_MAX_ANSWERS) ? 2 : 0;
    if (!bad) bad = (kind != DLM_LABEL_HARD && kind != DLM_LABEL_DIST && kind != DLM_LABEL_SET) ? 2 : 0;
    float z[4], v[4];
    int id[4];
    int n_one = 0, n_other = 0;    // label checks: values equal to 1, and not in {0, 1}
    int bad_id = 0, bad_dist = 0;
    #pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int k = lane + 32 * j;
        id[j] = -1; z[j] = -INFINITY; v[j] = 0.f;
        if (!bad && k < K) {
            id[j] = P.cand_ids[o0 + k];
            v[j] = P.val[o0 + k];
        }
    }
    #pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int k = lane + 32 * j;
        if (!bad && k < K) {
            if (id[j] < 0 || id[j] >= P.vocab) { bad_id = 1; id[j] = -1; }
            else z[j] = bf16_bits_to_float(x[id[j]]);
            n_one += (v[j] == 1.f);
            n_other += (v[j] != 0.f && v[j] != 1.f);
            bad_dist |= !(v[j] >= 0.f && v[j] < INFINITY);
            S.id[k] = id[j];
        }
    }
    __syncwarp();
    // repeated answer ids: each lane compares its answers with the earlier ones
    int dup = 0;
    if (!bad) {
        #pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = lane + 32 * j;
            if (k < K && id[j] >= 0)
                for (int i = 0; i < k; ++i) dup |= (S.id[i] == id[j]);
        }
    }
    n_one = warp_sum_i(n_one);
    n_other = warp_sum_i(n_other);
    bad_id = __any_sync(0xffffffffu, bad_id);
    dup = __any_sync(0xffffffffu, dup);
    bad_dist = __any_sync(0xffffffffu, bad_dist);
    if (!bad) {
        if (bad_id) bad = 1;
        else if (dup) bad = 2;
        else if (kind == DLM_LABEL_HARD && !(n_one == 1 && n_other == 0)) bad = 2;
        else if (kind == DLM_LABEL_SET && !(n_one >= 1 && n_other == 0)) bad = 2;
        else if (kind == DLM_LABEL_DIST && bad_dist) bad = 2;
    }
    if (!bad) {
        // candidate-restricted softmax
        const float cm = warp_max(fmaxf(fmaxf(z[0], z[1]), fmaxf(z[2], z[3])));
        float se = 0.f;
        #pragma unroll
        for (int j = 0; j < 4; ++j) se += (lane + 32 * j < K) ? expf(z[j] - cm) : 0.f;
        const float lse_r = cm + logf(warp_sum(se));
        const float n_set = float(n_one);
        float r[4], q[4], y[4];
        float Q = 0.f, qz = 0.f, ce_res = 0.f, brier = 0.f, D = 0.f;
        #pragma unroll
        for (int j = 0; j < 4; ++j) {
            const bool on = lane + 32 * j < K;
            r[j] = on ? expf(z[j] - lse_r) : 0.f;
            if (kind == DLM_LABEL_HARD) { y[j] = v[j]; q[j] = (1.f - P.smoothing) * v[j] + P.smoothing / float(K); }
            else if (kind == DLM_LABEL_SET) { y[j] = v[j] / n_set; q[j] = y[j]; }
            else { y[j] = v[j]; q[j] = v[j]; }
            if (!on) { q[j] = 0.f; y[j] = 0.f; }
            Q += q[j];
            qz += on ? q[j] * z[j] : 0.f;
            ce_res -= on ? q[j] * (z[j] - lse_r) : 0.f;
            const float d = r[j] - y[j];
            brier += d * d;
            D += r[j] * d;
        }
        Q = warp_sum(Q);
        qz = warp_sum(qz);
        ce_res = warp_sum(ce_res);
        brier = warp_sum(brier);
        D = warp_sum(D);
        #pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int k = lane + 32 * j;
            if (k < K) {
                float g = P.brier_w * 2.f * r[j] * ((r[j] - y[j]) - D);
                if (P.use_res) g += Q * r[j] - q[j];
                S.gr[k] = g;
                S.z[k] = z[j];
                S.q[k] = q[j];
            }
        }
        if (lane == 0) { S.Q = Q; S.qz = qz; S.ce_res = ce_res; S.brier = brier; }
    }
    if (lane == 0) {
        S.K = bad ? 0 : K;
        S.bad = bad == 0 ? 0u : bad == 1 ? DLM_DEV_BAD_TOKEN_ID : bad == 2 ? DLM_DEV_BAD_LABEL : DLM_DEV_BAD_LAYOUT;
    }
}

// One warp, once lse is known: the full-vocabulary CE and its share of each
// answer's gradient, the answers' final values (S.g), the dense coefficient
// (S.coef) and, from split 0, the slot's loss share.  Call after the
// prepare step is visible to the warp (same warp, or after a barrier).
__device__ __forceinline__ void dec_slot_finish(const DecParams& P, int slot, int split, float lse, int lane,
                                                DecSlot& S) {
    const int K = S.K;
    const float gw = P.grad_scale * P.w;
    const float Q = K > 0 ? S.Q : 0.f;
    for (int k = lane; k < K; k += 32) {
        float g = S.gr[k];
        if (P.use_full) g += Q * expf(S.z[k] - lse) - S.q[k];
        S.g[k] = gw * g;
    }
    if (lane == 0) {
        float slot_loss = 0.f;
        if (K > 0) {
            const float ce_full = Q * lse - S.qz;     // -sum q_k (z_k - lse)
            slot_loss = P.w * (P.use_res * S.ce_res + P.use_full * ce_full + P.brier_w * S.brier);
        }
        S.coef = gw * float(P.use_full) * Q;
        if (split == 0) P.slot_loss[slot] = slot_loss;
    }
}

__global__ void __launch_bounds__(kDecThreads) k_dec_grad(DecParams P) {
    __shared__ DecSlot S;
    __shared__ float s_lse;
    const int split = blockIdx.x, slot = blockIdx.y, tid = threadIdx.x;
    pdl_wait();                        // partials of k_dec_partial
    pdl_launch_dependents();
    int64_t row;
    const bool row_ok = slot_row_ok(P, slot, row);
    const uint16_t* x = P.logits + row * P.ld;
    if (tid == 0) {
        float M = -INFINITY, S = 0.f;
        for (int k = 0; k < P.n_split; ++k) {
            const float2 ps = P.partial[int64_t(slot) * P.n_split + k];
            lse_merge(M, S, ps.x, ps.y);
        }
        s_lse = M + logf(S);
    }
    __syncthreads();
    const float lse = s_lse;
    if (tid < 32) {
        dec_slot_prepare(P, slot, x, row_ok, tid, S);
        __syncwarp();
        dec_slot_finish(P, slot, split, lse, tid, S);
    }
    __syncthreads();
    if (tid == 0 && split == 0 && S.bad) atomicOr(P.status, S.bad);
    // the dense part of this split: coef * P_v (zeros for a restricted-only
    // loss or an invalid slot)
    const float coef = S.coef;
    const float sh = lse * kDecLog2e;
    uint16_t* out = P.dlogits + int64_t(slot) * P.ld_out;
    const int c0 = split * P.chunk;
    const int c1 = min(c0 + P.chunk, P.vocab);
    int cv = c0;
    if (P.vec) {
        const int nv = (c1 - c0) / 8;
        const uint4* xv = reinterpret_cast<const uint4*>(x + c0);
        uint4* ov = reinterpret_cast<uint4*>(out + c0);
        const uint64_t ef = policy_evict_first();
        int i = tid;
        for (; i + (kDecUnroll - 1) * kDecThreads < nv; i += kDecUnroll * kDecThreads) {
            uint4 rv[kDecUnroll];
            #pragma unroll
            for (int u = 0; u < kDecUnroll; ++u) rv[u] = __ldg(xv + i + u * kDecThreads);
            #pragma unroll
            for (int u = 0; u < kDecUnroll; ++u) {
                const uint32_t w4[4] = {rv[u].x, rv[u].y, rv[u].z, rv[u].w};
                uint32_t o4[4];
                #pragma unroll
                for (int k = 0; k < 4; ++k)
                    o4[k] = pack_bf16x2(coef * ex2(fmaf(bf16lo(w4[k]), kDecLog2e, -sh)),
                                        coef * ex2(fmaf(bf16hi(w4[k]), kDecLog2e, -sh)));
                st_global_v4_hint(ov + i + u * kDecThreads, make_uint4(o4[0], o4[1], o4[2], o4[3]), ef);
            }
        }
        for (; i < nv; i += kDecThreads) {
            const uint4 rv = __ldg(xv + i);
            const uint32_t w4[4] = {rv.x, rv.y, rv.z, rv.w};
            uint32_t o4[4];
            #pragma unroll
            for (int k = 0; k < 4; ++k)
                o4[k] = pack_bf16x2(coef * ex2(fmaf(bf16lo(w4[k]), kDecLog2e, -sh)),
                                    coef * ex2(fmaf(bf16hi(w4[k]), kDecLog2e, -sh)));
            st_global_v4_hint(ov + i, make_uint4(o4[0], o4[1], o4[2], o4[3]), ef);
        }
        cv = c0 + nv * 8;
    }
    for (int c = cv + tid; c < c1; c += kDecThreads) {
        const float g = coef * ex2(fmaf(bf16_bits_to_float(x[c]), kDecLog2e, -sh));
        out[c] = __bfloat16_as_ushort(__float2bfloat16_rn(g));
    }
    __syncthreads();                   // the dense stores of this CTA come first
    const int K = S.K;
    for (int k = tid; k < K; k += kDecThreads) {
        const int id = S.id[k];
        if (id >= c0 && id < c1) out[id] = __bfloat16_as_ushort(__float2bfloat16_rn(S.g[k]));
    }
}

// 16-byte read-only load with an L2 cache policy.
__device__ __forceinline__ uint4 ldg_v4_hint(const void* p, uint64_t pol) {
    uint4 r;
    asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p), "l"(pol));
    return r;
}

// Fast path: one thread-block cluster per slot, one CTA per split of the
// row (cluster rank = split; 1, 2, 4 or 8 splits).  Each CTA reads its split
// twice: the first time from HBM, kept in L2 with an evict_last policy (a
// call's label rows are tens of MB), for its (max, sum exp); the cluster
// exchanges only those two floats through distributed shared memory and
// every CTA merges the n_split partials in rank order into the same lse; the
// second read comes from L2 and writes the gradient, then the answer-token
// entries are rewritten as in k_dec_grad.  One warp works out the label
// meanwhile.  The CTAs hold nothing but a few KB of shared memory, so every
// cluster of a call is resident at once and no CTA waits for a second wave
// (holding each split in shared memory instead measured slower: the call's
// rows do not fit on chip at once).  The final cluster barrier keeps every
// CTA's partial alive until all peers have read it.
__global__ void __launch_bounds__(kDecThreads, 4) k_dec_cluster(DecParams P) {
    constexpr int kU = 4;              // 16-byte loads in flight per thread
    __shared__ __align__(8) float2 s_part;
    __shared__ float sm_m[kDecThreads / 32], sm_s[kDecThreads / 32];
    __shared__ DecSlot S;
    __shared__ float s_lse;
    const int tid = threadIdx.x, lane = tid & 31;
    const int split = int(cluster_ctarank()), slot = blockIdx.y;
    const int c0 = split * P.chunk;
    const int c1 = min(c0 + P.chunk, P.vocab);
    const int nvec = c1 > c0 ? (c1 - c0) / 8 : 0;
    pdl_wait();                        // inputs may come from the previous kernel
    pdl_launch_dependents();
    int64_t row;
    const bool row_ok = slot_row_ok(P, slot, row);
    const uint16_t* x = P.logits + row * P.ld;
    const uint4* xv = reinterpret_cast<const uint4*>(x + c0);
    const uint64_t keep = policy_evict_last(), drop = policy_evict_first();
    float m = -INFINITY, s = 0.f;
    {
        int i = tid;
        for (; i + (kU - 1) * kDecThreads < nvec; i += kU * kDecThreads) {
            uint4 r[kU];
            #pragma unroll
            for (int u = 0; u < kU; ++u) r[u] = ldg_v4_hint(xv + i + u * kDecThreads, keep);
            #pragma unroll
            for (int u = 0; u < kU; ++u) acc_vec(r[u], m, s);
        }
        for (; i < nvec; i += kDecThreads) acc_vec(ldg_v4_hint(xv + i, keep), m, s);
    }
    if (tid < 32) dec_slot_prepare(P, slot, x, row_ok, tid, S);
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
        lse_merge(m, s, m2, s2);
    }
    if (lane == 0) { sm_m[tid >> 5] = m; sm_s[tid >> 5] = s; }
    __syncthreads();
    if (tid == 0) {
        float M = sm_m[0], Ssum = sm_s[0];
        for (int k = 1; k < kDecThreads / 32; ++k) lse_merge(M, Ssum, sm_m[k], sm_s[k]);
        s_part = make_float2(M, Ssum);
    }
    cluster_sync_all();
    if (tid == 0) {
        float M = -INFINITY, Ssum = 0.f;
        for (int r = 0; r < P.n_split; ++r) {
            float pm, ps;
            const uint32_t a = mapa_shared(smem_addr(&s_part), uint32_t(r));
            asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(pm), "=f"(ps) : "r"(a) : "memory");
            lse_merge(M, Ssum, pm, ps);
        }
        s_lse = M + logf(Ssum);
    }
    __syncthreads();
    const float lse = s_lse;
    if (tid < 32) dec_slot_finish(P, slot, split, lse, tid, S);
    __syncthreads();
    if (tid == 0) P.err[int64_t(slot) * P.n_split + split] = split == 0 ? S.bad : 0u;
    const float coef = S.coef;
    const float sh = lse * kDecLog2e;
    uint16_t* out = P.dlogits + int64_t(slot) * P.ld_out;
    uint4* ov = reinterpret_cast<uint4*>(out + c0);
    {
        int i = tid;
        for (; i + (kU - 1) * kDecThreads < nvec; i += kU * kDecThreads) {
            uint4 r[kU];
            #pragma unroll
            for (int u = 0; u < kU; ++u) r[u] = ldg_v4_hint(xv + i + u * kDecThreads, drop);
            #pragma unroll
            for (int u = 0; u < kU; ++u) {
                const uint32_t w4[4] = {r[u].x, r[u].y, r[u].z, r[u].w};
                uint32_t o4[4];
                #pragma unroll
                for (int k = 0; k < 4; ++k)
                    o4[k] = pack_bf16x2(coef * ex2(fmaf(bf16lo(w4[k]), kDecLog2e, -sh)),
                                        coef * ex2(fmaf(bf16hi(w4[k]), kDecLog2e, -sh)));
                st_global_v4_hint(ov + i + u * kDecThreads, make_uint4(o4[0], o4[1], o4[2], o4[3]), drop);
            }
        }
        for (; i < nvec; i += kDecThreads) {
            const uint4 rv = ldg_v4_hint(xv + i, drop);
            const uint32_t w4[4] = {rv.x, rv.y, rv.z, rv.w};
            uint32_t o4[4];
            #pragma unroll
            for (int k = 0; k < 4; ++k)
                o4[k] = pack_bf16x2(coef * ex2(fmaf(bf16lo(w4[k]), kDecLog2e, -sh)),
                                    coef * ex2(fmaf(bf16hi(w4[k]), kDecLog2e, -sh)));
            st_global_v4_hint(ov + i, make_uint4(o4[0], o4[1], o4[2], o4[3]), drop);
        }
    }
    __syncthreads();
    const int K = S.K;
    for (int k = tid; k < K; k += kDecThreads) {
        const int id = S.id[k];
        if (id >= c0 && id < c1) out[id] = __bfloat16_as_ushort(__float2bfloat16_rn(S.g[k]));
    }
    cluster_sync_all();
}

constexpr int kDecRedThreads = 256;

// The mean over slots (fixed order, double) and, after the cluster path,
// the status word: the or of every CTA's error word (written on every call,
// so nothing needs zeroing between calls).
__global__ void __launch_bounds__(kDecRedThreads) k_dec_reduce(const float* __restrict__ slot_loss, int n,
                                                               float* __restrict__ loss,
                                                               const uint32_t* __restrict__ err, int n_err,
                                                               uint32_t* __restrict__ status) {
    __shared__ double red[kDecRedThreads];
    __shared__ uint32_t bits;
    const int tid = threadIdx.x;
    pdl_wait();                        // slot losses of the gradient kernel
    if (tid == 0) bits = 0u;
    __syncthreads();
    if (err) {
        uint32_t b = 0u;
        for (int i = tid; i < n_err; i += kDecRedThreads) b |= err[i];
        if (b) atomicOr(&bits, b);
    }
    double acc = 0.0;
    for (int i = tid; i < n; i += kDecRedThreads) acc += double(slot_loss[i]);
    red[tid] = acc;
    __syncthreads();
    if (err && tid == 0) *status = bits;
    for (int o = kDecRedThreads / 2; o > 0; o >>= 1) {
        if (tid < o) red[tid] += red[tid + o];
        __syncthreads();
    }
    if (tid == 0) *loss = float(red[0]);
}

struct DecPlan {
    int n_split, chunk;
    size_t partial_off, slot_loss_off, total;
};

// The cluster path: n_split in {1, 2, 4, 8} (a portable cluster size), the
// smallest that gives about 512 CTAs in all (3.5 per SM, every cluster
// resident at once) without cutting splits under 2,048 columns.  Needs
// vocab % 8 == 0 (16-byte vectors).
inline bool dec_cluster_plan(int n_slots, int vocab, int& n_split, int& chunk) {
    if (n_slots <= 0 || vocab % 8 != 0) return false;
    const int64_t want = (512 + n_slots - 1) / n_slots;   // CTAs wanted per slot
    int ns = 1;
    while (ns < 8 && ns < want && int64_t(vocab) / (2 * ns) >= 2048) ns *= 2;
    n_split = ns;
    chunk = int((int64_t(vocab) / 8 + ns - 1) / ns * 8);
    return true;
}

// Columns of a row per CTA: enough CTAs for two waves over 148 SMs, at
// least 2,048 columns each.
inline DecPlan dec_plan(int n_slots, int vocab) {
    DecPlan p{};
    const int want = n_slots > 0 ? (2 * 148 + n_slots - 1) / n_slots : 1;
    const int most = (vocab + 2047) / 2048;
    int ns = want < 1 ? 1 : (want > most ? most : want);
    if (ns < 1) ns = 1;
    p.chunk = int(((int64_t(vocab) + ns - 1) / ns + 7) / 8 * 8);
    p.n_split = int((int64_t(vocab) + p.chunk - 1) / p.chunk);
    size_t o = kWsAlign;               // status word in the first 256 bytes
    p.partial_off = o;                 // partials, or the cluster path's error words (up to 8 per slot)
    o = align_up(o + size_t(n_slots) * size_t(p.n_split > 8 ? p.n_split : 8) * sizeof(float2), kWsAlign);
    p.slot_loss_off = o;
    o = align_up(o + size_t(n_slots) * sizeof(float), kWsAlign);
    p.total = o;
    return p;
}

}  // namespace dlm

using namespace dlm;

extern "C" size_t dlm_decision_workspace_size(int32_t n_slots, int32_t vocab) {
    if (n_slots < 0 || n_slots > DLM_DECISION_MAX_SLOTS || vocab <= 0) return 0;
    return dec_plan(n_slots, vocab).total;
}

extern "C" dlm_status_t dlm_decision_loss_fwd_bwd(int32_t n_slots, const uint16_t* logits, int64_t n_rows,
                                                  int64_t ld, int32_t vocab, const int64_t* slot_rows,
                                                  const int32_t* cand_off, int64_t n_cands, const int32_t* cand_ids,
                                                  const int32_t* label_kind, const float* label_val,
                                                  int32_t label_softmax, float brier_weight,
                                                  float hard_label_smoothing, float grad_scale, float* loss,
                                                  float* slot_loss, uint16_t* dlogits, int64_t ld_out,
                                                  void* workspace, size_t workspace_bytes,
                                                  dlm_stream_t stream) {
    DLM_NVTX("dlm_decision_loss_fwd_bwd");
    if (n_slots < 0 || n_slots > DLM_DECISION_MAX_SLOTS || vocab <= 0) return DLM_ERR_INVALID_ARGUMENT;
    if (label_softmax < DLM_LABEL_SOFTMAX_RESTRICTED || label_softmax > DLM_LABEL_SOFTMAX_BOTH)
        return DLM_ERR_INVALID_ARGUMENT;
    if (!(brier_weight >= 0.f && brier_weight < INFINITY)) return DLM_ERR_INVALID_ARGUMENT;
    if (!(hard_label_smoothing >= 0.f && hard_label_smoothing <= 1.f)) return DLM_ERR_INVALID_ARGUMENT;
    if (!(grad_scale > -INFINITY && grad_scale < INFINITY)) return DLM_ERR_INVALID_ARGUMENT;
    if (!loss || !workspace) return DLM_ERR_INVALID_ARGUMENT;
    if (n_slots > 0 && (!logits || !cand_off || !cand_ids || !label_kind || !label_val || !dlogits))
        return DLM_ERR_INVALID_ARGUMENT;
    if (n_slots > 0 && (ld < vocab || ld_out < vocab || n_rows < 1 || n_cands < 0)) return DLM_ERR_INVALID_ARGUMENT;
    if (n_slots > 0 && !slot_rows && n_rows < n_slots) return DLM_ERR_INVALID_ARGUMENT;
    if (reinterpret_cast<uintptr_t>(workspace) % kWsAlign) return DLM_ERR_INVALID_ARGUMENT;
    const DecPlan plan = dec_plan(n_slots, vocab);
    if (workspace_bytes < plan.total) return DLM_ERR_WORKSPACE_TOO_SMALL;
    dlm_status_t st = check_device();
    if (st != DLM_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    DecParams P{};
    P.logits = logits;
    P.ld = ld;
    P.vocab = vocab;
    P.slot_rows = slot_rows;
    P.n_rows = n_rows;
    P.cand_off = cand_off;
    P.n_cands = n_cands;
    P.cand_ids = cand_ids;
    P.kind = label_kind;
    P.val = label_val;
    P.n_slots = n_slots;
    P.n_split = plan.n_split;
    P.chunk = plan.chunk;
    P.use_res = label_softmax != DLM_LABEL_SOFTMAX_FULL;
    P.use_full = label_softmax != DLM_LABEL_SOFTMAX_RESTRICTED;
    P.brier_w = brier_weight;
    P.smoothing = hard_label_smoothing;
    P.grad_scale = grad_scale;
    P.w = n_slots > 0 ? 1.0f / float(n_slots) : 0.f;
    P.partial = reinterpret_cast<float2*>(ws + plan.partial_off);
    P.slot_loss = slot_loss ? slot_loss : reinterpret_cast<float*>(ws + plan.slot_loss_off);
    P.loss = loss;
    P.dlogits = dlogits;
    P.ld_out = ld_out;
    P.status = reinterpret_cast<uint32_t*>(ws);
    P.vec = (ld % 8 == 0) && (ld_out % 8 == 0) && aligned16(logits) && aligned16(dlogits);
    int cl_split = 0, cl_chunk = 0;
    if (n_slots > 0 && P.vec && dec_cluster_plan(n_slots, vocab, cl_split, cl_chunk)) {
        // one cluster per slot: lse partials through distributed shared memory
        P.err = reinterpret_cast<uint32_t*>(ws + plan.partial_off);   // n_slots x cl_split words fit
        DecParams C = P;
        C.n_split = cl_split;
        C.chunk = cl_chunk;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(unsigned(cl_split), unsigned(n_slots));
        cfg.blockDim = dim3(kDecThreads);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = s;
        cudaLaunchAttribute at[2];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = unsigned(cl_split);
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = at;
        cfg.numAttrs = 2;
        const cudaError_t e = cudaLaunchKernelEx(&cfg, k_dec_cluster, C);
        if (e != cudaSuccess) { cudaGetLastError(); return cuda_status(e, "k_dec_cluster launch"); }
    } else if (n_slots > 0) {
        const dim3 grid(unsigned(plan.n_split), unsigned(n_slots));
        if ((st = launch_pdl(k_dec_partial, grid, dim3(kDecThreads), 0, s, "k_dec_partial launch", P)) != DLM_OK)
            return st;
        if ((st = launch_pdl(k_dec_grad, grid, dim3(kDecThreads), 0, s, "k_dec_grad launch", P)) != DLM_OK)
            return st;
    } else {
        cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(uint32_t), s);
        if (e != cudaSuccess) { cudaGetLastError(); return cuda_status(e, "status reset"); }
    }
    const bool clustered = cl_split > 0;
    return launch_pdl(k_dec_reduce, dim3(1), dim3(kDecRedThreads), 0, s, "k_dec_reduce launch",
                      (const float*)P.slot_loss, n_slots, loss, clustered ? (const uint32_t*)P.err : nullptr,
                      clustered ? n_slots * cl_split : 0, P.status);
}
