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
constexpr float kDecLn2 = 0.6931471805599453f;

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

// Warp max of a float in one instruction (redux.sync .f32, sm_100a).
__device__ __forceinline__ float warp_max_f32(float v) {
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
}

// Every lane's (m, s) merged over the warp: the warp max in one
// instruction, each lane's sum rescaled to it, then a butterfly sum.
// Every lane ends with the same bits (the butterfly's additions only swap
// operands between lanes).  An all-empty warp (max -inf) gives (-inf, 0).
__device__ __forceinline__ void warp_lse(float& m, float& s) {
    const float M = warp_max_f32(m);
    s = (M == -INFINITY) ? 0.f : s * ex2((m - M) * kDecLog2e);
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    m = M;
}

__device__ __forceinline__ void acc_value(float x, float& m, float& s) {
    if (x == -INFINITY) return;
    if (x > m) { s = s * ex2((m - x) * kDecLog2e); m = x; }   // s = 0 while m = -inf
    s += ex2((x - m) * kDecLog2e);
}

// (max, sum exp) over N 16-byte vectors: one max and at most one rescale
// per batch, the exponents by packed FMAs (two lanes per instruction) and
// two ex2 per pair.  Once the batch max is folded in, m is finite, so a
// -inf element gives ex2(-inf) = 0 with no test of its own.
template <int N>
__device__ __forceinline__ void acc_batch(const uint4 (&r)[N], float& m, float& s) {
    float cm = bf16x8_max(r[0]);
    #pragma unroll
    for (int u = 1; u < N; ++u) cm = fmaxf(cm, bf16x8_max(r[u]));
    if (cm == -INFINITY) return;
    if (cm > m) { s = s * ex2((m - cm) * kDecLog2e); m = cm; }   // s = 0 while m = -inf
    const uint64_t l2e = f2pack(kDecLog2e, kDecLog2e);
    const uint64_t nmb = f2pack(-m * kDecLog2e, -m * kDecLog2e);
    uint64_t acc = f2pack(0.f, 0.f);
    #pragma unroll
    for (int u = 0; u < N; ++u) {
        const uint32_t w4[4] = {r[u].x, r[u].y, r[u].z, r[u].w};
        #pragma unroll
        for (int k = 0; k < 4; ++k) {
            float t0, t1;
            f2unpack(f2fma(f2pack(bf16lo(w4[k]), bf16hi(w4[k])), l2e, nmb), t0, t1);
            acc = f2add(acc, f2pack(ex2(t0), ex2(t1)));
        }
    }
    float a0, a1;
    f2unpack(acc, a0, a1);
    s += a0 + a1;
}

// The dense gradient of one 16-byte vector: g = coef 2^(x log2e - lse log2e)
// by packed FMAs; for coef > 0 the factor is folded into the exponent
// (nlb = log2 coef - lse log2e), otherwise nlb = -lse log2e and each value
// is multiplied by `mul` = coef.
__device__ __forceinline__ uint4 dec_dense_vec(uint4 r, uint64_t l2e, uint64_t nlb, bool fold, float mul) {
    const uint32_t w4[4] = {r.x, r.y, r.z, r.w};
    uint32_t o4[4];
    #pragma unroll
    for (int k = 0; k < 4; ++k) {
        float t0, t1;
        f2unpack(f2fma(f2pack(bf16lo(w4[k]), bf16hi(w4[k])), l2e, nlb), t0, t1);
        float g0 = ex2(t0), g1 = ex2(t1);
        if (!fold) { g0 *= mul; g1 *= mul; }
        o4[k] = pack_bf16x2(g0, g1);
    }
    return make_uint4(o4[0], o4[1], o4[2], o4[3]);
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
            acc_batch<kDecUnroll>(r, m, s);
        }
        for (; i < nv; i += kDecThreads) {
            const uint4 r[1] = {__ldg(xv + i)};
            acc_batch<1>(r, m, s);
        }
        cv = c0 + nv * 8;
    }
    for (int c = cv + tid; c < c1; c += kDecThreads) acc_value(bf16_bits_to_float(x[c]), m, s);
    warp_lse(m, s);
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
// N independent warp sums, their butterflies interleaved (one shuffle
// latency per step for all N).
template <int N>
__device__ __forceinline__ void warp_sum_n(float (&v)[N]) {
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        #pragma unroll
        for (int i = 0; i < N; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
    }
}

// Per-slot state in shared memory: what one warp works out about the
// slot's answers and label.
struct DecSlot {
    int id[DLM_DECISION_MAX_ANSWERS];     // answer token ids, as given
    float z[DLM_DECISION_MAX_ANSWERS];    // the answers' logits
    float q[DLM_DECISION_MAX_ANSWERS];    // CE target
    float gr[DLM_DECISION_MAX_ANSWERS];   // restricted-CE + Brier part of d loss / dz (no g w)
    float g[DLM_DECISION_MAX_ANSWERS];    // the full gradient value written at each answer token
    float Q, qz, ce_res, brier, coef;     // sum q, sum q z, CE_res, Brier; dense coefficient g w [full] Q
    int K;                                // answer entries to write (0 for an invalid slot)
    uint32_t bad;                         // status bits the slot raises (0 when valid)
};

// A slot's answer range and label kind, and the first check of them:
// bad = 3 when the slot's row or its answer offsets lie outside the given
// arrays, 2 when K is outside 1..128 or the label kind is unknown, else 0.
struct DecHead {
    int o0, K, kind, bad;
};

__device__ __forceinline__ DecHead dec_slot_head(const DecParams& P, bool row_ok, int o0, int o1, int kind) {
    DecHead h;
    h.o0 = o0;
    h.K = o1 - o0;
    h.kind = kind;
    h.bad = (!row_ok || o0 < 0 || o1 < o0 || int64_t(o1) > P.n_cands) ? 3 : 0;
    if (!h.bad) h.bad = (h.K < 1 || h.K > DLM_DECISION_MAX_ANSWERS) ? 2 : 0;
    if (!h.bad) h.bad = (kind != DLM_LABEL_HARD && kind != DLM_LABEL_DIST && kind != DLM_LABEL_SET) ? 2 : 0;
    return h;
}

// One warp, before the row's lse is known, given each lane's answers
// (answer k = lane + 32 j: id, label value and the logit's bf16 bits; the
// ids also in S.id): the label's validity, the restricted softmax, the
// targets, CE_res, Brier and the restricted + Brier part of each answer's
// gradient.  Needs only the K answer logits, so it overlaps the row's
// stream; the logits are first used after the label checks, so their loads
// can still be in flight during them.
__device__ __forceinline__ void dec_slot_compute(const DecParams& P, const DecHead& h, int lane, DecSlot& S,
                                                 const int (&id_in)[4], const float (&v)[4],
                                                 const uint16_t (&zb)[4]) {
    const int K = h.K;
    const int kind = h.kind;
    // 3: the slot's row or its answer offsets lie outside the given arrays;
    // 2: a malformed label; 1: an answer id outside the vocabulary
    int bad = h.bad;
    int id[4];
    int n_one = 0, n_other = 0;    // label checks: values equal to 1, and not in {0, 1}
    int bad_id = 0, bad_dist = 0;
    #pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int k = lane + 32 * j;
        id[j] = -1;
        if (!bad && k < K) {
            id[j] = id_in[j];
            if (id[j] < 0 || id[j] >= P.vocab) { bad_id = 1; id[j] = -1; }
            n_one += (v[j] == 1.f);
            n_other += (v[j] != 0.f && v[j] != 1.f);
            bad_dist |= !(v[j] >= 0.f && v[j] < INFINITY);
        }
    }
    // repeated answer ids: lanes of one group of 32 that hold the same id
    // (one match instruction), and each id against the earlier groups (an
    // out-of-range id never equals a valid one)
    int dup = 0;
    if (!bad) {
        #pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (32 * j >= K) break;
            const int k = lane + 32 * j;
            const bool has = k < K && id[j] >= 0;
            dup |= __popc(__match_any_sync(0xffffffffu, has ? id[j] : -1 - lane)) > 1;
            if (has)
                for (int i = 0; i < 32 * j; ++i) dup |= (S.id[i] == id[j]);
        }
    }
    n_one = int(__reduce_add_sync(0xffffffffu, unsigned(n_one)));
    n_other = int(__reduce_add_sync(0xffffffffu, unsigned(n_other)));
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
        float z[4];
        #pragma unroll
        for (int j = 0; j < 4; ++j) z[j] = id[j] >= 0 ? bf16_bits_to_float(zb[j]) : -INFINITY;
        // candidate-restricted softmax (hardware ex2 / lg2: relative error
        // about 2^-22, far below the bf16 gradient and the loss tolerance)
        const float cm = warp_max_f32(fmaxf(fmaxf(z[0], z[1]), fmaxf(z[2], z[3])));
        float se = 0.f;
        #pragma unroll
        for (int j = 0; j < 4; ++j) se += (lane + 32 * j < K) ? ex2((z[j] - cm) * kDecLog2e) : 0.f;
        const float lse_r = cm + lg2(warp_sum(se)) * kDecLn2;
        const float n_set = float(n_one);
        float r[4], q[4], y[4];
        // sums over the answers: Q, sum q z, CE_res, Brier, D = sum r (r - y)
        float t[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
        #pragma unroll
        for (int j = 0; j < 4; ++j) {
            const bool on = lane + 32 * j < K;
            r[j] = on ? ex2((z[j] - lse_r) * kDecLog2e) : 0.f;
            if (kind == DLM_LABEL_HARD) { y[j] = v[j]; q[j] = (1.f - P.smoothing) * v[j] + P.smoothing / float(K); }
            else if (kind == DLM_LABEL_SET) { y[j] = v[j] / n_set; q[j] = y[j]; }
            else { y[j] = v[j]; q[j] = v[j]; }
            if (!on) { q[j] = 0.f; y[j] = 0.f; }
            t[0] += q[j];
            t[1] += on ? q[j] * z[j] : 0.f;
            t[2] -= on ? q[j] * (z[j] - lse_r) : 0.f;
            const float d = r[j] - y[j];
            t[3] += d * d;
            t[4] += r[j] * d;
        }
        warp_sum_n(t);                 // the five butterflies interleaved
        const float Q = t[0], D = t[4];
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
        if (lane == 0) { S.Q = Q; S.qz = t[1]; S.ce_res = t[2]; S.brier = t[3]; }
    }
    if (lane == 0) {
        S.K = bad ? 0 : K;
        S.bad = bad == 0 ? 0u : bad == 1 ? DLM_DEV_BAD_TOKEN_ID : bad == 2 ? DLM_DEV_BAD_LABEL : DLM_DEV_BAD_LAYOUT;
    }
}

// One warp: the slot's answers and label values, the answers' logits
// (loads issued before the label checks that do not need them), then
// dec_slot_compute.
__device__ __forceinline__ void dec_slot_prepare(const DecParams& P, int slot, const uint16_t* x, bool row_ok,
                                                 int lane, DecSlot& S) {
    const DecHead h = dec_slot_head(P, row_ok, P.cand_off[slot], P.cand_off[slot + 1], P.kind[slot]);
    int id[4];
    float v[4];
    uint16_t zb[4];
    #pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int k = lane + 32 * j;
        id[j] = -1; v[j] = 0.f;
        if (!h.bad && k < h.K) {
            id[j] = P.cand_ids[h.o0 + k];
            v[j] = P.val[h.o0 + k];
            S.id[k] = id[j];
        }
    }
    #pragma unroll
    for (int j = 0; j < 4; ++j) zb[j] = (id[j] >= 0 && id[j] < P.vocab) ? x[id[j]] : uint16_t(0);
    __syncwarp();                      // S.id of every lane, for the repeated-id check
    dec_slot_compute(P, h, lane, S, id, v, zb);
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
        if (P.use_full) g += Q * ex2((S.z[k] - lse) * kDecLog2e) - S.q[k];
        S.g[k] = gw * g;
    }
    if (lane == 0) {
        float slot_loss = 0.f;
        if (K > 0) {
            // -sum q_k (z_k - lse); lse is not formed (-inf) when the full CE is off
            const float ce_full = P.use_full ? Q * lse - S.qz : 0.f;
            slot_loss = P.w * (P.use_res * S.ce_res + ce_full + P.brier_w * S.brier);
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
    const bool fold = coef > 0.f;
    const float lb = lse * kDecLog2e - (fold ? log2f(coef) : 0.f);
    const float mul = fold ? 1.f : coef;
    uint16_t* out = P.dlogits + int64_t(slot) * P.ld_out;
    const int c0 = split * P.chunk;
    const int c1 = min(c0 + P.chunk, P.vocab);
    int cv = c0;
    if (P.vec) {
        const int nv = (c1 - c0) / 8;
        const uint4* xv = reinterpret_cast<const uint4*>(x + c0);
        uint4* ov = reinterpret_cast<uint4*>(out + c0);
        const uint64_t ef = policy_evict_first();
        const uint64_t l2e = f2pack(kDecLog2e, kDecLog2e), nlb = f2pack(-lb, -lb);
        int i = tid;
        for (; i + (kDecUnroll - 1) * kDecThreads < nv; i += kDecUnroll * kDecThreads) {
            uint4 rv[kDecUnroll];
            #pragma unroll
            for (int u = 0; u < kDecUnroll; ++u) rv[u] = __ldg(xv + i + u * kDecThreads);
            #pragma unroll
            for (int u = 0; u < kDecUnroll; ++u)
                st_global_v4_hint(ov + i + u * kDecThreads, dec_dense_vec(rv[u], l2e, nlb, fold, mul), ef);
        }
        for (; i < nv; i += kDecThreads) st_global_v4_hint(ov + i, dec_dense_vec(__ldg(xv + i), l2e, nlb, fold, mul), ef);
        cv = c0 + nv * 8;
    }
    for (int c = cv + tid; c < c1; c += kDecThreads) {
        const float g = mul * ex2(fmaf(bf16_bits_to_float(x[c]), kDecLog2e, -lb));
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

// loads in flight per thread: six per batch in the first read (seven
// streaming warps) and four in the second (eight warps) give three and four
// batches per thread for the 31,616-column splits of V = 126,464 -- fewer
// serial memory latencies measured faster than more loads per batch
#ifndef DLM_DEC_CU
#define DLM_DEC_CU 6
#endif
#ifndef DLM_DEC_CU2
#define DLM_DEC_CU2 4
#endif

// Fast path: one thread-block cluster per slot, one CTA per split of the
// row (cluster rank = split; 1, 2, 4 or 8 splits).  Each CTA reads its split
// twice: the first time from HBM, kept in L2 with an evict_last policy (a
// call's label rows are tens of MB), for its (max, sum exp); the cluster
// exchanges only those two floats per warp through distributed shared
// memory and one warp of every CTA merges them into the same lse; the
// second read comes from L2 and writes the gradient, then the answer-token
// entries are rewritten as in k_dec_grad.  Warp 0 is the label warp: it
// reads the slot's answers and works out the label while the other seven
// warps stream the first read (the label's chain of dependent loads and
// warp reductions stays off the critical path); all eight warps stream the
// second.  With the full CE off the first read is skipped (lse is not
// needed) and the dense gradient is zero.  The CTAs hold nothing but a few
// KB of shared memory, so every cluster of a call is resident at once and
// no CTA waits for a second wave (holding each split in shared memory
// instead measured slower: the call's rows do not fit on chip at once).
// The final cluster barrier keeps every CTA's partials alive until all
// peers have read them.  MINB = CTAs resident per SM (the launch bound): 4
// (58 registers) when the call's CTAs fit on the chip at once, 5 (48) when
// they come in waves -- more CTAs streaming while others sit in their
// barriers and tails (1,024 and 2,048 slots: 0.76 -> 0.80, 0.78 -> 0.83 of
// HBM; on 128 slots 5 was 1% slower).
template <int MINB>
__global__ void __launch_bounds__(kDecThreads, MINB) k_dec_cluster(DecParams P) {
    constexpr int kU = DLM_DEC_CU;     // 16-byte loads in flight per thread, first read
    constexpr int kU2 = DLM_DEC_CU2;   // the same, second read
    __shared__ __align__(8) float2 s_part[kDecThreads / 32];   // (max, sum exp) per warp
    __shared__ DecSlot S;
    __shared__ float s_lse;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
    if (warp == 0) {
        // the label warp: the slot's answers and label, while the others stream
        dec_slot_prepare(P, slot, x, row_ok, lane, S);
    } else if (P.use_full) {
        // batches of kU loads in flight per thread, the last one partial
        // (its missing vectors read as -inf, which adds nothing): one
        // memory latency per batch, none for a ragged tail
        constexpr int kStream = kDecThreads - 32;
        const uint4 ninf = make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);
        for (int i = tid - 32; i < nvec; i += kU * kStream) {
            uint4 r[kU];
            #pragma unroll
            for (int u = 0; u < kU; ++u)
                r[u] = i + u * kStream < nvec ? ldg_v4_hint(xv + i + u * kStream, keep) : ninf;
            acc_batch<kU>(r, m, s);
        }
    }
    warp_lse(m, s);
    if (lane == 0) s_part[warp] = make_float2(m, s);
    cluster_sync_all();                // every warp partial of the cluster is written
    if (warp == 0) {
        // lane l merges warp partials l and l + 32 of the cluster (CTA e / 8,
        // warp e % 8), then a butterfly: lse_merge is symmetric, so every
        // lane of every CTA ends with the same bits
        constexpr int kWarps = kDecThreads / 32;
        float M = -INFINITY, Ssum = 0.f;
        for (int e = lane; e < P.n_split * kWarps; e += 32) {
            float pm, ps;
            const uint32_t a = mapa_shared(smem_addr(&s_part[e % kWarps]), uint32_t(e / kWarps));
            asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(pm), "=f"(ps) : "r"(a) : "memory");
            lse_merge(M, Ssum, pm, ps);
        }
        warp_lse(M, Ssum);
        const float lse_w = M + logf(Ssum);
        dec_slot_finish(P, slot, split, lse_w, lane, S);
        if (lane == 0) s_lse = lse_w;
    }
    __syncthreads();
    const float lse = s_lse;
    if (tid == 0) P.err[int64_t(slot) * P.n_split + split] = split == 0 ? S.bad : 0u;
    const float coef = S.coef;
    uint16_t* out = P.dlogits + int64_t(slot) * P.ld_out;
    uint4* ov = reinterpret_cast<uint4*>(out + c0);
    if (coef == 0.f) {
        // restricted-only loss or an invalid slot: zeros, nothing to read
        for (int i = tid; i < nvec; i += kDecThreads) st_global_v4_hint(ov + i, make_uint4(0u, 0u, 0u, 0u), drop);
    } else {
        const bool fold = coef > 0.f;
        const float lb = lse * kDecLog2e - (fold ? log2f(coef) : 0.f);
        const float mul = fold ? 1.f : coef;
        const uint64_t l2e = f2pack(kDecLog2e, kDecLog2e), nlb = f2pack(-lb, -lb);
        for (int i = tid; i < nvec; i += kU2 * kDecThreads) {
            uint4 r[kU2];
            #pragma unroll
            for (int u = 0; u < kU2; ++u)
                if (i + u * kDecThreads < nvec) r[u] = ldg_v4_hint(xv + i + u * kDecThreads, drop);
            #pragma unroll
            for (int u = 0; u < kU2; ++u)
                if (i + u * kDecThreads < nvec)
                    st_global_v4_hint(ov + i + u * kDecThreads, dec_dense_vec(r[u], l2e, nlb, fold, mul), drop);
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
// so nothing needs zeroing between calls).  Warp butterflies and one CTA
// barrier: the kernel sits at the end of the call, so its latency counts.
__global__ void __launch_bounds__(kDecRedThreads) k_dec_reduce(const float* __restrict__ slot_loss, int n,
                                                               float* __restrict__ loss,
                                                               const uint32_t* __restrict__ err, int n_err,
                                                               uint32_t* __restrict__ status) {
    constexpr int kWarps = kDecRedThreads / 32;
    __shared__ double red[kWarps];
    __shared__ uint32_t bits[kWarps];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();                        // slot losses of the gradient kernel
    uint32_t b = 0u;
    if (err)
        for (int i = tid; i < n_err; i += kDecRedThreads) b |= err[i];
    double acc = 0.0;
    for (int i = tid; i < n; i += kDecRedThreads) acc += double(slot_loss[i]);
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    b = __reduce_or_sync(0xffffffffu, b);
    if (lane == 0) { red[warp] = acc; bits[warp] = b; }
    __syncthreads();
    if (tid == 0) {
        double t = 0.0;
        uint32_t bb = 0u;
        #pragma unroll
        for (int w = 0; w < kWarps; ++w) { t += red[w]; bb |= bits[w]; }
        *loss = float(t);
        if (err) *status = bb;
    }
}

struct DecPlan {
    int n_split, chunk;
    size_t partial_off, slot_loss_off, total;
};

// The cluster path: n_split in {1, 2, 4, 8} (a portable cluster size), the
// smallest that both gives about 512 CTAs in all (3.5 per SM, every cluster
// of a small call resident at once) and keeps the rows in flight -- the
// resident CTAs' rows, each read twice -- within an L2 budget, without
// cutting splits under 2,048 columns.  The second read must find its row in
// L2: on 2,048 slots of V = 126,464 at four CTAs per SM, one CTA per row
// (150 MB in flight) ran at 0.66 of HBM, two (75 MB) at 0.78, four (37 MB)
// at 0.80, eight at 0.60 (per-CTA overheads); 50 MB keeps four per row at
// five CTAs per SM too (47 MB).  Needs vocab % 8 == 0 (16-byte vectors).
constexpr int kDecOneWaveCtasPerSm = 4;      // k_dec_cluster<4>: calls whose CTAs fit at once
constexpr int kDecWaveCtasPerSm = 5;         // k_dec_cluster<5>: calls that come in waves
#ifndef DLM_DEC_L2_BUDGET
#define DLM_DEC_L2_BUDGET 50e6
#endif
constexpr double kDecL2RowBudget = DLM_DEC_L2_BUDGET;   // bytes of rows in flight between the two reads
inline bool dec_cluster_plan(int n_slots, int vocab, int sms, int& n_split, int& chunk) {
    if (n_slots <= 0 || vocab % 8 != 0) return false;
    const int64_t want = (512 + n_slots - 1) / n_slots;   // CTAs wanted per slot
    const int64_t resident = int64_t(sms > 0 ? sms : 148) * kDecWaveCtasPerSm;
    auto fits = [&](int ns) {
        const int64_t rows = resident / ns < n_slots ? resident / ns : n_slots;
        return double(rows) * 2.0 * double(vocab) <= kDecL2RowBudget;
    };
    int ns = 1;
    while (ns < 8 && (ns < want || !fits(ns)) && int64_t(vocab) / (2 * ns) >= 2048) ns *= 2;
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
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (n_slots > 0 && P.vec && dec_cluster_plan(n_slots, vocab, sms, cl_split, cl_chunk)) {
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
        const bool one_wave = int64_t(n_slots) * cl_split <= int64_t(sms) * kDecOneWaveCtasPerSm;
        const cudaError_t e = one_wave ? cudaLaunchKernelEx(&cfg, k_dec_cluster<kDecOneWaveCtasPerSm>, C)
                                       : cudaLaunchKernelEx(&cfg, k_dec_cluster<kDecWaveCtasPerSm>, C);
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
