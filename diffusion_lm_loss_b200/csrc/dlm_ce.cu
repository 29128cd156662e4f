// dlm_ce.cu -- inverse-time weighted cross-entropy over the vocabulary,
// forward and backward, from materialised bf16 logits.
//
// The method: "LLaDA-8B-MDLM-LoRA", Training table, row "Objective" (CE on
// masked tokens divided by the mask probability); "Native diffusion
// language-model training", model table (aligned vs shifted logits, uniform
// noise) and Packed training; "diffusiongemma-26B-A4B-it-ALWAYS-THINK",
// Finetuning notes (canvas CE + weight * encoder causal AR CE).
//
// Three launches per call, all on the caller's stream:
//   1. k_plan     one cluster of 8 CTAs: classifies every logits row (scored or not, its
//                 target, unit and weight), counts N, and writes a row list
//                 with the scored rows first; the CE kernel's CTAs take the
//                 list's rows by ticket.
//   2. k_ce_*     the hot kernel, HBM-bound: every scored row must be read
//                 (V*2 bytes) and every row's gradient written (V*2 bytes).
//                 Fast path (k_ce_stream): per SM one or two CTAs of a TMA
//                 producer warp and 24 or 8 consumer warps (chosen so that
//                 the rows in flight fit in L2); each scored row is streamed twice
//                 through a shared-memory ring -- pass 1 from HBM (kept in L2
//                 with an evict_last policy) for the online max / sum of exp,
//                 pass 2 from L2 for the bf16 gradient -- and unscored rows are
//                 zero-filled by bulk shared->global copies from the producer.
//                 A row of 126k-262k bf16 columns (253-524 KB) does not fit in
//                 one SM's shared memory, so it is not held on chip between the
//                 passes; L2 holds it instead.
//                 General path (k_ce_generic): any V / ld / alignment, one CTA
//                 per row, two passes over the row with plain loads.
//   3. k_reduce   one CTA per unit: per-unit sums and the total, fixed order,
//                 double.
#include <mutex>

#include "dlm_device.cuh"
#include "dlm_host.h"

namespace dlm {

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// workspace layout
// ---------------------------------------------------------------------------
struct WsLayout {
    size_t list, row_loss, unit_acc, unit_cnt, total;
};

inline WsLayout ws_layout(int64_t rows, int64_t units) {
    WsLayout w;
    size_t o = kWsAlign;
    w.list = o;      o = align_up(o + size_t(rows) * 16, kWsAlign);
    w.row_loss = o;  o = align_up(o + size_t(rows) * 4, kWsAlign);
    w.unit_acc = o;  o = align_up(o + size_t(units) * 8, kWsAlign);
    w.unit_cnt = o;  o = align_up(o + size_t(units) * 4, kWsAlign);
    w.total = o;
    return w;
}

// ---------------------------------------------------------------------------
// 1. row plan
// ---------------------------------------------------------------------------
struct LayoutDev {
    int n_units;
    int seq_len;
    int64_t n_tokens;
    const int32_t* cu;
    const uint8_t* pad;
};

struct PlanParams {
    LayoutDev a;                 // diffusion rows
    const int32_t* clean_a;
    const uint8_t* corrupted;
    const float* p;
    int mode, align;
    LayoutDev b;                 // encoder rows (n_tokens = 0 when absent)
    const int32_t* ids_b;
    float lam;
    int vocab;
    WsHeader* hdr;
    int4* list;
    // uniform canvas: time weighting, its cap, per-example mean (ObjOpts)
    int time_weighting;
    float weight_clip;
    int example_mean;
    int32_t* unit_cnt;
};

__device__ __forceinline__ void unit_pos(const LayoutDev& L, int64_t i, int& u, int64_t& end) {
    if (L.cu) {
        u = find_unit(L.cu, L.n_units, i);
        end = L.cu[u + 1];
    } else {
        u = int(i) / L.seq_len;   // token indices are < 2^31
        end = int64_t(u + 1) * L.seq_len;
    }
}

// Target of row q (or -1), its unit, and the row's unit's p (absorbing
// weight).  Rows [0, a.n_tokens) are diffusion rows, the rest encoder rows.
// All loads are issued unconditionally (in bounds), so the loads of several
// rows can be in flight together.
__device__ __forceinline__ void classify(const PlanParams& P, int64_t q, int& target, int& unit,
                                         bool& bad_id) {
    target = -1;
    bad_id = false;
    const bool in_a = q < P.a.n_tokens;
    const LayoutDev& L = in_a ? P.a : P.b;
    const int64_t i = in_a ? q : q - P.a.n_tokens;
    int64_t end;
    unit_pos(L, i, unit, end);
    const int64_t j = (in_a && P.align == DLM_ALIGNED) ? i : i + 1;
    const bool inr = j < end && j < L.n_tokens;
    const int64_t jj = inr ? j : 0;
    const bool pad = inr && L.pad && L.pad[jj];
    const bool cor = !(in_a && P.mode == DLM_ABSORBING) || (inr && P.corrupted[jj]);
    const int y = inr ? (in_a ? P.clean_a[jj] : P.ids_b[jj]) : -1;
    if (!inr || pad || !cor) return;
    if (y < 0 || y >= P.vocab) { bad_id = true; return; }
    target = y;
}

// The plan runs as one cluster of kPlanCluster CTAs (one per SM), each
// planning a contiguous slice of the rows: on a single SM the per-row
// instructions alone took ~9 us for 4,096 rows.
constexpr int kPlanCluster = 8;
constexpr int kPlanThreads = 512;
constexpr int kPlanWarps = kPlanThreads / 32;

// cu_seqlens consistency, split over all threads of the cluster
__device__ __forceinline__ bool layout_bad(const LayoutDev& L, int first, int stride) {
    if (!L.cu) return false;
    bool bad = false;
    for (int i = first; i <= L.n_units; i += stride) {
        const int32_t c = L.cu[i];
        if (i == 0 && c != 0) bad = true;
        if (i == L.n_units && int64_t(c) != L.n_tokens) bad = true;
        if (i > 0 && L.cu[i - 1] > c) bad = true;
    }
    return bad;
}

constexpr int kPlanCacheRows = 16384;   // rows per CTA whose classification stays in shared memory

// Exclusive prefix over the warps of the CTA of one count per warp, and the
// CTA total, from s_cnt[warp]; every lane of every warp gets the values for
// its own warp.
__device__ __forceinline__ void warp_prefix(const int* s_cnt, int warp, int lane, int& before, int& total) {
    const int c = lane < kPlanWarps ? s_cnt[lane] : 0;
    int x = c;
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    before = __shfl_sync(0xffffffffu, x - c, warp);
    total = __shfl_sync(0xffffffffu, x, 31);
}

constexpr int kPlanBatch = 4;   // rows per thread whose loads are in flight together

// Classification of the kPlanBatch rows q0, q0 + T, ... of one thread in two
// phases: every address first, then every load (flag, target id, pads, p)
// with nothing waiting on another, then the decisions -- one memory round
// trip for the batch instead of one per row.  Same result as classify().
__device__ __forceinline__ void classify_batch(const PlanParams& P, int64_t q0, int64_t hi, int (&tg)[kPlanBatch],
                                               int (&u)[kPlanBatch], float (&pu)[kPlanBatch], bool& any_bad,
                                               int& na, int& nb, int& nonpad) {
    int64_t jj[kPlanBatch];
    bool ok[kPlanBatch], ina[kPlanBatch], valid[kPlanBatch];
    #pragma unroll
    for (int k = 0; k < kPlanBatch; ++k) {
        const int64_t q = q0 + int64_t(k) * kPlanThreads;
        valid[k] = q < hi;
        ina[k] = q < P.a.n_tokens;
        const LayoutDev& L = ina[k] ? P.a : P.b;
        const int64_t i = !valid[k] ? 0 : (ina[k] ? q : q - P.a.n_tokens);
        int64_t end = 0;
        u[k] = 0;
        if (valid[k]) unit_pos(L, i, u[k], end);
        const int64_t j = (ina[k] && P.align == DLM_ALIGNED) ? i : i + 1;
        ok[k] = valid[k] && j < end && j < L.n_tokens;
        jj[k] = ok[k] ? j : 0;
    }
    const bool absorbing = P.mode == DLM_ABSORBING;
    const bool need_p = absorbing || P.time_weighting != DLM_TIME_WEIGHT_NONE;
    uint8_t cf[kPlanBatch], pd[kPlanBatch], pq[kPlanBatch];
    int y[kPlanBatch];
    #pragma unroll
    for (int k = 0; k < kPlanBatch; ++k) {
        const int64_t q = q0 + int64_t(k) * kPlanThreads;
        const LayoutDev& L = ina[k] ? P.a : P.b;
        const bool need_c = ok[k] && ina[k] && absorbing;
        cf[k] = need_c ? P.corrupted[jj[k]] : uint8_t(1);
        pd[k] = (ok[k] && L.pad) ? L.pad[jj[k]] : uint8_t(0);
        y[k] = ok[k] ? (ina[k] ? P.clean_a[jj[k]] : P.ids_b[jj[k]]) : -1;
        pu[k] = (valid[k] && ina[k] && need_p) ? __ldg(P.p + u[k]) : 0.f;
        pq[k] = (valid[k] && ina[k] && P.a.pad) ? P.a.pad[q] : uint8_t(0);
    }
    #pragma unroll
    for (int k = 0; k < kPlanBatch; ++k) {
        tg[k] = -1;
        if (valid[k] && ina[k]) nonpad += !pq[k];
        if (!ok[k] || pd[k] || !cf[k]) continue;
        if (y[k] < 0 || y[k] >= P.vocab) { any_bad = true; continue; }
        tg[k] = y[k];
        if (ina[k]) ++na; else ++nb;
    }
}

// Load a 32-bit value from the shared memory of another CTA of the cluster.
__device__ __forceinline__ int ld_cluster_s32(uint32_t addr_cluster) {
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr_cluster) : "memory");
    return v;
}

// One cluster; CTA c plans rows [lo, hi) of an even split.  In its slice
// thread t takes rows lo + t, lo + t + T, ... (T = kPlanThreads), so a warp
// always works on 32 consecutive rows: its loads are coalesced, and in pass 2
// its scored rows (and its other rows) land in consecutive list slots, found
// from a warp ballot plus a prefix over the warps -- 16-byte list stores
// that coalesce.  The CTAs exchange their slices' counts through distributed
// shared memory, so each knows N, the totals and where its slice's rows go:
// the list holds the scored rows in row order, then all other rows in row
// order.  Up to kPlanCacheRows rows per CTA, pass 1 keeps each row's
// classification and every warp's counts in shared memory and pass 2 needs
// no global load and no barrier; beyond that, pass 2 classifies again, T rows
// at a time.
__global__ void __launch_bounds__(kPlanThreads, 1) k_plan(PlanParams P) {
    constexpr int kTiles = kPlanCacheRows / kPlanThreads;
    __shared__ int s_cnt[2][kTiles][kPlanWarps];   // per T-row tile and warp: scored / other rows
    __shared__ int s_sum[3][kPlanWarps];
    __shared__ uint32_t s_status;
    __shared__ int s_pub[6];    // this slice: scored, other, scored diffusion, scored encoder, non-pad, status
    __shared__ int s_glob[6];   // scored / other rows of the slices before this one; n_a, n_b, N, status
    pdl_launch_dependents();   // the CE kernel may start its prologue now
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = int(cluster_ctarank()), C = int(cluster_dims_x());
    if (tid == 0) s_status = 0;
    pdl_wait();                // inputs written by earlier kernels are visible
    __syncthreads();
    if (layout_bad(P.a, c * kPlanThreads + tid, C * kPlanThreads) ||
        layout_bad(P.b, c * kPlanThreads + tid, C * kPlanThreads))
        atomicOr(&s_status, DLM_DEV_BAD_LAYOUT);
    if (P.example_mean) {
        // per-unit counts of scored canvas rows, for the per-example mean
        for (int u = c * kPlanThreads + tid; u < P.a.n_units; u += C * kPlanThreads) P.unit_cnt[u] = 0;
        __syncwarp();
        cluster_sync_all();
    }

    const int64_t R = P.a.n_tokens + P.b.n_tokens;
    const int64_t per = ((R + C - 1) / C + 31) / 32 * 32;
    const int64_t lo = min(R, int64_t(c) * per), hi = min(R, lo + per);
    const int64_t Rc = hi - lo;
    const bool cached = Rc <= kPlanCacheRows;
    extern __shared__ int2 s_rows[];   // cached: {target, unit} per row of the slice, then p of the row's unit
    float* s_p = reinterpret_cast<float*>(s_rows + (cached ? Rc : 0));

    // pass 1: classify and count (the bound is the same for every thread:
    // the ballots below need whole warps)
    int na = 0, nb = 0, nonpad = 0;
    bool any_bad = false;
    for (int64_t base = 0; base < Rc; base += int64_t(kPlanThreads) * kPlanBatch) {
        const int64_t q0 = lo + base + tid;
        int tg[kPlanBatch], u[kPlanBatch];
        float pu[kPlanBatch];
        classify_batch(P, q0, hi, tg, u, pu, any_bad, na, nb, nonpad);
        if (P.example_mean) {
            // one atomic per unit per warp (a warp's 32 rows are consecutive)
            #pragma unroll
            for (int k = 0; k < kPlanBatch; ++k) {
                const bool me = tg[k] >= 0 && q0 + int64_t(k) * kPlanThreads < P.a.n_tokens;
                const unsigned act = __ballot_sync(0xffffffffu, me);
                if (me) {
                    const unsigned peers = __match_any_sync(act, u[k]);
                    if (lane == __ffs(peers) - 1) atomicAdd(&P.unit_cnt[u[k]], __popc(peers));
                }
            }
        }
        if (cached) {
            #pragma unroll
            for (int k = 0; k < kPlanBatch; ++k) {
                const int64_t r = base + tid + int64_t(k) * kPlanThreads;   // row within the slice
                const unsigned bs = __ballot_sync(0xffffffffu, r < Rc && tg[k] >= 0);
                const unsigned bv = __ballot_sync(0xffffffffu, r < Rc);
                const int t = int((r - tid) / kPlanThreads);
                if (r - tid < Rc && lane == 0) {
                    s_cnt[0][t][warp] = __popc(bs);
                    s_cnt[1][t][warp] = __popc(bv & ~bs);
                }
                if (r < Rc) {
                    s_rows[r] = make_int2(tg[k], u[k]);
                    s_p[r] = pu[k];
                }
            }
        }
    }
    if (any_bad) atomicOr(&s_status, DLM_DEV_BAD_TOKEN_ID);
    {
        int v0 = na, v1 = nb, v2 = nonpad;
        #pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            v0 += __shfl_xor_sync(0xffffffffu, v0, o);
            v1 += __shfl_xor_sync(0xffffffffu, v1, o);
            v2 += __shfl_xor_sync(0xffffffffu, v2, o);
        }
        if (lane == 0) { s_sum[0][warp] = v0; s_sum[1][warp] = v1; s_sum[2][warp] = v2; }
    }
    __syncthreads();
    if (tid == 0) {
        int la = 0, lb = 0, lnp = 0;
        for (int w = 0; w < kPlanWarps; ++w) { la += s_sum[0][w]; lb += s_sum[1][w]; lnp += s_sum[2][w]; }
        s_pub[0] = la + lb;
        s_pub[1] = int(Rc) - (la + lb);
        s_pub[2] = la;
        s_pub[3] = lb;
        s_pub[4] = lnp;
        s_pub[5] = int(s_status);
    }
    __syncwarp();
    cluster_sync_all();   // every slice's counts are published
    if (warp == 0) {
        int v[6];
        #pragma unroll
        for (int j = 0; j < 6; ++j)
            v[j] = lane < C ? ld_cluster_s32(mapa_shared(smem_addr(&s_pub[j]), uint32_t(lane))) : 0;
        #pragma unroll
        for (int j = 0; j < 5; ++j) {
            // sums over the slices before this CTA's (scored, other) or over all of them
            int x = (j >= 2 || lane < c) ? v[j] : 0;
            #pragma unroll
            for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
            if (lane == 0) s_glob[j] = x;
        }
        int st = v[5];
        #pragma unroll
        for (int o = 16; o > 0; o >>= 1) st |= __shfl_xor_sync(0xffffffffu, st, o);
        if (lane == 0) s_glob[5] = st;
    }
    __syncwarp();
    cluster_sync_all();   // all remote reads are done (no CTA leaves before), s_glob is visible
    const int n_a = s_glob[2], n_b = s_glob[3], N = s_glob[4];
    const int n_scored = n_a + n_b;
    // per-example mean: the number of units with scored canvas rows (the
    // counts are complete: every CTA counted before the barrier above)
    int b_eff = 0;
    if (P.example_mean) {
        int x = 0;
        for (int u = tid; u < P.a.n_units; u += kPlanThreads) x += __ldcg(P.unit_cnt + u) > 0;
        #pragma unroll
        for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        if (lane == 0) s_sum[0][warp] = x;
        __syncthreads();
        for (int w = 0; w < kPlanWarps; ++w) b_eff += s_sum[0][w];
    }
    const float w_canvas = n_a > 0 ? 1.0f / float(n_a) : 0.0f;
    const float w_enc = n_b > 0 ? P.lam / float(n_b) : 0.0f;
    auto weight = [&](int64_t q, int u, float pu) {
        if (q >= P.a.n_tokens) return w_enc;
        if (P.mode == DLM_ABSORBING) return 1.0f / (pu * float(N));
        // uniform canvas: optional 1 / (1 - t) time factor (capped), then the
        // token mean or the mean of per-example means
        float f = 1.0f;
        if (P.time_weighting == DLM_TIME_WEIGHT_INV_ONE_MINUS_T) {
            f = 1.0f / (1.0f - pu);
            if (P.weight_clip > 0.f) f = fminf(f, P.weight_clip);
        }
        // (counts written by this kernel's atomics: an L2 load, not the read-only path)
        if (P.example_mean) return f / (float(b_eff) * float(__ldcg(P.unit_cnt + u)));
        return f * w_canvas;
    };

    // pass 2: weights and this slice's list entries, T rows at a time in row order
    int64_t base_s = s_glob[0], base_u = int64_t(n_scored) + s_glob[1];   // next scored / other slot
    const unsigned below = (1u << lane) - 1u;
    if (cached) {
        for (int t = 0; int64_t(t) * kPlanThreads < Rc; ++t) {
            const int64_t r = int64_t(t) * kPlanThreads + tid;
            const int64_t q = lo + r;
            const bool in = r < Rc;
            const int2 cl = in ? s_rows[r] : make_int2(-1, 0);
            const unsigned bs = __ballot_sync(0xffffffffu, in && cl.x >= 0);
            const unsigned bu = __ballot_sync(0xffffffffu, in && cl.x < 0);
            int ps, ts, pu, tu;
            warp_prefix(s_cnt[0][t], warp, lane, ps, ts);
            warp_prefix(s_cnt[1][t], warp, lane, pu, tu);
            if (in) {
                if (cl.x >= 0)
                    P.list[base_s + ps + __popc(bs & below)] =
                        make_int4(int(q), cl.x, __float_as_int(weight(q, cl.y, s_p[r])), cl.y);
                else
                    P.list[base_u + pu + __popc(bu & below)] = make_int4(int(q), -1, 0, cl.y);
            }
            base_s += ts;
            base_u += tu;
        }
    } else {
        for (int64_t t0 = 0; t0 < Rc; t0 += kPlanThreads) {
            const int64_t q = lo + t0 + tid;
            const bool in = q < hi;
            int tg = -1, u = 0;
            bool bad;
            if (in) classify(P, q, tg, u, bad);
            const unsigned bs = __ballot_sync(0xffffffffu, in && tg >= 0);
            const unsigned bu = __ballot_sync(0xffffffffu, in && tg < 0);
            if (lane == 0) { s_cnt[0][0][warp] = __popc(bs); s_cnt[1][0][warp] = __popc(bu); }
            __syncthreads();
            int ps, ts, pu, tu;
            warp_prefix(s_cnt[0][0], warp, lane, ps, ts);
            warp_prefix(s_cnt[1][0], warp, lane, pu, tu);
            __syncthreads();   // s_cnt is rewritten for the next rows
            if (in) {
                if (tg >= 0) {
                    const bool need_p = P.mode == DLM_ABSORBING || P.time_weighting != DLM_TIME_WEIGHT_NONE;
                    const float pv = (q < P.a.n_tokens && need_p) ? __ldg(P.p + u) : 0.f;
                    P.list[base_s + ps + __popc(bs & below)] = make_int4(int(q), tg, __float_as_int(weight(q, u, pv)), u);
                } else {
                    P.list[base_u + pu + __popc(bu & below)] = make_int4(int(q), -1, 0, u);
                }
            }
            base_s += ts;
            base_u += tu;
        }
    }
    if (c == 0 && tid == 0) {
        P.hdr->status = uint32_t(s_glob[5]);
        P.hdr->n_scored = n_scored;
        P.hdr->n_rows = int(R);
        P.hdr->n_nonpad = N;
        P.hdr->n_scored_a = n_a;
        P.hdr->n_scored_b = n_b;
        P.hdr->ticket = 0u;
        P.hdr->next_s = 0u;
        P.hdr->next_u = 0u;
    }
}

// ---------------------------------------------------------------------------
// 2. CE forward + backward
// ---------------------------------------------------------------------------
struct CeParams {
    const int4* list;
    const WsHeader* hdr;
    uint32_t* status;
    WsHeader* hdr_w;         // the same header, written: the row tickets
    int keep_unscored;       // 1: unscored rows of the gradient are not written
    const uint16_t* xa; uint16_t* da; int64_t lda; int64_t rows_a;
    const uint16_t* xb; uint16_t* db; int64_t ldb;
    int vocab;
    float grad_scale;
    float* row_loss;
};

// (max, sum exp(x - max)) pairs combine associatively; an empty side has
// max = -inf and sum = 0.
__device__ __forceinline__ void lse_combine(float& m, float& s, float m2, float s2) {
    if (m2 == -INFINITY) return;
    if (m == -INFINITY) { m = m2; s = s2; return; }
    const float M = fmaxf(m, m2);
    s = s * ex2((m - M) * kLog2e) + s2 * ex2((m2 - M) * kLog2e);
    m = M;
}

__device__ __forceinline__ void unit_range(const LayoutDev& L, int u, int64_t& lo, int64_t& hi) {
    if (L.n_tokens == 0) { lo = hi = 0; return; }
    if (L.cu) {
        const int64_t a = L.cu[u], b = L.cu[u + 1];
        lo = a < 0 ? 0 : (a > L.n_tokens ? L.n_tokens : a);
        hi = b < lo ? lo : (b > L.n_tokens ? L.n_tokens : b);
    } else {
        lo = int64_t(u) * L.seq_len;
        hi = lo + L.seq_len;
    }
}

__device__ __forceinline__ void row_ptrs(const CeParams& P, int q, const uint16_t*& x, uint16_t*& d) {
    if (q < P.rows_a) {
        x = P.xa + int64_t(q) * P.lda;
        d = P.da + int64_t(q) * P.lda;
    } else {
        const int64_t r = q - P.rows_a;
        x = P.xb + r * P.ldb;
        d = P.db + r * P.ldb;
    }
}

// Fast path.  Each CTA = one TMA producer warp + WARPS consumer warps; it
// takes scored rows of the list by ticket and streams each twice through a
// ring of kStages shared-memory chunks:
//   pass 1: bulk loads from HBM with an L2 evict_last policy; per-thread
//           online (max, sum exp) -> one block combine -> lse of the row;
//   pass 2: the same chunks again (L2 hits), loaded evict_first; the
//           gradient g*w*(exp(x - lse) - [v == y]) goes out as 128-bit
//           stores with an L2 evict_first policy.
// The producer warp also zero-fills unscored rows (taken by ticket too) with
// bulk shared->global copies from a zeroed shared block, interleaved with
// the scored rows so the zero stream overlaps the consumers' work.
#ifndef DLM_CE_RESIDENT
#define DLM_CE_RESIDENT -1          // chunks held in the ring between the passes (-1: stages - 2)
#endif
constexpr int kChunk = 8192;        // bf16 elements per ring stage (16 KB)
constexpr int kZeroBytes = 4096;    // zero block the producer copies over unscored rows

// Two shapes of the kernel, chosen per call from the L2 footprint (every row
// in flight lives in L2 between its two passes, 2V bytes each):
//   StreamShape<8, 6>   2 CTAs/SM x 8 consumer warps, 6-stage ring of 16 KB  (296 rows in flight)
//   StreamShape<24, 8>  1 CTA/SM x 24 consumer warps, 8-stage ring of 24 KB  (148 rows in flight)
template <int WARPS, int STAGES>
struct StreamShape {
    static constexpr int kWarps = WARPS;
    static constexpr int kConsumers = WARPS * 32;
    static constexpr int kThreads = kConsumers + 32;
    static constexpr int kStages = STAGES;
    // bf16 elements per ring stage: 16 KB, or two 16-byte vectors per
    // consumer thread for the wide shapes (24 warps: 24 KB)
    static constexpr int kChunkE = WARPS >= 24 ? WARPS * 512 : kChunk;
    static constexpr int kVec = kChunkE / 8 / kConsumers;   // 16-byte vectors per thread per chunk
    static_assert(kVec * 8 * kConsumers == kChunkE, "chunk split");
    // Chunks of a scored row that stay in the ring between the two passes:
    // the last kResident chunks of pass 1 are not released, pass 2 uses
    // them first, and only the rest of the row is read again (from L2).  Two
    // stages stay free for the producer to run ahead meanwhile.
    static constexpr int kResident = DLM_CE_RESIDENT < 0 ? STAGES - 2
                                   : (DLM_CE_RESIDENT < STAGES ? DLM_CE_RESIDENT : STAGES);
};

constexpr int kRowQ = 16;          // row entries in flight between producer and consumers (> stages / 2)

template <int WARPS, int STAGES>
struct __align__(128) StreamSmem {
    uint4 ring[STAGES][StreamShape<WARPS, STAGES>::kChunkE / 8];
    uint4 zero[kZeroBytes / 16];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    float red_m[2][WARPS];
    float red_s[2][WARPS];
    float xy[2];
    int4 rowq[kRowQ];           // list entries of the rows the producer has started
    int4 cur[2];                // the consumers' current row entry
    int abort;
};

template <int WARPS, int STAGES, int CTAS>
__global__ void __launch_bounds__(StreamShape<WARPS, STAGES>::kThreads, CTAS) k_ce_stream(const CeParams P) {
    using Sh = StreamShape<WARPS, STAGES>;
    constexpr int kConsumerWarps = Sh::kWarps;
    constexpr int kConsumers = Sh::kConsumers;
    constexpr int kStreamThreads = Sh::kThreads;
    constexpr int kStages = Sh::kStages;
    constexpr int kVecPerThread = Sh::kVec;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    StreamSmem<WARPS, STAGES>& S = *reinterpret_cast<StreamSmem<WARPS, STAGES>*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int V = P.vocab;
    constexpr int kChunkE = Sh::kChunkE;
    const int nch = (V + kChunkE - 1) / kChunkE;
    const int res = Sh::kResident < nch ? Sh::kResident : nch;   // chunks kept in the ring between the passes
    volatile int* abort = &S.abort;

    for (int i = tid; i < kZeroBytes / 16; i += kStreamThreads) S.zero[i] = make_uint4(0, 0, 0, 0);
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(smem_addr(&S.full[i]), 1);
            mbar_init(smem_addr(&S.empty[i]), kConsumerWarps);
        }
        S.abort = 0;
        fence_mbar_init_cluster();
    }
    fence_proxy_async_smem();   // zero block visible to the bulk-copy engine
    __syncthreads();
    pdl_wait();                 // the row plan is complete
    pdl_launch_dependents();    // the reduction may start its prologue

    const int n_scored = P.hdr->n_scored;
    const int n_rows = P.hdr->n_rows;

    if (warp == kConsumerWarps) {
        // ------------------------------ producer ------------------------------
        // Rows come from the plan's list through two tickets in the workspace
        // header (scored rows, unscored rows; zeroed by the plan kernel), so a
        // CTA that streams faster simply takes more rows and all CTAs finish
        // together (a fixed deal left the last CTAs finishing ~70 us after the
        // first on a 0.3 ms call, with HBM idling behind them).  Unscored rows are
        // interleaved with the scored ones in the global ratio so the zero
        // stream overlaps the consumers' work.  Each scored row's list entry
        // is published in S.rowq before its first chunk's arrival, and an
        // arrival without data (entry row -1) ends the consumers' loop.
        if (lane == 0) {
            const uint64_t pol_keep = policy_evict_last();
            const uint64_t pol_drop = policy_evict_first();
            const int n_uns = n_rows - n_scored;
            uint32_t* const tick_s = &P.hdr_w->next_s;
            uint32_t* const tick_u = &P.hdr_w->next_u;
            int seq = 0, k = 0, zdone = 0;
            bool zleft = true, ok = true;
            auto zero_next = [&]() {   // zero-fill one more unscored row, if any is left
                const int j = int(atomicAdd(tick_u, 1u));
                if (j >= n_uns) { zleft = false; return; }
                const int q = P.list[n_scored + j].x;
                if (!P.keep_unscored) {
                    const uint16_t* xr;
                    uint16_t* dr;
                    row_ptrs(P, q, xr, dr);
                    const uint32_t bytes = uint32_t(V) * 2u;
                    for (uint32_t off = 0; off < bytes; off += kZeroBytes) {
                        const uint32_t n = bytes - off < uint32_t(kZeroBytes) ? bytes - off : uint32_t(kZeroBytes);
                        bulk_s2g_hint(reinterpret_cast<uint8_t*>(dr) + off, smem_addr(S.zero), n, pol_drop);
                    }
                    bulk_commit_group();
                }
                P.row_loss[q] = 0.f;
                ++zdone;
            };
            int i = int(atomicAdd(tick_s, 1u));
            while (ok && i < n_scored) {
                const int4 e = P.list[i];
                i = int(atomicAdd(tick_s, 1u));   // the next row's ticket, in flight meanwhile
                S.rowq[k % kRowQ] = e;
                const uint16_t* xr;
                uint16_t* dr;
                row_ptrs(P, e.x, xr, dr);
                for (int pass = 0; pass < 2 && ok; ++pass) {
                    // pass 2 reads again only the chunks the ring did not keep
                    const int nc = pass == 0 ? nch : nch - res;
                    for (int c = 0; c < nc; ++c, ++seq) {
                        const int st = seq % kStages;
                        if (!mbar_wait_or_abort(smem_addr(&S.empty[st]), ((seq / kStages) & 1) ^ 1, P.status,
                                                abort)) { ok = false; break; }
                        const int e0 = c * kChunkE;
                        const uint32_t bytes = uint32_t(min(kChunkE, V - e0)) * 2u;
                        const uint32_t fb = smem_addr(&S.full[st]);
                        mbar_arrive_expect_tx(fb, bytes);
                        // only the chunks read again need to stay in L2
                        const bool again = pass == 0 && c < nch - res;
                        bulk_g2s_hint(smem_addr(S.ring[st]), xr + e0, bytes, fb, again ? pol_keep : pol_drop);
                    }
                }
                ++k;
                const int64_t want = int64_t(k) * n_uns / n_scored;
                while (ok && zleft && zdone < want) zero_next();
            }
            while (ok && zleft) zero_next();
            if (ok) {
                // end marker: the next stage arrives without data
                const int st = seq % kStages;
                if (mbar_wait_or_abort(smem_addr(&S.empty[st]), ((seq / kStages) & 1) ^ 1, P.status, abort)) {
                    S.rowq[k % kRowQ] = make_int4(-1, -1, 0, 0);
                    mbar_arrive(smem_addr(&S.full[st]));
                } else {
                    ok = false;
                }
            }
            if (!ok) {
                // let the copies already issued land before this thread leaves
                for (int j = seq - 1; j >= 0 && j >= seq - kStages; --j)
                    mbar_wait_bounded<false>(smem_addr(&S.full[j % kStages]), (j / kStages) & 1, nullptr);
            }
            bulk_wait_group_read<0>();   // shared zero block no longer read
        }
    } else {
    // ------------------------------ consumers ------------------------------
    const uint64_t pol_drop = policy_evict_first();
    int seq = 0;
    for (int k = 0;; ++k) {
        // The first chunk of the next row; its arrival also publishes the
        // row's entry.  Thread 0 reads it (or decides to stop after an abort)
        // and hands it to every consumer warp, so all of them leave the loop
        // together and every barrier below is met by all.
        mbar_wait_or_abort(smem_addr(&S.full[seq % kStages]), (seq / kStages) & 1, P.status, abort);
        if (tid == 0) {
            int4 e0 = S.rowq[k % kRowQ];
            if (*abort) e0.x = -1;
            S.cur[k & 1] = e0;
        }
        named_barrier_sync(2, kConsumers);
        const int4 e = S.cur[k & 1];
        if (e.x < 0) break;
        const int seq0 = seq;            // ring sequence number of the row's first chunk
        const int q = e.x, y = e.y;
        const float w = __int_as_float(e.z);
        const int par = k & 1;
        const uint16_t* xr;
        uint16_t* dr;
        row_ptrs(P, q, xr, dr);

        // pass 1: online (max, sum exp).  After an abort (a bounded wait gave
        // up somewhere in the CTA) the waits return at once and the loops run
        // on with garbage, so every consumer still meets every barrier.
        float m = -INFINITY, s = 0.f;
        for (int c = 0; c < nch; ++c, ++seq) {
            const int st = seq % kStages;
            if (c > 0) mbar_wait_or_abort(smem_addr(&S.full[st]), (seq / kStages) & 1, P.status, abort);
            const int e0 = c * kChunkE;
            uint4 raw[kVecPerThread];
            float cm = -INFINITY;
            #pragma unroll
            for (int j = 0; j < kVecPerThread; ++j) {
                const int vi = tid + j * kConsumers;
                const int col = e0 + vi * 8;
                if (col < V) {
                    raw[j] = S.ring[st][vi];
                    cm = fmaxf(cm, bf16x8_max(raw[j]));
                    const unsigned dy = unsigned(y - col);
                    if (dy < 8u) {
                        const uint32_t wv = dy < 2u ? raw[j].x : dy < 4u ? raw[j].y : dy < 6u ? raw[j].z : raw[j].w;
                        S.xy[par] = (dy & 1u) ? bf16hi(wv) : bf16lo(wv);
                    }
                } else {
                    raw[j] = make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);   // bf16 -inf
                }
            }
            __syncwarp();
            // the row's last `res` chunks stay in the ring for pass 2
            if (lane == 0 && c < nch - res) mbar_arrive(smem_addr(&S.empty[st]));
            if (cm > m) {
                s = (m == -INFINITY) ? 0.f : s * ex2((m - cm) * kLog2e);
                m = cm;
            }
            if (m != -INFINITY) {
                // exp(x - m) for both halves of each bf16 pair: one packed FMA,
                // two ex2, one packed add into the (even, odd) partial sums
                const uint64_t l2e = f2pack(kLog2e, kLog2e);
                const uint64_t nmb = f2pack(-m * kLog2e, -m * kLog2e);
                uint64_t acc = f2pack(0.f, 0.f);
                #pragma unroll
                for (int j = 0; j < kVecPerThread; ++j) {
                    const uint32_t wv[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
                    #pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        float t0, t1;
                        f2unpack(f2fma(f2pack(bf16lo(wv[h]), bf16hi(wv[h])), l2e, nmb), t0, t1);
                        acc = f2add(acc, f2pack(ex2(t0), ex2(t1)));
                    }
                }
                float a0, a1;
                f2unpack(acc, a0, a1);
                s += a0 + a1;
            }
        }
        // block combine among the consumer warps
        #pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
            lse_combine(m, s, m2, s2);
        }
        if (lane == 0) { S.red_m[par][warp] = m; S.red_s[par][warp] = s; }
        named_barrier_sync(1, kConsumers);
        float M = S.red_m[par][0], Ssum = S.red_s[par][0];
        #pragma unroll
        for (int i = 1; i < kConsumerWarps; ++i) lse_combine(M, Ssum, S.red_m[par][i], S.red_s[par][i]);
        const float lse = M + logf(Ssum);
        const float coef = P.grad_scale * w;
        // g = coef * 2^(x log2e - lse log2e); for coef > 0 the factor folds
        // into the exponent (one FFMA + one exp2 per element)
        const bool fold = coef > 0.f;
        const float lb = lse * kLog2e - (fold ? log2f(coef) : 0.f);
        const float mul = fold ? 1.f : coef;
        const uint64_t l2e = f2pack(kLog2e, kLog2e);
        const uint64_t nlb = f2pack(-lb, -lb);

        // pass 2: gradient -- first the chunks still in the ring (the row's
        // tail, no wait), then the head, delivered again by the producer
        for (int i = 0; i < nch; ++i) {
            const bool kept = i < res;
            const int c = kept ? nch - res + i : i - res;
            int st;
            if (kept) {
                st = (seq0 + c) % kStages;
            } else {
                st = seq % kStages;
                mbar_wait_or_abort(smem_addr(&S.full[st]), (seq / kStages) & 1, P.status, abort);
                ++seq;
            }
            const int e0 = c * kChunkE;
            uint4 outv[kVecPerThread];
            #pragma unroll
            for (int j = 0; j < kVecPerThread; ++j) {
                const int vi = tid + j * kConsumers;
                const int col = e0 + vi * 8;
                if (col < V) {
                    const uint4 r = S.ring[st][vi];
                    const uint32_t wv[4] = {r.x, r.y, r.z, r.w};
                    float g[8];
                    #pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        float t0, t1;
                        f2unpack(f2fma(f2pack(bf16lo(wv[h]), bf16hi(wv[h])), l2e, nlb), t0, t1);
                        g[2 * h] = ex2(t0);
                        g[2 * h + 1] = ex2(t1);
                    }
                    if (!fold) {
                        #pragma unroll
                        for (int h = 0; h < 8; ++h) g[h] *= mul;
                    }
                    const unsigned dy = unsigned(y - col);
                    if (dy < 8u) {
                        #pragma unroll
                        for (int h = 0; h < 8; ++h)
                            if (dy == unsigned(h)) g[h] -= coef;
                    }
                    outv[j] = make_uint4(pack_bf16x2(g[0], g[1]), pack_bf16x2(g[2], g[3]),
                                         pack_bf16x2(g[4], g[5]), pack_bf16x2(g[6], g[7]));
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&S.empty[st]));
            #pragma unroll
            for (int j = 0; j < kVecPerThread; ++j) {
                const int col = e0 + (tid + j * kConsumers) * 8;
                if (col < V) st_global_v4_hint(dr + col, outv[j], pol_drop);
            }
        }
        if (tid == 0) P.row_loss[q] = w * (lse - S.xy[par]);
    }
    }   // consumers

}

// General path: one CTA per row (grid-stride), any vocab / stride / alignment.
constexpr int kGenThreads = 256;

__global__ void __launch_bounds__(kGenThreads) k_ce_generic(const CeParams P) {
    __shared__ float red_m[kGenThreads / 32], red_s[kGenThreads / 32];
    __shared__ float s_lse;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();
    pdl_launch_dependents();
    const int n_rows = P.hdr->n_rows;
    const int V = P.vocab;
    for (int i = blockIdx.x; i < n_rows; i += gridDim.x) {
        const int4 e = P.list[i];
        const int q = e.x, y = e.y;
        const float w = __int_as_float(e.z);
        const uint16_t* x;
        uint16_t* d;
        row_ptrs(P, q, x, d);
        if (y < 0) {
            if (!P.keep_unscored)
                for (int v = tid; v < V; v += kGenThreads) d[v] = 0;
            if (tid == 0) P.row_loss[q] = 0.f;
            continue;
        }
        float m = -INFINITY, s = 0.f;
        for (int v = tid; v < V; v += kGenThreads) {
            const float xv = bf16_bits_to_float(x[v]);
            if (xv > m) { s = s * ex2((m - xv) * kLog2e) + 1.f; m = xv; }
            else        { s += ex2((xv - m) * kLog2e); }
        }
        #pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
            lse_combine(m, s, m2, s2);
        }
        if (lane == 0) { red_m[warp] = m; red_s[warp] = s; }
        __syncthreads();
        if (tid == 0) {
            float bm = red_m[0], bs = red_s[0];
            for (int j = 1; j < kGenThreads / 32; ++j) lse_combine(bm, bs, red_m[j], red_s[j]);
            const float lse = bm + logf(bs);
            s_lse = lse;
            P.row_loss[q] = w * (lse - bf16_bits_to_float(x[y]));
        }
        __syncthreads();
        const float lse = s_lse;
        const float coef = P.grad_scale * w;
        for (int v = tid; v < V; v += kGenThreads) {
            const float xv = bf16_bits_to_float(x[v]);
            float g = coef * ex2((xv - lse) * kLog2e);
            if (v == y) g -= coef;
            d[v] = __bfloat16_as_ushort(__float2bfloat16_rn(g));
        }
        __syncthreads();   // red_* / s_lse reused by the next row
    }
}

// ---------------------------------------------------------------------------
// 3. per-unit sums and total (fixed order, double accumulation)
// ---------------------------------------------------------------------------
struct ReduceParams {
    LayoutDev a, b;
    const float* row_loss;   // [a.n_tokens + b.n_tokens]
    double* unit_acc;        // [n_units]
    float* unit_loss;        // may be null
    float* loss;
    unsigned int* ticket;    // zero on entry (the plan kernel clears it); left zero
};

constexpr int kRedThreads = 256;


// Fixed-order block sum of double values (one per thread).
__device__ __forceinline__ double block_sum(double v, double* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double t = 0.0;
    if (warp == 0) {
        t = lane < int(blockDim.x >> 5) ? red[lane] : 0.0;
        #pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    }
    __syncthreads();
    return t;   // valid in warp 0
}

// One CTA per unit (grid-stride for very many units): the unit's rows of both
// terms summed in a fixed order; the CTA that finishes last adds the units up
// in a fixed order.  Bitwise reproducible.
__global__ void __launch_bounds__(kRedThreads) k_reduce(ReduceParams R) {
    __shared__ double red[kRedThreads / 32];
    __shared__ bool last;
    const int tid = threadIdx.x;
    const int U = R.a.n_units;
    pdl_wait();   // row losses of the CE kernel are complete
    for (int u = blockIdx.x; u < U; u += gridDim.x) {
        // four independent accumulators (loads in flight together), combined
        // in a fixed order
        double acc[4] = {0.0, 0.0, 0.0, 0.0};
        int64_t lo, hi;
        unit_range(R.a, u, lo, hi);
        {
            int64_t i = lo + tid;
            for (; i + 3 * kRedThreads < hi; i += 4 * kRedThreads) {
                #pragma unroll
                for (int k = 0; k < 4; ++k) acc[k] += double(R.row_loss[i + k * kRedThreads]);
            }
            for (; i < hi; i += kRedThreads) acc[0] += double(R.row_loss[i]);
        }
        unit_range(R.b, u, lo, hi);
        {
            const float* rb = R.row_loss + R.a.n_tokens;
            int64_t i = lo + tid;
            for (; i + 3 * kRedThreads < hi; i += 4 * kRedThreads) {
                #pragma unroll
                for (int k = 0; k < 4; ++k) acc[k] += double(rb[i + k * kRedThreads]);
            }
            for (; i < hi; i += kRedThreads) acc[0] += double(rb[i]);
        }
        const double t = block_sum((acc[0] + acc[1]) + (acc[2] + acc[3]), red);
        if (tid == 0) {
            R.unit_acc[u] = t;
            if (R.unit_loss) R.unit_loss[u] = float(t);
        }
    }
    if (gridDim.x == 1) {
        // at most one unit: its sum is the total (no hand-off between CTAs)
        if (tid == 0) R.loss[0] = U > 0 ? float(R.unit_acc[0]) : 0.f;
        return;
    }
    // last CTA: the total
    if (tid == 0) {
        __threadfence();
        last = atomicAdd(R.ticket, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (!last) return;
    __threadfence();
    const int per = (U + kRedThreads - 1) / kRedThreads;
    double acc = 0.0;
    for (int u = tid * per; u < min(U, (tid + 1) * per); ++u) acc += __ldcg(R.unit_acc + u);
    const double t = block_sum(acc, red);
    if (tid == 0) {
        R.loss[0] = float(t);
        *R.ticket = 0u;
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// Shared-memory attribute of a streaming-kernel shape, set once per device.
template <int WARPS, int STAGES, int CTAS>
static bool stream_kernel_ready(int dev) {
    static std::mutex mu;
    static int state[64];   // 0 unknown, 1 ok, 2 failed
    if (dev < 0 || dev >= 64) return false;
    std::lock_guard<std::mutex> g(mu);
    if (state[dev] == 0) {
        const cudaError_t e = cudaFuncSetAttribute(k_ce_stream<WARPS, STAGES, CTAS>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   int(sizeof(StreamSmem<WARPS, STAGES>)));
        if (e != cudaSuccess) cudaGetLastError();
        state[dev] = e == cudaSuccess ? 1 : 2;
    }
    return state[dev] == 1;
}

// Launch the streaming kernel of the given shape: CTAS CTAs per SM.
template <int WARPS, int STAGES, int CTAS>
static dlm_status_t launch_stream(const CeParams& cp, int64_t R, int sms, int dev, cudaStream_t s, bool& done) {
    done = false;
    if (!stream_kernel_ready<WARPS, STAGES, CTAS>(dev)) return DLM_OK;
    const int64_t grid = R < int64_t(sms) * CTAS ? R : int64_t(sms) * CTAS;
    done = true;
    return launch_pdl(k_ce_stream<WARPS, STAGES, CTAS>, dim3(unsigned(grid)), dim3(StreamShape<WARPS, STAGES>::kThreads),
                      sizeof(StreamSmem<WARPS, STAGES>), s, "k_ce_stream launch", cp);
}

// Rows in flight x 2V bytes must stay within this much L2 between the passes.
constexpr double kL2RowBudget = 80e6;

static LayoutDev to_dev(const dlm_layout_t* L) {
    LayoutDev d{};
    if (!L) return d;
    d.n_units = L->n_units;
    d.seq_len = L->seq_len;
    d.n_tokens = L->n_tokens;
    d.cu = L->cu_seqlens;
    d.pad = L->pad_mask;
    return d;
}

dlm_status_t launch_plan(const dlm_layout_t* a, const int32_t* clean, const uint8_t* corrupted,
                         const float* p, int mode, int align, const dlm_layout_t* b,
                         const int32_t* ids_b, float lam, int vocab, WsHeader* hdr, int4* list,
                         cudaStream_t s, const ObjOpts& opts) {
    PlanParams pp{};
    pp.time_weighting = opts.time_weighting;
    pp.weight_clip = opts.weight_clip;
    pp.example_mean = opts.reduction == DLM_REDUCE_EXAMPLE_MEAN ? 1 : 0;
    pp.unit_cnt = opts.unit_cnt;
    pp.a = to_dev(a);
    pp.clean_a = clean;
    pp.corrupted = corrupted;
    pp.p = p;
    pp.mode = mode;
    pp.align = align;
    pp.b = to_dev(b);
    pp.ids_b = ids_b;
    pp.lam = lam;
    pp.vocab = vocab;
    pp.hdr = hdr;
    pp.list = list;
    const int64_t R = (a ? a->n_tokens : 0) + (b ? b->n_tokens : 0);
    const int64_t per = ((R + kPlanCluster - 1) / kPlanCluster + 31) / 32 * 32;   // rows per CTA (as the kernel splits)
    const size_t smem = per <= kPlanCacheRows ? size_t(per) * (sizeof(int2) + sizeof(float)) : 0;
    static std::mutex mu;
    static bool attr[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    {
        std::lock_guard<std::mutex> g(mu);
        if (dev >= 0 && dev < 64 && !attr[dev]) {
            cudaError_t e = cudaFuncSetAttribute(k_plan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 int(kPlanCacheRows * (sizeof(int2) + sizeof(float))));
            if (e != cudaSuccess) return cuda_status(e, "k_plan smem attribute");
            attr[dev] = true;
        }
    }
    // one cluster of kPlanCluster CTAs, launched with programmatic stream
    // serialization like the other kernels of the call
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kPlanCluster);
    cfg.blockDim = dim3(kPlanThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = kPlanCluster;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, k_plan, pp);
    if (e != cudaSuccess) cudaGetLastError();
    return cuda_status(e, "k_plan launch");
}

dlm_status_t launch_reduce(const dlm_layout_t* a, const dlm_layout_t* b, const float* row_loss,
                           double* unit_acc, float* unit_loss, float* loss, WsHeader* hdr,
                           cudaStream_t s) {
    ReduceParams rp{};
    rp.a = to_dev(a);
    rp.b = to_dev(b);
    rp.row_loss = row_loss;
    rp.unit_acc = unit_acc;
    rp.unit_loss = unit_loss;
    rp.loss = loss;
    rp.ticket = &hdr->ticket;
    const int U = a->n_units;
    const int rgrid = U < 1 ? 1 : (U > 65536 ? 65536 : U);
    return launch_pdl(k_reduce, dim3(rgrid), dim3(kRedThreads), 0, s, "k_reduce launch", rp);
}

}  // namespace dlm

using namespace dlm;

extern "C" size_t dlm_loss_workspace_size(const dlm_layout_t* layout, const dlm_layout_t* enc_layout) {
    if (!layout) return 0;
    const int64_t rows = layout->n_tokens + (enc_layout ? enc_layout->n_tokens : 0);
    return ws_layout(rows, layout->n_units).total;
}

static dlm_status_t loss_fwd_bwd(const dlm_layout_t* layout, const uint16_t* logits, int64_t ld,
                                 int32_t vocab, const int32_t* clean_ids, const uint8_t* corrupted,
                                 const float* p, int32_t mode, int32_t align,
                                 const dlm_layout_t* enc_layout, const uint16_t* enc_logits,
                                 int64_t enc_ld, const int32_t* enc_ids, float enc_ar_weight,
                                 float grad_scale, ObjOpts opts, float* loss, float* unit_loss,
                                 uint16_t* dlogits, uint16_t* enc_dlogits,
                                 void* workspace, size_t workspace_bytes, dlm_stream_t stream) {
    // ---- host-side argument checks (nothing is enqueued on failure) ----
    if (!layout_ok(layout)) return DLM_ERR_INVALID_ARGUMENT;
    if (mode != DLM_ABSORBING && mode != DLM_UNIFORM) return DLM_ERR_INVALID_ARGUMENT;
    if (align != DLM_ALIGNED && align != DLM_SHIFTED) return DLM_ERR_INVALID_ARGUMENT;
    if (vocab <= 0 || ld < vocab) return DLM_ERR_INVALID_ARGUMENT;
    if (!loss || !workspace) return DLM_ERR_INVALID_ARGUMENT;
    const bool has_enc = enc_logits != nullptr;
    if (has_enc) {
        if (mode != DLM_UNIFORM) return DLM_ERR_INVALID_ARGUMENT;
        if (!layout_ok(enc_layout) || enc_layout->n_units != layout->n_units) return DLM_ERR_INVALID_ARGUMENT;
        if (enc_ld < vocab || !enc_ids || !enc_dlogits) return DLM_ERR_INVALID_ARGUMENT;
        if (!enc_layout->cu_seqlens && enc_layout->seq_len == 0 && enc_layout->n_tokens > 0)
            return DLM_ERR_INVALID_ARGUMENT;
    }
    const int64_t rows_a = layout->n_tokens;
    const int64_t rows_b = has_enc ? enc_layout->n_tokens : 0;
    const int64_t R = rows_a + rows_b;
    if (R >= (int64_t(1) << 31)) return DLM_ERR_INVALID_ARGUMENT;
    if (rows_a > 0 && (!logits || !dlogits || !clean_ids)) return DLM_ERR_INVALID_ARGUMENT;
    if (rows_a > 0 && mode == DLM_ABSORBING && (!corrupted || !p)) return DLM_ERR_INVALID_ARGUMENT;
    if (opts.time_weighting != DLM_TIME_WEIGHT_NONE && rows_a > 0 && !p) return DLM_ERR_INVALID_ARGUMENT;
    if (rows_a > 0 && !layout->cu_seqlens && layout->seq_len == 0) return DLM_ERR_INVALID_ARGUMENT;
    if (reinterpret_cast<uintptr_t>(workspace) % kWsAlign) return DLM_ERR_INVALID_ARGUMENT;
    const dlm_layout_t* lb = has_enc ? enc_layout : nullptr;
    const WsLayout W = ws_layout(R, layout->n_units);
    if (workspace_bytes < W.total) return DLM_ERR_WORKSPACE_TOO_SMALL;
    dlm_status_t st = check_device();
    if (st != DLM_OK) return st;

    cudaStream_t s = (cudaStream_t)stream;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    int4* list = reinterpret_cast<int4*>(ws + W.list);
    float* row_loss = reinterpret_cast<float*>(ws + W.row_loss);
    double* unit_acc = reinterpret_cast<double*>(ws + W.unit_acc);
    opts.unit_cnt = reinterpret_cast<int32_t*>(ws + W.unit_cnt);

    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);

    // kernel choice: the streaming kernel when the rows are 16-byte streamable,
    // one or two CTAs per SM so that the rows in flight fit in L2
    bool fast = R > 0 && (vocab % 8 == 0) && (ld % 8 == 0) && vocab >= 4096 &&
                (rows_a == 0 || (aligned16(logits) && aligned16(dlogits)));
    if (has_enc) fast = fast && (enc_ld % 8 == 0) && aligned16(enc_logits) && aligned16(enc_dlogits);
    const bool two_per_sm = double(sms) * 2.0 * 2.0 * double(vocab) <= kL2RowBudget;
    // one CTA per SM: 24 consumer warps, 24 KB chunks, 8 stages (measured
    // against 16 warps with 16 KB chunks and 12 stages: 3-5% faster on the
    // V = 152k-262k workloads, where the consumers are latency-bound; 28
    // warps with 28 KB chunks and 7 stages: 1-2% slower again)
#ifndef DLM_CE_WIDE_WARPS
#define DLM_CE_WIDE_WARPS 24
#endif
#if DLM_CE_WIDE_WARPS == 24
#define DLM_CE_WIDE 24, 8, 1
#else
#define DLM_CE_WIDE 16, 12, 1
#endif
    if (fast) fast = two_per_sm ? stream_kernel_ready<8, 6, 2>(dev) : stream_kernel_ready<DLM_CE_WIDE>(dev);

    // ---- 1. plan ----
    if ((st = launch_plan(layout, clean_ids, corrupted, p, mode, align, lb, enc_ids, enc_ar_weight, vocab,
                          hdr, list, s, opts)) != DLM_OK)
        return st;

    // ---- 2. CE ----
    if (R > 0) {
        CeParams cp{};
        cp.list = list;
        cp.hdr = hdr;
        cp.status = &hdr->status;
        cp.xa = logits; cp.da = dlogits; cp.lda = ld; cp.rows_a = rows_a;
        cp.xb = enc_logits; cp.db = enc_dlogits; cp.ldb = enc_ld;
        cp.vocab = vocab;
        cp.grad_scale = grad_scale;
        cp.row_loss = row_loss;
        cp.hdr_w = hdr;
        cp.keep_unscored = opts.keep_unscored_rows;

        bool launched = false;
        if (fast) {
            st = two_per_sm ? launch_stream<8, 6, 2>(cp, R, sms, dev, s, launched)
                            : launch_stream<DLM_CE_WIDE>(cp, R, sms, dev, s, launched);
            if (st != DLM_OK) return st;
        }
        if (!launched) {
            const int64_t grid = R < int64_t(sms) * 8 ? R : int64_t(sms) * 8;
            if ((st = launch_pdl(k_ce_generic, dim3(unsigned(grid)), dim3(kGenThreads), 0, s,
                                 "k_ce_generic launch", cp)) != DLM_OK)
                return st;
        }
    }

    // ---- 3. reduce ----
    return launch_reduce(layout, lb, row_loss, unit_acc, unit_loss, loss, hdr, s);
}

extern "C" dlm_status_t dlm_loss_fwd_bwd(const dlm_layout_t* layout, const uint16_t* logits, int64_t ld,
                                         int32_t vocab, const int32_t* clean_ids, const uint8_t* corrupted,
                                         const float* p, int32_t mode, int32_t align,
                                         const dlm_layout_t* enc_layout, const uint16_t* enc_logits,
                                         int64_t enc_ld, const int32_t* enc_ids, float enc_ar_weight,
                                         float grad_scale, float* loss, float* unit_loss,
                                         uint16_t* dlogits, uint16_t* enc_dlogits,
                                         void* workspace, size_t workspace_bytes, dlm_stream_t stream) {
    DLM_NVTX("dlm_loss_fwd_bwd");
    return loss_fwd_bwd(layout, logits, ld, vocab, clean_ids, corrupted, p, mode, align, enc_layout, enc_logits,
                        enc_ld, enc_ids, enc_ar_weight, grad_scale, ObjOpts(), loss, unit_loss, dlogits,
                        enc_dlogits, workspace, workspace_bytes, stream);
}

extern "C" dlm_status_t dlm_loss_fwd_bwd_ex(const dlm_layout_t* layout, const uint16_t* logits, int64_t ld,
                                            int32_t vocab, const int32_t* clean_ids, const uint8_t* corrupted,
                                            const float* p, int32_t mode, int32_t align,
                                            const dlm_layout_t* enc_layout, const uint16_t* enc_logits,
                                            int64_t enc_ld, const int32_t* enc_ids, float enc_ar_weight,
                                            float grad_scale, const dlm_loss_options_t* options, float* loss,
                                            float* unit_loss, uint16_t* dlogits, uint16_t* enc_dlogits,
                                            void* workspace, size_t workspace_bytes, dlm_stream_t stream) {
    DLM_NVTX("dlm_loss_fwd_bwd_ex");
    ObjOpts o;
    if (options) {
        // 16 bytes: the struct before keep_unscored_rows was added
        if (options->struct_size < 16) return DLM_ERR_INVALID_ARGUMENT;
        if (options->time_weighting != DLM_TIME_WEIGHT_NONE &&
            options->time_weighting != DLM_TIME_WEIGHT_INV_ONE_MINUS_T)
            return DLM_ERR_INVALID_ARGUMENT;
        if (options->reduction != DLM_REDUCE_TOKEN_MEAN && options->reduction != DLM_REDUCE_EXAMPLE_MEAN)
            return DLM_ERR_INVALID_ARGUMENT;
        if (!(options->weight_clip == options->weight_clip)) return DLM_ERR_INVALID_ARGUMENT;   // NaN
        const bool non_default = options->time_weighting != DLM_TIME_WEIGHT_NONE ||
                                 options->reduction != DLM_REDUCE_TOKEN_MEAN;
        if (non_default && mode != DLM_UNIFORM) return DLM_ERR_INVALID_ARGUMENT;
        o.time_weighting = options->time_weighting;
        o.weight_clip = options->weight_clip;
        o.reduction = options->reduction;
        if (options->struct_size >= offsetof(dlm_loss_options_t, keep_unscored_rows) + sizeof(int32_t)) {
            if (options->keep_unscored_rows != 0 && options->keep_unscored_rows != 1)
                return DLM_ERR_INVALID_ARGUMENT;
            o.keep_unscored_rows = options->keep_unscored_rows;
        }
    }
    return loss_fwd_bwd(layout, logits, ld, vocab, clean_ids, corrupted, p, mode, align, enc_layout, enc_logits,
                        enc_ld, enc_ids, enc_ar_weight, grad_scale, o, loss, unit_loss, dlogits, enc_dlogits,
                        workspace, workspace_bytes, stream);
}
