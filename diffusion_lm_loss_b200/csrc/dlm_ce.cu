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
//   1. k_plan     one CTA: classifies every logits row (scored or not, its
//                 target, unit and weight), counts N, and writes a row list
//                 with the scored rows first -- so the CE kernel can deal the
//                 expensive rows out evenly.
//   2. k_ce_*     the hot kernel.  HBM-bound: each scored row is read once
//                 (V*2 bytes) and each row's gradient written once (V*2 bytes).
//                 Fast path (k_ce_cluster): a cluster of K CTAs owns one row at
//                 a time, CTA j holding columns [j*S, (j+1)*S) -- the row does
//                 not fit one SM's shared memory for V >= ~110k, so it is split
//                 across the cluster.  Each CTA streams its slice with a bulk
//                 async copy (TMA engine, no multicast) into a ring of shared
//                 buffers, pulls it into registers, computes its (max, sum of
//                 exp) pair, exchanges the pair with the other K-1 CTAs through
//                 distributed shared memory (st.async + mbarrier), and writes
//                 grad = g*w*(softmax - onehot) as bf16 with 128-bit streaming
//                 stores.  Unscored rows are zero-filled with the same stores.
//                 General path (k_ce_generic): any V / ld / alignment, one CTA
//                 per row, two passes over the row (the second hits L2).
//   3. k_reduce   one CTA: per-unit sums and the total, fixed order, double.
#include <mutex>

#include "dlm_device.cuh"
#include "dlm_host.h"

namespace dlm {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------------------
// workspace layout
// ---------------------------------------------------------------------------
struct WsHeader {
    uint32_t status;
    int32_t n_scored;     // scored rows, both terms
    int32_t n_rows;       // rows, both terms
    int32_t n_nonpad;     // N of the diffusion layout
    int32_t n_scored_a;   // scored diffusion rows
    int32_t n_scored_b;   // scored encoder rows
};
static_assert(sizeof(WsHeader) <= kWsAlign, "header");

struct WsLayout {
    size_t list, row_loss, unit_acc, total;
};

inline WsLayout ws_layout(int64_t rows, int64_t units) {
    WsLayout w;
    size_t o = kWsAlign;
    w.list = o;      o = align_up(o + size_t(rows) * 16, kWsAlign);
    w.row_loss = o;  o = align_up(o + size_t(rows) * 4, kWsAlign);
    w.unit_acc = o;  o = align_up(o + size_t(units) * 8, kWsAlign);
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
};

__device__ __forceinline__ void unit_pos(const LayoutDev& L, int64_t i, int& u, int64_t& end) {
    if (L.cu) {
        u = find_unit(L.cu, L.n_units, i);
        end = L.cu[u + 1];
    } else {
        u = int(i / L.seq_len);
        end = int64_t(u + 1) * L.seq_len;
    }
}

// Target of row q (or -1) and its unit.  Rows [0, a.n_tokens) are diffusion
// rows, the rest encoder rows.
__device__ __forceinline__ void classify(const PlanParams& P, int64_t q, int& target, int& unit,
                                         bool& bad_id) {
    target = -1;
    bad_id = false;
    if (q < P.a.n_tokens) {
        int64_t end;
        unit_pos(P.a, q, unit, end);
        int64_t j = P.align == DLM_ALIGNED ? q : q + 1;
        if (j >= end || j >= P.a.n_tokens) return;
        if (P.a.pad && P.a.pad[j]) return;
        if (P.mode == DLM_ABSORBING && !P.corrupted[j]) return;
        int y = P.clean_a[j];
        if (y < 0 || y >= P.vocab) { bad_id = true; return; }
        target = y;
    } else {
        const int64_t i = q - P.a.n_tokens;
        int64_t end;
        unit_pos(P.b, i, unit, end);
        const int64_t j = i + 1;
        if (j >= end || j >= P.b.n_tokens) return;
        if (P.b.pad && P.b.pad[j]) return;
        int y = P.ids_b[j];
        if (y < 0 || y >= P.vocab) { bad_id = true; return; }
        target = y;
    }
}

constexpr int kPlanThreads = 1024;

__device__ __forceinline__ bool layout_bad(const LayoutDev& L) {
    // every thread checks a strided part of cu_seqlens
    if (!L.cu) return false;
    bool bad = false;
    for (int i = threadIdx.x; i <= L.n_units; i += blockDim.x) {
        const int32_t c = L.cu[i];
        if (i == 0 && c != 0) bad = true;
        if (i == L.n_units && int64_t(c) != L.n_tokens) bad = true;
        if (i > 0 && L.cu[i - 1] > c) bad = true;
    }
    return bad;
}

__global__ void __launch_bounds__(kPlanThreads) k_plan(PlanParams P) {
    __shared__ int s_cnt[kPlanThreads];
    __shared__ int s_red[4][32];
    __shared__ int s_tot[4];
    __shared__ uint32_t s_status;
    const int tid = threadIdx.x;
    if (tid == 0) s_status = 0;
    __syncthreads();
    if (layout_bad(P.a) || layout_bad(P.b)) atomicOr(&s_status, DLM_DEV_BAD_LAYOUT);

    const int64_t R = P.a.n_tokens + P.b.n_tokens;
    const int64_t chunk = (R + kPlanThreads - 1) / kPlanThreads;
    const int64_t r0 = min(R, int64_t(tid) * chunk), r1 = min(R, r0 + chunk);

    // pass 1: counts
    int na = 0, nb = 0, nonpad = 0;
    bool any_bad = false;
    for (int64_t q = r0; q < r1; ++q) {
        int tg, u;
        bool bad;
        classify(P, q, tg, u, bad);
        any_bad |= bad;
        if (tg >= 0) { if (q < P.a.n_tokens) ++na; else ++nb; }
        if (q < P.a.n_tokens && !(P.a.pad && P.a.pad[q])) ++nonpad;
    }
    if (any_bad) atomicOr(&s_status, DLM_DEV_BAD_TOKEN_ID);
    s_cnt[tid] = na + nb;
    // block sums of na, nb, nonpad
    {
        int v0 = na, v1 = nb, v2 = nonpad;
        for (int o = 16; o > 0; o >>= 1) {
            v0 += __shfl_xor_sync(0xffffffffu, v0, o);
            v1 += __shfl_xor_sync(0xffffffffu, v1, o);
            v2 += __shfl_xor_sync(0xffffffffu, v2, o);
        }
        if ((tid & 31) == 0) { s_red[0][tid >> 5] = v0; s_red[1][tid >> 5] = v1; s_red[2][tid >> 5] = v2; }
    }
    __syncthreads();
    if (tid < 32) {
        int v0 = s_red[0][tid], v1 = s_red[1][tid], v2 = s_red[2][tid];
        for (int o = 16; o > 0; o >>= 1) {
            v0 += __shfl_xor_sync(0xffffffffu, v0, o);
            v1 += __shfl_xor_sync(0xffffffffu, v1, o);
            v2 += __shfl_xor_sync(0xffffffffu, v2, o);
        }
        if (tid == 0) { s_tot[0] = v0; s_tot[1] = v1; s_tot[2] = v2; }
    }
    // exclusive scan of per-thread scored counts (Hillis-Steele, in place)
    for (int o = 1; o < kPlanThreads; o <<= 1) {
        __syncthreads();
        const int add = tid >= o ? s_cnt[tid - o] : 0;
        __syncthreads();
        s_cnt[tid] += add;
    }
    __syncthreads();
    const int n_a = s_tot[0], n_b = s_tot[1], N = s_tot[2];
    const int n_scored = n_a + n_b;
    const int scored_before = s_cnt[tid] - (na + nb);
    int64_t so = scored_before;                          // next scored slot
    int64_t uo = n_scored + (r0 - scored_before);        // next unscored slot

    const float w_canvas = n_a > 0 ? 1.0f / float(n_a) : 0.0f;
    const float w_enc = n_b > 0 ? P.lam / float(n_b) : 0.0f;

    // pass 2: weights and the row list
    for (int64_t q = r0; q < r1; ++q) {
        int tg, u;
        bool bad;
        classify(P, q, tg, u, bad);
        if (tg >= 0) {
            float w;
            if (q < P.a.n_tokens) {
                w = P.mode == DLM_ABSORBING ? 1.0f / (__ldg(P.p + u) * float(N)) : w_canvas;
            } else {
                w = w_enc;
            }
            P.list[so++] = make_int4(int(q), tg, __float_as_int(w), u);
        } else {
            P.list[uo++] = make_int4(int(q), -1, 0, u);
        }
    }
    __syncthreads();
    if (tid == 0) {
        P.hdr->status = s_status;
        P.hdr->n_scored = n_scored;
        P.hdr->n_rows = int(R);
        P.hdr->n_nonpad = N;
        P.hdr->n_scored_a = n_a;
        P.hdr->n_scored_b = n_b;
    }
}

// ---------------------------------------------------------------------------
// 2. CE forward + backward
// ---------------------------------------------------------------------------
struct CeParams {
    const int4* list;
    const WsHeader* hdr;
    uint32_t* status;
    const uint16_t* xa; uint16_t* da; int64_t lda; int64_t rows_a;
    const uint16_t* xb; uint16_t* db; int64_t ldb;
    int vocab;
    float grad_scale;
    float* row_loss;
    // cluster path
    int slice;       // S: columns per CTA (multiple of 8)
    int nbuf;        // shared-memory ring depth
};

// (max, sum exp(x - max)) pairs combine associatively; an empty side has
// max = -inf and sum = 0.
__device__ __forceinline__ void lse_combine(float& m, float& s, float m2, float s2) {
    if (m2 == -INFINITY) return;
    if (m == -INFINITY) { m = m2; s = s2; return; }
    const float M = fmaxf(m, m2);
    s = s * exp2f((m - M) * kLog2e) + s2 * exp2f((m2 - M) * kLog2e);
    m = M;
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

constexpr int kCeThreads = 512;
constexpr int kCeWarps = kCeThreads / 32;
constexpr int kMaxCluster = 8;
constexpr int kMaxBuf = 4;

struct __align__(16) CeSmemTail {
    uint64_t full[kMaxBuf];
    uint64_t xbar[2];
    float4 xslot[2][kMaxCluster];
    float red_m[kCeWarps];
    float red_s[kCeWarps];
    float xy;
    int abort;
};

template <int CHUNKS>
__global__ void __launch_bounds__(kCeThreads, 1) k_ce_cluster(const CeParams P) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int K = int(cluster_dims_x());
    const int rank = int(cluster_ctarank());
    const int cid = int(cluster_id_x()), C = int(nclusters_x());
    const int S = P.slice;
    const int c0 = rank * S;
    const int c1 = min(P.vocab, c0 + S);
    const int ncols = c1 - c0;                // multiple of 8 on this path
    const int nch = ncols >> 3;
    const int nbuf = P.nbuf;
    CeSmemTail* tail = reinterpret_cast<CeSmemTail*>(smem + size_t(nbuf) * S * 2);
    const uint32_t buf0 = smem_addr(smem);

    if (tid == 0) {
        for (int b = 0; b < nbuf; ++b) mbar_init(smem_addr(&tail->full[b]), 1);
        mbar_init(smem_addr(&tail->xbar[0]), 1);
        mbar_init(smem_addr(&tail->xbar[1]), 1);
        tail->abort = 0;
        fence_mbar_init_cluster();
    }
    // peers' barriers must exist before any remote arrive
    cluster_sync_all();

    const int n_scored = P.hdr->n_scored;
    const int n_rows = P.hdr->n_rows;
    const int my_scored = cid < n_scored ? (n_scored - cid + C - 1) / C : 0;

    auto issue = [&](int k) {
        const int4 e = P.list[cid + k * C];
        const uint16_t* x;
        uint16_t* d;
        row_ptrs(P, e.x, x, d);
        const int b = k % nbuf;
        const uint32_t bar = smem_addr(&tail->full[b]);
        mbar_arrive_expect_tx(bar, uint32_t(ncols) * 2u);
        bulk_g2s(buf0 + uint32_t(b) * uint32_t(S) * 2u, x + c0, uint32_t(ncols) * 2u, bar);
    };

    int issued = 0;      // meaningful in thread 0 only
    int waited = 0;      // full-barrier waits completed
    if (tid == 0) {
        const int pre = min(nbuf, my_scored);
        for (; issued < pre; ++issued) issue(issued);
    }

    int k = 0;
    bool ok = true;
    for (; k < my_scored; ++k) {
        const int4 e = P.list[cid + k * C];
        const int q = e.x, y = e.y;
        const float w = __int_as_float(e.z);
        const int b = k % nbuf;
        if (!mbar_wait_bounded<false>(smem_addr(&tail->full[b]), uint32_t(k / nbuf) & 1u, P.status)) {
            ok = false;
        }
        if (__syncthreads_or(!ok)) { ok = false; break; }
        waited = k + 1;

        // registers <- shared slice
        const uint4* sb = reinterpret_cast<const uint4*>(smem + size_t(b) * S * 2);
        uint4 raw[CHUNKS];
        #pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
            const int ci = tid + c * kCeThreads;
            raw[c] = ci < nch ? sb[ci] : make_uint4(0, 0, 0, 0);
        }
        if (tid == 0) {
            tail->xy = (y >= c0 && y < c1)
                ? bf16_bits_to_float(reinterpret_cast<const uint16_t*>(sb)[y - c0]) : -INFINITY;
        }
        // per-thread max over its columns
        float m = -INFINITY;
        #pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
            if (tid + c * kCeThreads < nch) {
                const uint32_t wv[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
                #pragma unroll
                for (int h = 0; h < 4; ++h) m = fmaxf(m, fmaxf(bf16lo(wv[h]), bf16hi(wv[h])));
            }
        }
        // e_v = exp(x_v - m), kept in registers until the row's lse is known
        float ev[CHUNKS * 8];
        float s = 0.f;
        const float mb = m * kLog2e;
        #pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
            const bool valid = tid + c * kCeThreads < nch;
            const uint32_t wv[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
            #pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float a0 = valid ? exp2f(fmaf(bf16lo(wv[h]), kLog2e, -mb)) : 0.f;
                const float a1 = valid ? exp2f(fmaf(bf16hi(wv[h]), kLog2e, -mb)) : 0.f;
                ev[c * 8 + 2 * h] = a0;
                ev[c * 8 + 2 * h + 1] = a1;
                s += a0 + a1;
            }
        }
        // warp, then block combine of (m, s)
        float wm = m, ws = s;
        #pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, wm, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, ws, o);
            lse_combine(wm, ws, m2, s2);
        }
        if (lane == 0) { tail->red_m[warp] = wm; tail->red_s[warp] = ws; }
        __syncthreads();   // all threads are done with buffer b and wrote red_*

        const int xs = k;  // exchange index (every scored row exchanges once)
        const uint32_t xbar = smem_addr(&tail->xbar[xs & 1]);
        if (tid == 0) {
            if (issued < my_scored) issue(issued++);
            float bm = tail->red_m[0], bs = tail->red_s[0];
            for (int i = 1; i < kCeWarps; ++i) lse_combine(bm, bs, tail->red_m[i], tail->red_s[i]);
            mbar_arrive_expect_tx(xbar, uint32_t(K) * 16u);
            const uint32_t slot = smem_addr(&tail->xslot[xs & 1][rank]);
            for (int r = 0; r < K; ++r) {
                st_async_v4(mapa_shared(slot, uint32_t(r)), bm, bs, tail->xy, 0.f,
                            mapa_shared(xbar, uint32_t(r)));
            }
        }
        if (!mbar_wait_bounded<true>(xbar, uint32_t(xs >> 1) & 1u, P.status)) ok = false;
        if (__syncthreads_or(!ok)) { ok = false; break; }

        float M = -INFINITY, Ssum = 0.f, XY = -INFINITY;
        for (int r = 0; r < K; ++r) {
            const float4 v = tail->xslot[xs & 1][r];
            lse_combine(M, Ssum, v.x, v.y);
            XY = fmaxf(XY, v.z);
        }
        const float lse = M + logf(Ssum);
        const float coef = P.grad_scale * w;
        const float sc = m == -INFINITY ? 0.f : coef * exp2f((m - lse) * kLog2e);

        const uint16_t* xrow;
        uint16_t* drow;
        row_ptrs(P, q, xrow, drow);
        uint4* dst = reinterpret_cast<uint4*>(drow + c0);
        #pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
            const int ci = tid + c * kCeThreads;
            if (ci < nch) {
                float g[8];
                #pragma unroll
                for (int h = 0; h < 8; ++h) g[h] = ev[c * 8 + h] * sc;
                const int col = c0 + ci * 8;
                if (y >= col && y < col + 8) g[y - col] -= coef;
                uint4 o;
                o.x = pack_bf16x2(g[0], g[1]);
                o.y = pack_bf16x2(g[2], g[3]);
                o.z = pack_bf16x2(g[4], g[5]);
                o.w = pack_bf16x2(g[6], g[7]);
                __stcs(dst + ci, o);
            }
        }
        if (rank == 0 && tid == 0) P.row_loss[q] = w * (lse - XY);
    }

    if (ok) {
        // unscored rows: exact zeros
        const uint4 z = make_uint4(0, 0, 0, 0);
        for (int i = n_scored + cid; i < n_rows; i += C) {
            const int q = P.list[i].x;
            const uint16_t* xrow;
            uint16_t* drow;
            row_ptrs(P, q, xrow, drow);
            uint4* dst = reinterpret_cast<uint4*>(drow + c0);
            #pragma unroll
            for (int c = 0; c < CHUNKS; ++c) {
                const int ci = tid + c * kCeThreads;
                if (ci < nch) __stcs(dst + ci, z);
            }
            if (rank == 0 && tid == 0) P.row_loss[q] = 0.f;
        }
    } else if (tid == 0) {
        // drain this CTA's own copies still in flight before leaving
        for (int j = waited; j < issued; ++j)
            mbar_wait_bounded<false>(smem_addr(&tail->full[j % nbuf]), uint32_t(j / nbuf) & 1u, P.status);
    }
    // no CTA leaves while a peer may still write into its shared memory
    cluster_sync_all();
}

// General path: one CTA per row (grid-stride), any vocab / stride / alignment.
constexpr int kGenThreads = 256;

__global__ void __launch_bounds__(kGenThreads) k_ce_generic(const CeParams P) {
    __shared__ float red_m[kGenThreads / 32], red_s[kGenThreads / 32];
    __shared__ float s_lse;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
            for (int v = tid; v < V; v += kGenThreads) d[v] = 0;
            if (tid == 0) P.row_loss[q] = 0.f;
            continue;
        }
        float m = -INFINITY, s = 0.f;
        for (int v = tid; v < V; v += kGenThreads) {
            const float xv = bf16_bits_to_float(x[v]);
            if (xv > m) { s = s * exp2f((m - xv) * kLog2e) + 1.f; m = xv; }
            else        { s += exp2f((xv - m) * kLog2e); }
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
            float g = coef * exp2f((xv - lse) * kLog2e);
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
};

constexpr int kRedThreads = 1024;

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

__global__ void __launch_bounds__(kRedThreads) k_reduce(ReduceParams R) {
    __shared__ double red[kRedThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int U = R.a.n_units;
    for (int u = warp; u < U; u += kRedThreads / 32) {
        double acc = 0.0;
        int64_t lo, hi;
        unit_range(R.a, u, lo, hi);
        for (int64_t i = lo + lane; i < hi; i += 32) acc += double(R.row_loss[i]);
        unit_range(R.b, u, lo, hi);
        for (int64_t i = lo + lane; i < hi; i += 32) acc += double(R.row_loss[R.a.n_tokens + i]);
        #pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) {
            R.unit_acc[u] = acc;
            if (R.unit_loss) R.unit_loss[u] = float(acc);
        }
    }
    __syncthreads();
    // total: each thread a contiguous run of units, then a fixed tree
    const int per = (U + kRedThreads - 1) / kRedThreads;
    double acc = 0.0;
    for (int u = tid * per; u < min(U, (tid + 1) * per); ++u) acc += R.unit_acc[u];
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) red[warp] = acc;
    __syncthreads();
    if (warp == 0) {
        double v = red[lane];
        #pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) R.loss[0] = float(v);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
constexpr size_t kSmemBudget = 227 * 1024;

struct ClusterCfg {
    int K = 0, S = 0, chunks = 0, nbuf = 0;
    size_t smem = 0;
};

// Smallest cluster K (1..8) whose per-CTA slice fits CHUNKS <= 8 per thread
// and leaves room for at least two shared buffers.
static ClusterCfg pick_cluster(int V) {
    ClusterCfg c;
    for (int K = 1; K <= kMaxCluster; ++K) {
        const int S = int(align_up(size_t((V + K - 1) / K), 8));
        if ((K - 1) * S >= V) break;
        const int chunks = (S / 8 + kCeThreads - 1) / kCeThreads;
        if (chunks > 8) continue;
        const size_t tail = sizeof(CeSmemTail);
        int nbuf = int((kSmemBudget - tail - 128) / (size_t(S) * 2));
        nbuf = nbuf > kMaxBuf ? kMaxBuf : nbuf;
        if (nbuf < 2) continue;
        c.K = K; c.S = S; c.chunks = chunks; c.nbuf = nbuf;
        c.smem = size_t(nbuf) * S * 2 + tail;
        return c;
    }
    return c;
}

using CeKernel = void (*)(const CeParams);

static CeKernel cluster_kernel(int chunks) {
    switch (chunks) {
        case 1: return k_ce_cluster<1>;
        case 2: return k_ce_cluster<2>;
        case 3: return k_ce_cluster<3>;
        case 4: return k_ce_cluster<4>;
        case 5: return k_ce_cluster<5>;
        case 6: return k_ce_cluster<6>;
        case 7: return k_ce_cluster<7>;
        case 8: return k_ce_cluster<8>;
        default: return nullptr;
    }
}

// Occupancy of a cluster configuration, cached per (device, K, chunks, smem).
static int max_active_clusters(int dev, CeKernel kern, const ClusterCfg& c) {
    struct Entry { int dev, K, chunks; size_t smem; int n; };
    static std::mutex mu;
    static Entry cache[64];
    static int n_cache = 0;
    std::lock_guard<std::mutex> g(mu);
    for (int i = 0; i < n_cache; ++i)
        if (cache[i].dev == dev && cache[i].K == c.K && cache[i].chunks == c.chunks && cache[i].smem == c.smem)
            return cache[i].n;
    int n = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(c.smem)) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(c.K * 148, 1, 1);
        cfg.blockDim = dim3(kCeThreads, 1, 1);
        cfg.dynamicSmemBytes = c.smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = c.K;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();
    if (n_cache < 64) cache[n_cache++] = Entry{dev, c.K, c.chunks, c.smem, n};
    return n;
}

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

}  // namespace dlm

using namespace dlm;

extern "C" size_t dlm_loss_workspace_size(const dlm_layout_t* layout, const dlm_layout_t* enc_layout) {
    if (!layout) return 0;
    const int64_t rows = layout->n_tokens + (enc_layout ? enc_layout->n_tokens : 0);
    return ws_layout(rows, layout->n_units).total;
}

extern "C" dlm_status_t dlm_loss_fwd_bwd(const dlm_layout_t* layout, const uint16_t* logits, int64_t ld,
                                         int32_t vocab, const int32_t* clean_ids, const uint8_t* corrupted,
                                         const float* p, int32_t mode, int32_t align,
                                         const dlm_layout_t* enc_layout, const uint16_t* enc_logits,
                                         int64_t enc_ld, const int32_t* enc_ids, float enc_ar_weight,
                                         float grad_scale, float* loss, float* unit_loss,
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

    // ---- 1. plan ----
    PlanParams pp{};
    pp.a = to_dev(layout);
    pp.clean_a = clean_ids;
    pp.corrupted = corrupted;
    pp.p = p;
    pp.mode = mode;
    pp.align = align;
    pp.b = to_dev(lb);
    pp.ids_b = enc_ids;
    pp.lam = enc_ar_weight;
    pp.vocab = vocab;
    pp.hdr = hdr;
    pp.list = list;
    k_plan<<<1, kPlanThreads, 0, s>>>(pp);
    if ((st = last_launch_status()) != DLM_OK) return st;

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

        bool fast = (vocab % 8 == 0) && (ld % 8 == 0) && vocab >= 4096 &&
                    (rows_a == 0 || (aligned16(logits) && aligned16(dlogits)));
        if (has_enc) fast = fast && (enc_ld % 8 == 0) && aligned16(enc_logits) && aligned16(enc_dlogits);
        ClusterCfg cc;
        int n_clusters = 0;
        CeKernel kern = nullptr;
        if (fast) {
            cc = pick_cluster(vocab);
            kern = cc.K ? cluster_kernel(cc.chunks) : nullptr;
            if (kern) {
                int dev = 0;
                cudaGetDevice(&dev);
                n_clusters = max_active_clusters(dev, kern, cc);
            }
            fast = kern && n_clusters > 0;
        }
        if (fast) {
            if (n_clusters > R) n_clusters = int(R);
            cp.slice = cc.S;
            cp.nbuf = cc.nbuf;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(unsigned(n_clusters * cc.K), 1, 1);
            cfg.blockDim = dim3(kCeThreads, 1, 1);
            cfg.dynamicSmemBytes = cc.smem;
            cfg.stream = s;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = cc.K;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaLaunchKernelEx(&cfg, kern, cp) != cudaSuccess) { cudaGetLastError(); return DLM_ERR_CUDA; }
        } else {
            int dev = 0, sms = 148;
            cudaGetDevice(&dev);
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            const int64_t grid = R < int64_t(sms) * 8 ? R : int64_t(sms) * 8;
            k_ce_generic<<<unsigned(grid), kGenThreads, 0, s>>>(cp);
            if ((st = last_launch_status()) != DLM_OK) return st;
        }
    }

    // ---- 3. reduce ----
    ReduceParams rp{};
    rp.a = to_dev(layout);
    rp.b = to_dev(lb);
    rp.row_loss = row_loss;
    rp.unit_acc = unit_acc;
    rp.unit_loss = unit_loss;
    rp.loss = loss;
    k_reduce<<<1, kRedThreads, 0, s>>>(rp);
    return last_launch_status();
}
