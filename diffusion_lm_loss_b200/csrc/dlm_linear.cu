// dlm_linear.cu -- the diffusion loss computed from hidden states and a
// linear output head, logits never written to memory ("Native diffusion
// language-model training", Adapters, merging and inference: Cut Cross
// Entropy -- full-vocabulary CE from hidden states, aligned targets, plain
// linear head).  Absorbing noise (aligned or shifted rows), and uniform noise
// with its encoder next-token term ("diffusiongemma-26B-A4B-it-ALWAYS-THINK",
// Finetuning notes): the row plan lists the scored rows of both hidden-state
// arrays (canvas rows first, then encoder rows) and everything after the
// gather sees one set of M rows against one head.  The head is a dense
// contraction, so it runs on the 5th-gen
// tensor cores: tcgen05.mma from shared memory into tensor-memory
// accumulators, operands brought in by TMA tile loads (no multicast).
//
// With H_M = the M masked rows of H (gathered), W the [V, D] head:
//   forward   Z = H_M W^T, tile by tile; the epilogue reads each 128x256
//             accumulator half-tile out of tensor memory and keeps only per-row
//             (max, sum exp) partials and the target logit -> lse per row.
//   backward  per vocabulary chunk of kVc columns (a bounded buffer, never a
//             [M, V] tensor): Z_c recomputed, dZ_c = w (softmax - onehot) in
//             bf16; dH_M += dZ_c W_c; dW_c = dZ_c^T H_M.
// Executed flops 8 M D V (the recompute adds 2 M D V to the 6 M D V the
// method needs); every GEMM is the same warp-specialized persistent kernel,
// launched as clusters of two CTAs (one per SM) that share each MMA:
//   warp 0   TMA producer (one thread per CTA): this CTA's 128 A rows and
//            its half of the 256 B rows per K step, a 6-stage ring
//   warp 1   MMA issuer (one thread, even CTA only): 256x256x16 bf16
//            cta_group::2 MMAs; the accumulator's rows are split 128/128
//            over the two CTAs' tensor memory, two 256-column buffers each
//            (the epilogue of tile i overlaps the main loop of tile i+1)
//   warps 2-5  epilogue, in both CTAs: tensor memory -> registers ->
//            (partials | dZ | dH accumulate | dW store)
// Tile raster: the forward and dZ GEMMs walk M fastest (H_M, the small
// operand, stays in L2 while W streams once); the dH and dW GEMMs walk N
// fastest so the dZ chunk (the large operand) streams once per wave.
// Every wait is bounded (a broken pipeline sets DLM_DEV_WAIT_TIMEOUT and the
// kernel winds down instead of hanging).
#include <cstdio>
#include <mutex>

#include <cudaTypedefs.h>

#include "dlm_device.cuh"
#include "dlm_host.h"
#include "dlm_tc.cuh"

namespace dlm {

constexpr int kBM = 128, kBN = 256, kBK = 64;   // per-CTA accumulator tile 128 x 256, K step 64
constexpr int kGemmThreads = 192;
constexpr uint32_t kStageA = kBM * kBK * 2;   // 16 KB: this CTA's 128 A rows x 64
#ifndef DLM_LIN_VC
#define DLM_LIN_VC 16384
#endif
#ifndef DLM_DH_N_FASTEST
#define DLM_DH_N_FASTEST 1
#endif
constexpr int kVc = DLM_LIN_VC;               // vocabulary chunk of the backward pass
constexpr int kRowPad = 256;                  // masked-row buffers are padded to the paired tile height

// PAIR = 2: a CTA pair (cluster of 2) computes a 256 x 256 tile with
// cta_group::2 MMAs -- each CTA loads its own 128 A rows and half of the 256
// B rows, so a CTA streams 32 KB per K step instead of 48 KB and the ring
// holds 6 stages.  PAIR = 1: one CTA per 128 x 256 tile, 4 stages.
template <int PAIR>
struct GemmCfg {
    static constexpr int kStages = PAIR == 2 ? 6 : 4;
    static constexpr int kBRows = kBN / PAIR;                  // B rows (N) loaded by one CTA
    static constexpr uint32_t kStageB = kBRows * kBK * 2;      // 16 or 32 KB
    static constexpr int kTileM = kBM * PAIR;                  // C rows per tile
};

enum Epi { EPI_LSE = 0, EPI_DZ = 1, EPI_DH = 2, EPI_DW = 3 };

struct GemmArgs {
    const WsHeader* hdr;     // hdr->n_scored = M (masked rows)
    uint32_t* status;
    const int4* list;        // row plan: {token row, target, weight bits, unit}
    int m_dev;               // 1: C rows = round_up(M, 128); 0: m_rows
    int m_rows;
    int n_cols;              // C columns
    int k_dev;               // 1: K = round_up(M, 128); 0: k_len
    int k_len;
    int n_fastest;           // tile raster: 0 = consecutive tiles share the B tile, 1 = share the A tile
    int b_off;               // row offset of W (forward / dZ) or K offset into W rows (dH)
    int col0;                // vocabulary index of C column 0 (LSE, DZ) or C row 0 (DW)
    int vocab;
    int d_model;
    float grad_scale;
    float2* part;            // LSE: [Mp, part_ld] (max, sum exp)
    int part_ld;
    float* xy;               // LSE: target logit per masked row
    const float* lse;        // DZ
    uint16_t* dz;            // DZ out: [Mp, dz_ld] bf16
    int dz_ld;
    float* dh;               // DH: [Mp, D] f32
    int accumulate;
    uint16_t* dw;            // DW: [V, D] bf16
};

constexpr uint32_t kStageRowBytes = 128;                // one staged row: 64 bf16 or 32 f32
constexpr uint32_t kStageBytes = 32 * kStageRowBytes;   // 32 rows (one epilogue warp)

template <int PAIR>
struct __align__(1024) GemmSmem {
    uint8_t a[GemmCfg<PAIR>::kStages][kStageA];
    uint8_t b[GemmCfg<PAIR>::kStages][GemmCfg<PAIR>::kStageB];
    uint8_t stage[4][2][kStageBytes];   // per epilogue warp, double-buffered TMA-store staging
    uint64_t full[GemmCfg<PAIR>::kStages];
    uint64_t empty[GemmCfg<PAIR>::kStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ int round_up_dev(int x, int a) { return (x + a - 1) / a * a; }

// Write one 128-byte row (8 x 16 B) of lane `row` into a 32-row staging tile
// laid out for a 128-byte-swizzled TMA box: 16-byte unit j of row r sits at
// unit (j ^ (r % 8)) -- which also keeps the 32 lanes' stores bank-conflict
// free.  The tile must be 1024-byte aligned.
__device__ __forceinline__ void stage_row(uint8_t* tile, int row, const uint4 (&v)[8]) {
    uint4* r = reinterpret_cast<uint4*>(tile + row * kStageRowBytes);
    #pragma unroll
    for (int j = 0; j < 8; ++j) r[j ^ (row & 7)] = v[j];
}

template <int EPI, bool A_MN, bool B_MN, int PAIR>
__global__ void __launch_bounds__(kGemmThreads, 1)
k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
       const __grid_constant__ CUtensorMap tmC, const GemmArgs g) {
    using Cfg = GemmCfg<PAIR>;
    constexpr int kStages = Cfg::kStages;
    constexpr uint32_t kStageB = Cfg::kStageB;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    GemmSmem<PAIR>& S = *reinterpret_cast<GemmSmem<PAIR>*>(smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* abort = &S.abort;
    // the pair: rank 0 issues the MMAs for both CTAs; tiles go to clusters
    const uint32_t rank = PAIR == 2 ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    const int unit = PAIR == 2 ? int(cluster_id_x()) : int(blockIdx.x);
    const int n_units = PAIR == 2 ? int(nclusters_x()) : int(gridDim.x);

    const int M = g.hdr->n_scored;
    const int Mp = round_up_dev(M, kBM);
    const int rows = g.m_dev ? Mp : g.m_rows;
    const int K = g.k_dev ? Mp : g.k_len;
    const int m_tiles = (rows + Cfg::kTileM - 1) / Cfg::kTileM;
    const int n_tiles = (g.n_cols + kBN - 1) / kBN;
    const int tiles = m_tiles * n_tiles;
    const int nkb = K / kBK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(smem_addr(&S.full[i]), 1);
            mbar_init(smem_addr(&S.empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_addr(&S.tfull[i]), 1);
            mbar_init(smem_addr(&S.tempty[i]), 4 * PAIR);   // every epilogue warp of the pair
        }
        mbar_init(smem_addr(&S.drain), 1);
        S.abort = 0;
        fence_mbar_init_cluster();
        tc::prefetch_tensormap(&tmA);
        tc::prefetch_tensormap(&tmB);
        if (EPI != EPI_LSE) tc::prefetch_tensormap(&tmC);
    }
    if (warp == 1) {
        if (PAIR == 2) { tc::tmem_alloc_pair(smem_addr(&S.tmem_base), 512); tc::tmem_relinquish_pair(); }
        else           { tc::tmem_alloc(smem_addr(&S.tmem_base), 512);      tc::tmem_relinquish(); }
    }
    tc::fence_before_thread_sync();
    __syncthreads();
    if (PAIR == 2) cluster_sync_all();   // the peer's barriers exist before anyone signals them
    tc::fence_after_thread_sync();
    const uint32_t tmem = S.tmem_base;

    // tile -> (first C row of this CTA, first C column)
    auto tile_coords = [&](int tile, int& m0, int& nt) {
        const int mt = g.n_fastest ? tile / n_tiles : tile % m_tiles;
        nt = g.n_fastest ? tile % n_tiles : tile / m_tiles;
        m0 = mt * Cfg::kTileM + int(rank) * kBM;
    };

    if (warp == 0 && lane == 0) {
        // ------------------------------ TMA producer ------------------------------
        // Each CTA loads its own A rows and its share of the B rows; the bytes
        // of both CTAs complete on the leader's full barrier.
        uint64_t pol_a, pol_b;
        if (EPI == EPI_LSE || EPI == EPI_DZ) { pol_a = policy_evict_last(); pol_b = policy_evict_first(); }
        else                                 { pol_a = policy_evict_normal(); pol_b = policy_evict_normal(); }
        int it = 0;
        bool ok = true;
        for (int tile = unit; tile < tiles && ok; tile += n_units) {
            int m0, nt;
            tile_coords(tile, m0, nt);
            const int nb = nt * kBN + int(rank) * Cfg::kBRows;   // this CTA's first B row (N)
            for (int kb = 0; kb < nkb; ++kb, ++it) {
                const int s = it % kStages;
                if (!mbar_wait_or_abort(smem_addr(&S.empty[s]), ((it / kStages) & 1) ^ 1, g.status, abort)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = smem_addr(&S.full[s]);
                const uint32_t fb_lead = PAIR == 2 ? mapa_shared(fb, 0) : fb;
                if (leader) mbar_arrive_expect_tx(fb, PAIR * (kStageA + kStageB));
                const int k0 = kb * kBK;
                const uint32_t a_s = smem_addr(S.a[s]), b_s = smem_addr(S.b[s]);
                auto load = [&](uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t pol) {
                    if (PAIR == 2) tc::tma_load_2d_pair(dst, map, x, y, fb_lead, pol);
                    else           tc::tma_load_2d(dst, map, x, y, fb, pol);
                };
                if (!A_MN) {
                    load(a_s, &tmA, k0, m0, pol_a);
                } else {
                    load(a_s, &tmA, m0, k0, pol_a);
                    load(a_s + 8192, &tmA, m0 + 64, k0, pol_a);
                }
                if (!B_MN) {
                    load(b_s, &tmB, k0, nb + g.b_off, pol_b);
                } else {
                    #pragma unroll
                    for (int j = 0; j < Cfg::kBRows / 64; ++j)
                        load(b_s + 8192 * j, &tmB, nb + 64 * j, k0 + g.b_off, pol_b);
                }
            }
        }
        if (!ok && (PAIR == 1 || leader)) {
            // let the copies already issued land before the CTA can exit (a
            // pair's second CTA cannot observe its own copies -- they complete
            // on the leader's barrier -- but it only gets here after a wait of
            // seconds, long after any copy it issued has landed)
            for (int j = it - 1; j >= 0 && j >= it - kStages; --j)
                mbar_wait_bounded<false>(smem_addr(&S.full[j % kStages]), (j / kStages) & 1, nullptr);
        }
    } else if (warp == 1 && lane == 0 && leader) {
        // ------------------------------ MMA issuer ------------------------------
        constexpr uint32_t idesc = tc::idesc_bf16(Cfg::kTileM, kBN, A_MN ? 1 : 0, B_MN ? 1 : 0);
        int it = 0, lt = 0;
        bool ok = nkb > 0;
        for (int tile = unit; tile < tiles && ok; tile += n_units, ++lt) {
            const int acc = lt & 1;
            const bool free_acc = PAIR == 2
                ? mbar_wait_or_abort_cluster(smem_addr(&S.tempty[acc]), ((lt >> 1) & 1) ^ 1, g.status, abort)
                : mbar_wait_or_abort(smem_addr(&S.tempty[acc]), ((lt >> 1) & 1) ^ 1, g.status, abort);
            if (!free_acc) {
                ok = false;
                break;
            }
            tc::fence_after_thread_sync();
            const uint32_t d_tmem = tmem + uint32_t(acc * kBN);
            for (int kb = 0; kb < nkb; ++kb, ++it) {
                const int s = it % kStages;
                if (!mbar_wait_or_abort(smem_addr(&S.full[s]), (it / kStages) & 1, g.status, abort)) {
                    ok = false;
                    break;
                }
                tc::fence_after_thread_sync();
                const uint32_t a_s = smem_addr(S.a[s]), b_s = smem_addr(S.b[s]);
                #pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
                    const uint64_t ad = A_MN ? tc::smem_desc_sw128(a_s + kk * 2048, 8192, 1024)
                                             : tc::smem_desc_sw128(a_s + kk * 32, 16, 1024);
                    const uint64_t bd = B_MN ? tc::smem_desc_sw128(b_s + kk * 2048, 8192, 1024)
                                             : tc::smem_desc_sw128(b_s + kk * 32, 16, 1024);
                    if (PAIR == 2) tc::mma_bf16_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
                    else           tc::mma_bf16(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
                }
                // the stage is reusable (in both CTAs) once these MMAs retire
                if (PAIR == 2) tc::mma_commit_pair(smem_addr(&S.empty[s]), 0x3);
                else           tc::mma_commit(smem_addr(&S.empty[s]));
            }
            if (!ok) break;
            // accumulator ready for the epilogue (of both CTAs)
            if (PAIR == 2) tc::mma_commit_pair(smem_addr(&S.tfull[acc]), 0x3);
            else           tc::mma_commit(smem_addr(&S.tfull[acc]));
        }
        // no MMA may still be running when tensor memory is released
        if (PAIR == 2) tc::mma_commit_pair(smem_addr(&S.drain), 0x3);
        else           tc::mma_commit(smem_addr(&S.drain));
        mbar_wait_bounded<false>(smem_addr(&S.drain), 0, nullptr);
    } else if (warp == 1 && lane == 0) {
        // the pair's second CTA: its tensor memory is written by the leader's
        // MMAs; wait for the leader's final completion signal before release
        mbar_wait_bounded<false>(smem_addr(&S.drain), 0, nullptr);
    } else if (warp >= 2) {
        // ------------------------------ epilogue ------------------------------
        const int quarter = warp & 3;               // tensor-memory lanes 32*quarter .. +31
        const int r_in_tile = quarter * 32 + lane;
        const bool kempty = nkb == 0;
        int lt = 0;
        int sc = 0;   // staging boxes written by this warp (buffer parity)
        // accumulator release: the leader's barrier counts the epilogue warps of both CTAs
        auto release_acc = [&](int acc) {
            tc::fence_before_thread_sync();
            __syncwarp();
            if (lane == 0) {
                if (PAIR == 2) mbar_arrive_remote(mapa_shared(smem_addr(&S.tempty[acc]), 0));
                else           mbar_arrive(smem_addr(&S.tempty[acc]));
            }
        };
        for (int tile = unit; tile < tiles; tile += n_units, ++lt) {
            const int acc = lt & 1;
            int m0, nt;
            tile_coords(tile, m0, nt);
            const int n0 = nt * kBN;
            const int m = m0 + r_in_tile;
            if (!kempty) {
                // warp-uniform exit: tcgen05.ld below needs all 32 lanes
                const bool got = mbar_wait_or_abort(smem_addr(&S.tfull[acc]), (lt >> 1) & 1, g.status, abort);
                if (__any_sync(0xffffffffu, !got)) break;
                tc::fence_after_thread_sync();
            }
            const uint32_t taddr = tmem + uint32_t(acc * kBN) + (uint32_t(quarter * 32) << 16);

            if (EPI == EPI_LSE) {
                const bool rv = m < M;
                const int tg = rv ? __ldg(&g.list[m].y) : -1;
                float mx = -INFINITY, sm = 0.f, xyv = 0.f;
                bool have_xy = false;
                for (int c = 0; c < kBN / 32; ++c) {
                    uint32_t r[32];
                    tc::tmem_ld_32x32b_x32(taddr + c * 32, r);
                    tc::tmem_ld_wait();
                    const int cb = g.col0 + n0 + c * 32;
                    float cm = -INFINITY;
                    #pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float f = __uint_as_float(r[j]);
                        if (cb + j < g.vocab) cm = fmaxf(cm, f);
                        if (cb + j == tg) { xyv = f; have_xy = true; }
                    }
                    if (cm > mx) {
                        sm = (mx == -INFINITY) ? 0.f : sm * ex2((mx - cm) * 1.4426950408889634f);
                        mx = cm;
                    }
                    if (mx != -INFINITY) {
                        const float mb = mx * 1.4426950408889634f;
                        #pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (cb + j < g.vocab) sm += ex2(fmaf(__uint_as_float(r[j]), 1.4426950408889634f, -mb));
                    }
                }
                release_acc(acc);
                if (rv) {
                    g.part[size_t(m) * g.part_ld + nt] = make_float2(mx, sm);
                    if (have_xy) g.xy[m] = xyv;
                }
            } else {
                // stores go out through TMA from a per-warp staging tile:
                // 64 bf16 columns (dZ, dW) or 32 f32 columns (dH) per box
                constexpr int kColsPerBox = EPI == EPI_DH ? 32 : 64;
                constexpr int kBoxes = kBN / kColsPerBox;
                const bool rv = m < M;
                int tg = -1;
                float coef = 0.f, lb = 0.f;
                if (EPI == EPI_DZ && rv) {
                    const int4 e = __ldg(&g.list[m]);
                    tg = e.y;
                    coef = g.grad_scale * __int_as_float(e.z);
                    lb = g.lse[m] * 1.4426950408889634f;
                }
                const int ew = warp - 2;                       // epilogue warp index 0..3
                const int y0 = (EPI == EPI_DW ? g.col0 : 0) + m0 + quarter * 32;
                for (int bx = 0; bx < kBoxes; ++bx) {
                    uint4 v[8];
                    if (EPI == EPI_DH) {
                        uint32_t r[32];
                        if (!kempty) {
                            tc::tmem_ld_32x32b_x32(taddr + bx * 32, r);
                            tc::tmem_ld_wait();
                        } else {
                            #pragma unroll
                            for (int j = 0; j < 32; ++j) r[j] = 0u;
                        }
                        #pragma unroll
                        for (int j = 0; j < 8; ++j) v[j] = make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
                    } else {
                        uint32_t pk[32];
                        #pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            uint32_t r[32];
                            if (!kempty) {
                                tc::tmem_ld_32x32b_x32(taddr + bx * 64 + half * 32, r);
                                tc::tmem_ld_wait();
                            } else {
                                #pragma unroll
                                for (int j = 0; j < 32; ++j) r[j] = 0u;
                            }
                            if (EPI == EPI_DZ) {
                                const int cb = g.col0 + n0 + bx * 64 + half * 32;
                                #pragma unroll
                                for (int j = 0; j < 32; j += 2) {
                                    float v0 = 0.f, v1 = 0.f;
                                    if (rv && cb + j < g.vocab)
                                        v0 = coef * ex2(fmaf(__uint_as_float(r[j]), 1.4426950408889634f, -lb)) -
                                             (cb + j == tg ? coef : 0.f);
                                    if (rv && cb + j + 1 < g.vocab)
                                        v1 = coef * ex2(fmaf(__uint_as_float(r[j + 1]), 1.4426950408889634f, -lb)) -
                                             (cb + j + 1 == tg ? coef : 0.f);
                                    pk[half * 16 + j / 2] = pack_bf16x2(v0, v1);
                                }
                            } else {
                                #pragma unroll
                                for (int j = 0; j < 16; ++j)
                                    pk[half * 16 + j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
                            }
                        }
                        #pragma unroll
                        for (int j = 0; j < 8; ++j) v[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                    }
                    // all of this tile's accumulator is in registers: free it
                    if (bx == kBoxes - 1 && !kempty) release_acc(acc);
                    const int buf = sc & 1;
                    if (lane == 0) bulk_wait_group_read<1>();   // the store from this buffer two boxes ago is done reading
                    __syncwarp();
                    uint8_t* tile_s = S.stage[ew][buf];
                    stage_row(tile_s, lane, v);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        // boxes that start outside the tensor are skipped (partial
                        // boxes are clipped by the TMA unit); coordinates >= 0
                        const int x = n0 + bx * kColsPerBox;
                        const int xlim = EPI == EPI_DZ ? g.dz_ld : g.d_model;
                        const int ylim = EPI == EPI_DW ? g.vocab : 0x7fffffff;
                        if (x < xlim && y0 < ylim) {
                            if (EPI == EPI_DH && g.accumulate) tc::tma_reduce_add_2d(&tmC, x, y0, smem_addr(tile_s));
                            else                                tc::tma_store_2d(&tmC, x, y0, smem_addr(tile_s));
                        }
                        bulk_commit_group();
                    }
                    ++sc;
                }
            }
        }
        if (EPI != EPI_LSE && lane == 0) bulk_wait_group<0>();   // all stores complete before the CTA ends
    }
    __syncthreads();
    __syncwarp();
    // neither CTA of a pair leaves (or frees tensor memory) while the other
    // may still signal its barriers
    if (PAIR == 2) cluster_sync_all();
    if (warp == 1) {
        tc::fence_after_thread_sync();
        if (PAIR == 2) tc::tmem_dealloc_pair(tmem, 512);
        else           tc::tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
// small kernels around the GEMMs
// ---------------------------------------------------------------------------
// H_M[m] = row list[m].row of the hidden states for m < M, zero rows up to
// round_up(M, 256) (the height of a paired tile).  Rows [0, Ta) are rows of H,
// rows from Ta on are rows of He (the encoder's hidden states, uniform noise).
__global__ void k_gather(const WsHeader* hdr, const int4* list, const uint16_t* __restrict__ H,
                         const uint16_t* __restrict__ He, int64_t Ta, int D, uint16_t* __restrict__ HM) {
    const int M = hdr->n_scored;
    const int Mp = round_up_dev(M, kRowPad);
    const int vecs = D / 8;
    for (int r = blockIdx.x; r < Mp; r += gridDim.x) {
        uint4* dst = reinterpret_cast<uint4*>(HM + size_t(r) * D);
        if (r < M) {
            const int64_t q = __ldg(&list[r].x);
            const uint16_t* row = q < Ta ? H + size_t(q) * D : He + size_t(q - Ta) * D;
            const uint4* src = reinterpret_cast<const uint4*>(row);
            for (int i = threadIdx.x; i < vecs; i += blockDim.x) dst[i] = __ldg(src + i);
        } else {
            for (int i = threadIdx.x; i < vecs; i += blockDim.x) dst[i] = make_uint4(0, 0, 0, 0);
        }
    }
}

// lse per masked row from the per-tile partials (fixed order), row losses:
// row_loss[row] = w (lse - z_target) for masked rows, 0 for all other rows.
__global__ void k_lse(const WsHeader* hdr, const int4* list, const float2* __restrict__ part, int part_ld,
                      const float* __restrict__ xy, float* __restrict__ lse, float* __restrict__ row_loss) {
    const int M = hdr->n_scored;
    const int R = hdr->n_rows;
    const int warp_g = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int m = warp_g; m < R; m += nwarps) {
        const int4 e = list[m];
        if (m >= M) {
            if (lane == 0) row_loss[e.x] = 0.f;
            continue;
        }
        float mx = -INFINITY, s = 0.f;
        for (int t = lane; t < part_ld; t += 32) {
            const float2 v = part[size_t(m) * part_ld + t];
            if (v.x == -INFINITY) continue;
            if (v.x > mx) { s = (mx == -INFINITY ? 0.f : s * ex2((mx - v.x) * 1.4426950408889634f)) + v.y; mx = v.x; }
            else          { s += v.y * ex2((v.x - mx) * 1.4426950408889634f); }
        }
        #pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, mx, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
            if (m2 != -INFINITY) {
                if (mx == -INFINITY) { mx = m2; s = s2; }
                else {
                    const float Mx = fmaxf(mx, m2);
                    s = s * ex2((mx - Mx) * 1.4426950408889634f) + s2 * ex2((m2 - Mx) * 1.4426950408889634f);
                    mx = Mx;
                }
            }
        }
        if (lane == 0) {
            const float l = mx + logf(s);
            lse[m] = l;
            row_loss[e.x] = __int_as_float(e.z) * (l - xy[m]);
        }
    }
}

// d_hidden[row] = bf16(dH_M[m]) for the masked rows, 0 for all other rows
// (rows from Ta on go to d_enc_hidden[row - Ta]).
__global__ void k_scatter_dh(const WsHeader* hdr, const int4* list, const float* __restrict__ dh, int D,
                             int64_t Ta, uint16_t* __restrict__ d_hidden, uint16_t* __restrict__ d_enc_hidden) {
    const int M = hdr->n_scored;
    const int R = hdr->n_rows;
    const int vecs = D / 8;
    for (int i = blockIdx.x; i < R; i += gridDim.x) {
        const int64_t row = list[i].x;
        uint4* dst = reinterpret_cast<uint4*>(row < Ta ? d_hidden + size_t(row) * D
                                                        : d_enc_hidden + size_t(row - Ta) * D);
        if (i < M) {
            const float4* src = reinterpret_cast<const float4*>(dh + size_t(i) * D);
            for (int v = threadIdx.x; v < vecs; v += blockDim.x) {
                const float4 a = src[2 * v], b = src[2 * v + 1];
                dst[v] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                                    pack_bf16x2(b.z, b.w));
            }
        } else {
            for (int v = threadIdx.x; v < vecs; v += blockDim.x) dst[v] = make_uint4(0, 0, 0, 0);
        }
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct LinWs {
    size_t list, row_loss, unit_acc, hm, part, xy, lse, dz, dh, total;
    int tpad, n_tiles;
};

// Rows (canvas + encoder) the fused head accepts: the row count padded to
// the 256-row pair tile must stay an int.
constexpr int64_t kMaxLinRows = (int64_t(1) << 31) - 1 - kRowPad;

static LinWs lin_ws(int64_t T, int64_t units, int D, int V) {
    LinWs w;
    w.tpad = int(align_up(size_t(T > 0 ? T : 1), kRowPad));
    w.n_tiles = (V + kBN - 1) / kBN;
    size_t o = kWsAlign;
    w.list = o;     o = align_up(o + size_t(T) * 16, kWsAlign);
    w.row_loss = o; o = align_up(o + size_t(T) * 4, kWsAlign);
    w.unit_acc = o; o = align_up(o + size_t(units) * 8, kWsAlign);
    w.hm = o;       o = align_up(o + size_t(w.tpad) * D * 2, 1024);
    w.part = o;     o = align_up(o + size_t(w.tpad) * w.n_tiles * 8, kWsAlign);
    w.xy = o;       o = align_up(o + size_t(w.tpad) * 4, kWsAlign);
    w.lse = o;      o = align_up(o + size_t(w.tpad) * 4, kWsAlign);
    w.dz = o;       o = align_up(o + size_t(w.tpad) * kVc * 2, 1024);
    w.dh = o;       o = align_up(o + size_t(w.tpad) * D * 4, kWsAlign);
    w.total = o;
    return w;
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::mutex mu;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::lock_guard<std::mutex> g(mu);
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        else
            cudaGetLastError();
    }
    return fn;
}

// 2-D tensor [outer, inner] of bf16 (or f32), row stride `stride_elems`,
// box [box_outer, box_inner] with 128-byte swizzle (box_inner * elem size must
// be 128 bytes).
static bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t stride_elems,
                     uint32_t box_inner, uint32_t box_outer, bool f32 = false) {
    auto fn = encode_fn();
    if (!fn) return false;
    const uint64_t esz = f32 ? 4 : 2;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {stride_elems * esz};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                    const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

#ifndef DLM_GEMM_PAIR
#define DLM_GEMM_PAIR 2
#endif
constexpr int kPair = DLM_GEMM_PAIR;   // CTAs per MMA tile (2: cta_group::2 pairs)
static_assert(kPair == 1 || kPair == 2, "CTAs per tile");

// One persistent CTA per SM (clusters of kPair CTAs; the grid is a multiple
// of kPair).
template <int EPI, bool A_MN, bool B_MN>
static dlm_status_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c,
                                const GemmArgs& g, int grid, cudaStream_t s) {
    auto kern = k_gemm<EPI, A_MN, B_MN, kPair>;
    const size_t smem = sizeof(GemmSmem<kPair>) + 1024;
    static_assert(sizeof(GemmSmem<kPair>) + 1024 <= 227 * 1024, "shared memory per CTA");
    static std::mutex mu;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    {
        std::lock_guard<std::mutex> lk(mu);
        if (dev >= 0 && dev < 64 && !attr_done[dev]) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
            if (e != cudaSuccess) return cuda_status(e, "k_gemm smem attribute");
            attr_done[dev] = true;
        }
    }
    grid -= grid % kPair;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(unsigned(grid));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kPair;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a, b, c, g);
    if (e != cudaSuccess) return cuda_status(e, "k_gemm launch");
    return DLM_OK;
}

}  // namespace dlm

using namespace dlm;

extern "C" size_t dlm_linear_loss_workspace_size(const dlm_layout_t* layout, int32_t d_model, int32_t vocab) {
    if (!layout || d_model <= 0 || vocab <= 0 || layout->n_tokens < 0 || layout->n_tokens > kMaxLinRows) return 0;
    return lin_ws(layout->n_tokens, layout->n_units, d_model, vocab).total;
}

extern "C" size_t dlm_linear_loss_uniform_workspace_size(const dlm_layout_t* layout,
                                                         const dlm_layout_t* enc_layout, int32_t d_model,
                                                         int32_t vocab) {
    if (!layout || d_model <= 0 || vocab <= 0 || layout->n_tokens < 0) return 0;
    if (enc_layout && enc_layout->n_tokens < 0) return 0;
    const int64_t rows = layout->n_tokens + (enc_layout ? enc_layout->n_tokens : 0);
    if (rows > kMaxLinRows) return 0;
    return lin_ws(rows, layout->n_units, d_model, vocab).total;
}

// Both entry families: absorbing noise (corrupted + p select and weight the
// rows; no encoder) or uniform noise (every canvas target scored, plus the
// encoder's next-token rows when enc_layout is given).
static dlm_status_t linear_loss_fwd_bwd(const dlm_layout_t* layout, const uint16_t* hidden,
                                        const uint16_t* weight, int32_t d_model, int32_t vocab,
                                        const int32_t* clean_ids, const uint8_t* corrupted, const float* p,
                                        int32_t mode, int32_t align, const dlm_layout_t* enc_layout,
                                        const uint16_t* enc_hidden, const int32_t* enc_ids,
                                        float enc_ar_weight, float grad_scale, float* loss, float* unit_loss,
                                        uint16_t* d_hidden, uint16_t* d_enc_hidden, uint16_t* d_weight,
                                        void* workspace, size_t workspace_bytes, dlm_stream_t stream) {
    if (!layout_ok(layout)) return DLM_ERR_INVALID_ARGUMENT;
    if (mode != DLM_ABSORBING && mode != DLM_UNIFORM) return DLM_ERR_INVALID_ARGUMENT;
    if (align != DLM_ALIGNED && align != DLM_SHIFTED) return DLM_ERR_INVALID_ARGUMENT;
    if (d_model <= 0 || d_model % 64 != 0 || vocab <= 0 || vocab % 8 != 0) return DLM_ERR_INVALID_ARGUMENT;
    if (!loss || !workspace) return DLM_ERR_INVALID_ARGUMENT;
    const bool has_enc = enc_layout != nullptr;
    if (has_enc) {
        if (mode != DLM_UNIFORM) return DLM_ERR_INVALID_ARGUMENT;
        if (!layout_ok(enc_layout) || enc_layout->n_units != layout->n_units) return DLM_ERR_INVALID_ARGUMENT;
        if (enc_layout->n_tokens > 0 &&
            (!enc_hidden || !enc_ids || !d_enc_hidden || !weight ||
             (!enc_layout->cu_seqlens && enc_layout->seq_len == 0)))
            return DLM_ERR_INVALID_ARGUMENT;
        if (!aligned16(enc_hidden) || !aligned16(d_enc_hidden)) return DLM_ERR_INVALID_ARGUMENT;
    }
    const int64_t T = layout->n_tokens;
    const int64_t Te = has_enc ? enc_layout->n_tokens : 0;
    const int64_t R = T + Te;
    if (R > kMaxLinRows) return DLM_ERR_INVALID_ARGUMENT;
    if (T > 0 && (!hidden || !weight || !clean_ids || !d_hidden)) return DLM_ERR_INVALID_ARGUMENT;
    if (T > 0 && mode == DLM_ABSORBING && (!corrupted || !p)) return DLM_ERR_INVALID_ARGUMENT;
    if (T > 0 && !layout->cu_seqlens && layout->seq_len == 0) return DLM_ERR_INVALID_ARGUMENT;
    if (!aligned16(hidden) || !aligned16(weight) || !aligned16(d_hidden) || (d_weight && !aligned16(d_weight)))
        return DLM_ERR_INVALID_ARGUMENT;
    if (reinterpret_cast<uintptr_t>(workspace) % 1024) return DLM_ERR_INVALID_ARGUMENT;
    const LinWs W = lin_ws(R, layout->n_units, d_model, vocab);
    if (workspace_bytes < W.total) return DLM_ERR_WORKSPACE_TOO_SMALL;
    dlm_status_t st = check_device();
    if (st != DLM_OK) return st;

    cudaStream_t s = (cudaStream_t)stream;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    int4* list = reinterpret_cast<int4*>(ws + W.list);
    float* row_loss = reinterpret_cast<float*>(ws + W.row_loss);
    double* unit_acc = reinterpret_cast<double*>(ws + W.unit_acc);
    uint16_t* HM = reinterpret_cast<uint16_t*>(ws + W.hm);
    float2* part = reinterpret_cast<float2*>(ws + W.part);
    float* xy = reinterpret_cast<float*>(ws + W.xy);
    float* lse = reinterpret_cast<float*>(ws + W.lse);
    uint16_t* dz = reinterpret_cast<uint16_t*>(ws + W.dz);
    float* dh = reinterpret_cast<float*>(ws + W.dh);

    // 1. which rows are scored, their targets and weights (row i scores token
    //    i, or token i+1 of the same unit when shifted; absorbing noise only
    //    the corrupted ones; encoder rows after the canvas rows)
    const dlm_layout_t* lb = has_enc ? enc_layout : nullptr;
    if ((st = launch_plan(layout, clean_ids, corrupted, p, mode, align, lb, enc_ids, enc_ar_weight,
                          vocab, hdr, list, s)) != DLM_OK)
        return st;
    if (R == 0) {
        if (d_weight) {
            cudaError_t e = cudaMemsetAsync(d_weight, 0, size_t(vocab) * d_model * 2, s);
            if (e != cudaSuccess) return cuda_status(e, "cudaMemsetAsync d_weight");
        }
        return launch_reduce(layout, lb, row_loss, unit_acc, unit_loss, loss, hdr, s);
    }

    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);

    // 2. gather the masked rows of H (zero padding to a 128-row tile)
    k_gather<<<sms * 4, 256, 0, s>>>(hdr, list, hidden, enc_hidden, T, d_model, HM);
    if ((st = last_launch_status("k_gather launch")) != DLM_OK) return st;

    // tensor maps (shapes are host-known upper bounds; the kernels read M)
    CUtensorMap mHM_K, mW_K, mDZ_K, mW_MN, mDZ_MN, mHM_MN, oDZ, oDH, oDW;
    bool ok = make_map(&mHM_K, HM, d_model, W.tpad, d_model, 64, kBM) &&
              make_map(&mW_K, weight, d_model, vocab, d_model, 64, kBN / kPair) &&
              make_map(&mDZ_K, dz, kVc, W.tpad, kVc, 64, kBM) &&
              make_map(&mW_MN, weight, d_model, vocab, d_model, 64, 64) &&
              make_map(&mDZ_MN, dz, kVc, W.tpad, kVc, 64, 64) &&
              make_map(&mHM_MN, HM, d_model, W.tpad, d_model, 64, 64) &&
              // epilogue outputs, 32-row boxes of 128 bytes
              make_map(&oDZ, dz, kVc, W.tpad, kVc, 64, 32) &&
              make_map(&oDH, dh, d_model, W.tpad, d_model, 32, 32, true) &&
              (!d_weight || make_map(&oDW, d_weight, d_model, vocab, d_model, 64, 32));
    if (!d_weight) oDW = oDZ;   // unused
    if (!ok) {
        record_cuda_error(cudaErrorInvalidValue, "cuTensorMapEncodeTiled");
        return DLM_ERR_CUDA;
    }

    GemmArgs g{};
    g.hdr = hdr;
    g.status = &hdr->status;
    g.list = list;
    g.vocab = vocab;
    g.d_model = d_model;
    g.grad_scale = grad_scale;

    // 3. forward: lse partials over the whole vocabulary
    {
        GemmArgs a = g;
        a.m_dev = 1; a.n_cols = vocab; a.k_dev = 0; a.k_len = d_model; a.b_off = 0; a.col0 = 0;
        a.part = part; a.part_ld = W.n_tiles; a.xy = xy;
        if ((st = launch_gemm<EPI_LSE, false, false>(mHM_K, mW_K, mHM_K, a, sms, s)) != DLM_OK) return st;
    }
    k_lse<<<sms, 256, 0, s>>>(hdr, list, part, W.n_tiles, xy, lse, row_loss);
    if ((st = last_launch_status("k_lse launch")) != DLM_OK) return st;

    // 4. backward, one vocabulary chunk at a time
    for (int c0 = 0; c0 < vocab; c0 += kVc) {
        const int vc = vocab - c0 < kVc ? vocab - c0 : kVc;
        GemmArgs a = g;
        a.m_dev = 1; a.n_cols = int(align_up(vc, kBN)); a.k_dev = 0; a.k_len = d_model; a.b_off = c0; a.col0 = c0;
        a.lse = lse; a.dz = dz; a.dz_ld = kVc;
        if ((st = launch_gemm<EPI_DZ, false, false>(mHM_K, mW_K, oDZ, a, sms, s)) != DLM_OK) return st;

        GemmArgs h = g;
        h.m_dev = 1; h.n_cols = d_model; h.k_dev = 0; h.k_len = int(align_up(vc, kBK)); h.b_off = c0;
        h.dh = dh; h.accumulate = c0 > 0; h.n_fastest = DLM_DH_N_FASTEST;
        if ((st = launch_gemm<EPI_DH, false, true>(mDZ_K, mW_MN, oDH, h, sms, s)) != DLM_OK) return st;

        if (d_weight) {
            GemmArgs w = g;
            w.m_dev = 0; w.m_rows = int(align_up(vc, kBM)); w.n_cols = d_model; w.k_dev = 1; w.b_off = 0;
            w.col0 = c0; w.dw = d_weight; w.n_fastest = 1;
            if ((st = launch_gemm<EPI_DW, true, true>(mDZ_MN, mHM_MN, oDW, w, sms, s)) != DLM_OK) return st;
        }
    }

    // 5. d_hidden (zero rows for unscored tokens) and the reductions
    k_scatter_dh<<<sms * 4, 256, 0, s>>>(hdr, list, dh, d_model, T, d_hidden, d_enc_hidden);
    if ((st = last_launch_status("k_scatter_dh launch")) != DLM_OK) return st;
    return launch_reduce(layout, lb, row_loss, unit_acc, unit_loss, loss, hdr, s);
}

extern "C" dlm_status_t dlm_linear_loss_fwd_bwd(const dlm_layout_t* layout, const uint16_t* hidden,
                                                const uint16_t* weight, int32_t d_model, int32_t vocab,
                                                const int32_t* clean_ids, const uint8_t* corrupted,
                                                const float* p, float grad_scale, float* loss,
                                                float* unit_loss, uint16_t* d_hidden, uint16_t* d_weight,
                                                void* workspace, size_t workspace_bytes, dlm_stream_t stream) {
    DLM_NVTX("dlm_linear_loss_fwd_bwd");
    return linear_loss_fwd_bwd(layout, hidden, weight, d_model, vocab, clean_ids, corrupted, p, DLM_ABSORBING,
                               DLM_ALIGNED, nullptr, nullptr, nullptr, 0.f, grad_scale, loss, unit_loss,
                               d_hidden, nullptr, d_weight, workspace, workspace_bytes, stream);
}

extern "C" dlm_status_t dlm_linear_loss_fwd_bwd_ex(const dlm_layout_t* layout, const uint16_t* hidden,
                                                   const uint16_t* weight, int32_t d_model, int32_t vocab,
                                                   const int32_t* clean_ids, const uint8_t* corrupted,
                                                   const float* p, int32_t align, float grad_scale,
                                                   float* loss, float* unit_loss, uint16_t* d_hidden,
                                                   uint16_t* d_weight, void* workspace, size_t workspace_bytes,
                                                   dlm_stream_t stream) {
    DLM_NVTX("dlm_linear_loss_fwd_bwd_ex");
    return linear_loss_fwd_bwd(layout, hidden, weight, d_model, vocab, clean_ids, corrupted, p, DLM_ABSORBING,
                               align, nullptr, nullptr, nullptr, 0.f, grad_scale, loss, unit_loss, d_hidden,
                               nullptr, d_weight, workspace, workspace_bytes, stream);
}

extern "C" dlm_status_t dlm_linear_loss_uniform_fwd_bwd(const dlm_layout_t* layout, const uint16_t* hidden,
                                                        const dlm_layout_t* enc_layout, const uint16_t* enc_hidden,
                                                        const int32_t* enc_ids, const uint16_t* weight,
                                                        int32_t d_model, int32_t vocab, const int32_t* clean_ids,
                                                        int32_t align, float enc_ar_weight, float grad_scale,
                                                        float* loss, float* unit_loss, uint16_t* d_hidden,
                                                        uint16_t* d_enc_hidden, uint16_t* d_weight,
                                                        void* workspace, size_t workspace_bytes,
                                                        dlm_stream_t stream) {
    DLM_NVTX("dlm_linear_loss_uniform_fwd_bwd");
    return linear_loss_fwd_bwd(layout, hidden, weight, d_model, vocab, clean_ids, nullptr, nullptr, DLM_UNIFORM,
                               align, enc_layout, enc_hidden, enc_ids, enc_ar_weight, grad_scale, loss,
                               unit_loss, d_hidden, d_enc_hidden, d_weight, workspace, workspace_bytes, stream);
}
