// decode_mla.cuh -- MLA absorbed-latent decode (the MQA form of multi-head
// latent attention) for sm_100a.
//
// Every query head reads the same latent cache row c_j (576 wide: the 512
// compressed values followed by the 64-wide decoupled RoPE key): the score of
// head h is s = <q_h, c_j> * scale over all 576 columns, and its value is the
// first 512 columns of the same row ("Attention Engineering: From MHA to GQA,
// MLA & FlashAttention", section 3, complete MLA attention score with the
// absorbed content term and the shared RoPE term; "Attention, Worked Out by
// Hand (Part 2)", section 3).
//
// One query token per sequence, 128 heads = one MMA M tile. The fp32 output
// of 128 heads x 512 values alone fills the 512 TMEM columns of an SM, so a
// sequence is handled by two CTAs (a cluster of two, so that they run at
// the same time and the second read of each cache tile hits L2):
//   * both CTAs compute the full score tile S = Q K^T (128 heads x 64 keys)
//     with tcgen05 MMAs: Q columns 256-575 sit in shared memory, Q columns
//     0-255 in TMEM as the A operand of a TMEM-sourced MMA (shared memory
//     holds Q's other part and a 2-stage ring of 64-key cache tiles);
//   * both run the same online softmax on the same scores (the MMAs are the
//     same instructions in the same order, so both CTAs hold identical S, P,
//     m and l);
//   * CTA r accumulates its half of the output, O[:, 256r .. 256r+255] +=
//     P V, V being the first 512 columns of the very tile it loaded.
// The score MMAs are done twice (1.5x the algorithmic FLOPs in all); in
// exchange the two SMs never wait on each other. TMA loads are plain (no
// multicast).
// Split-KV (the decode against the cache of "Attention deep dive", section 5,
// cut across SMs): a batch too small to occupy every SM by whole sequences
// has each sequence's keys cut into chunks, one cluster per chunk; each
// cluster then writes its unnormalised partial output and (m, l) to the
// workspace, and the merge kernel of the GQA decode combines the chunks by
// their log-sum-exp weights (the section 4 recurrence of "Attention
// Engineering" across chunks). A batch that fills the SMs keeps one chunk per
// sequence and writes O and LSE directly.
#pragma once

#include "sm100.cuh"

namespace attn {
namespace mla {

constexpr int M = 128;            // heads per CTA tile
constexpr int KT = 64;            // keys per tile (MMA N of Q K^T)
constexpr int DL = 576;           // latent row: key width
constexpr int DV = 512;           // value width (first 512 columns of the row)
constexpr int NB = 9;             // 64-column boxes of a latent row
constexpr int NBT = 4;            // Q boxes 0-3 (columns 0-255) in TMEM
constexpr int NBS = NB - NBT;     // Q boxes 4-8 (columns 256-575) in shared memory
constexpr int QBOX = M * 128;     // one 64-column box of Q: 128 rows x 128 B
constexpr int KBOX = KT * 128;    // one 64-column box of a key tile: 64 rows x 128 B
constexpr int NSTAGE = 2;
// A ring stage is filled in two groups with their own barriers: group A, the
// boxes only the score MMAs read (for CTA r: the five boxes outside its value
// columns 256r .. 256r+255), freed once the tile's score MMAs complete, and
// group B, its four value boxes 4r .. 4r+3, freed once the tile's P.V
// completes. Group A of tile j+2 so loads while tile j's softmax and P.V run.
constexpr int NA = 5, NBV = 4;    // boxes of group A and of group B
constexpr int THREADS = 256;      // warp 0 TMA (group A), warps 1-2 MMAs (even / odd tiles), warp 3 TMA
                                  // (group B), warps 4-7 softmax
constexpr float kRescaleThreshold = 8.0f;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_S0 = 0, COL_S1 = 64;   // S double buffer (P over its first half)
constexpr uint32_t COL_QT = 128;              // Q columns 0-255 as bf16 pairs (128 columns)
constexpr uint32_t COL_O = 256;               // this CTA's half of O (256 columns)

struct Smem {
    uint8_t q[NBS][QBOX];                  // 80 KB
    uint8_t k[NSTAGE][NB][KBOX];           // 144 KB; stage 1 first stages Q boxes 0-3
    uint64_t q_full;
    uint64_t kv_full[NSTAGE][2], kv_empty[NSTAGE][2];   // [stage][group A, group B]
    uint64_t s_full[2], p_full[2];
    uint64_t s_done[2];                    // every MMA of issuing thread t has completed
    uint64_t qt_ready;                     // Q columns 0-255 copied into TMEM
    uint64_t pv_done[2];                   // P.V of tile k done: barrier k & 1, phase k >> 1
    uint64_t o_done;
    uint64_t tail_ready;                   // value rows past the length cleared (last tile)
    uint32_t tmem_base;
    int abort_flag;
};

constexpr size_t smem_bytes() { return sizeof(Smem) + 1024; }
static_assert(smem_bytes() <= kMaxSmemPerCta, "MLA decode shared memory exceeds a CTA's");

struct Params {
    int B, n_q, S_max;
    const int32_t *seqlens;
    __nv_bfloat16 *o;      // [B, n_q, 512]
    float *lse;            // [B, n_q] or null
    float scale_log2;
    // Split-KV: cluster c takes keys [s * ch, (s + 1) * ch) of sequence
    // c / n_splits, s = c % n_splits. With one split the cluster writes O and
    // LSE; with more it writes its unnormalised partial output o_s (fp32,
    // [B, n_q, n_splits, 512]) and (m_s, l_s) ([B, n_q, n_splits], log2
    // units) for the merge kernel.
    int n_splits, ch;
    float *ws_o;
    float2 *ws_ml;
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__global__ void __launch_bounds__(THREADS, 1)
mla_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_c,
                  const Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t warp = warp_id(), lane = lane_id();
    const uint32_t rank = cluster_rank();            // which half of the output
    const int b = (int)(blockIdx.x / 2) / p.n_splits;
    const int split = (int)(blockIdx.x / 2) % p.n_splits;
    const int hb = blockIdx.y;                        // block of 128 heads
    int seqlen = p.seqlens[b];
    if (seqlen > p.S_max) {
        if (threadIdx.x == 0 && rank == 0 && hb == 0 && split == 0) atomicOr(&g_status, kStatusRange);
        seqlen = p.S_max;
    }
    if (seqlen < 0) seqlen = 0;
    // this cluster's keys: key0 .. key0 + nkeys - 1 of the sequence
    const int key0 = split * p.ch;
    const int nkeys = max(0, min(p.ch, seqlen - key0));
    const int nt = (nkeys + KT - 1) / KT;
    const int tail = nt > 0 ? nkeys - (nt - 1) * KT : KT;   // valid rows of the last tile

    if (warp == 0 && lane == 0) {
        mbar_init(smem_u32(&sm.q_full), 1);
        for (int s = 0; s < NSTAGE; ++s) {
            for (int g = 0; g < 2; ++g) {
                mbar_init(smem_u32(&sm.kv_full[s][g]), 1);
                mbar_init(smem_u32(&sm.kv_empty[s][g]), 1);
            }
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&sm.s_full[i]), 1);
            mbar_init(smem_u32(&sm.p_full[i]), 128);
        }
        mbar_init(smem_u32(&sm.qt_ready), 128);
        mbar_init(smem_u32(&sm.pv_done[0]), 1);
        mbar_init(smem_u32(&sm.pv_done[1]), 1);
        mbar_init(smem_u32(&sm.o_done), 1);
        mbar_init(smem_u32(&sm.s_done[0]), 1);
        mbar_init(smem_u32(&sm.s_done[1]), 1);
        mbar_init(smem_u32(&sm.tail_ready), 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&sm.tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort_flag = &sm.abort_flag;

    // box bx of a 576-column row belongs to group B of this CTA iff it is one
    // of its value boxes
    auto box_of = [rank](int g, int i) -> int {
        // group A: the other CTA's value boxes, then box 8; group B: own value boxes
        return g == 0 ? (i < NBV ? 4 * (1 - (int)rank) + i : 8) : 4 * (int)rank + i;
    };
    if (warp == 0 || warp == 3) {
        // ============ TMA producers: warp 0 group A (and Q), warp 3 group B ============
        const int g = warp == 0 ? 0 : 1;
        const int nbox = g == 0 ? NA : NBV;
        if (lane == 0 && nt > 0) {
            tma_prefetch_desc(&tm_c);
            const uint32_t qbar = smem_u32(&sm.q_full);
            if (g == 0) {
                tma_prefetch_desc(&tm_q);
                // Q: boxes 4-8 to their home, boxes 0-3 staged in ring stage 1
                mbar_arrive_expect_tx(qbar, (uint32_t)(NB * QBOX));
                for (int bx = 0; bx < NB; ++bx) {
                    const uint32_t dst = bx < NBT ? smem_u32(sm.k[1][0]) + bx * QBOX : smem_u32(sm.q[bx - NBT]);
                    tma_load_3d(dst, &tm_q, qbar, 64 * bx, hb * M, b);
                }
            }
            bool ok = true;
            int issued = 0;
            for (int j = 0; ok && j < nt; ++j) {
                const int s = j % NSTAGE;
                // Q boxes 0-3 (4 x 16 KB) are staged over boxes 0-7 of stage 1
                if (j == 1) ok = mbar_wait(smem_u32(&sm.qt_ready), 0, abort_flag, 0x410);
                if (ok && j >= NSTAGE)
                    ok = mbar_wait(smem_u32(&sm.kv_empty[s][g]), ((j / NSTAGE) + 1) & 1, abort_flag, 0x411);
                if (!ok) break;
                const uint32_t fb = smem_u32(&sm.kv_full[s][g]);
                mbar_arrive_expect_tx(fb, (uint32_t)(nbox * KBOX));
                for (int i = 0; i < nbox; ++i) {
                    const int bx = box_of(g, i);
                    tma_load_3d(smem_u32(sm.k[s][bx]), &tm_c, fb, 64 * bx, key0 + j * KT, b);
                }
                ++issued;
            }
            if (g == 0) mbar_wait(qbar, 0, nullptr, 0x412);
            for (int j = issued - 1; j >= 0 && j >= issued - NSTAGE; --j)
                mbar_wait(smem_u32(&sm.kv_full[j % NSTAGE][g]), (j / NSTAGE) & 1, nullptr, 0x413);
        }
        __syncwarp();
        if (g == 1 && tail < KT) {
            // Rows past the length get weight 0, but 0 * (NaN or Inf) is not
            // 0: clear this CTA's value columns of those rows so that whatever
            // the cache holds there cannot reach the output. Done before the
            // last tile's group-B score MMAs are issued (they wait for tail_ready).
            const int s = (nt - 1) % NSTAGE;
            bool ok = mbar_wait(smem_u32(&sm.kv_full[s][1]), ((nt - 1) / NSTAGE) & 1, abort_flag, 0x414);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                for (int e = tail * 8 + (int)lane; e < KT * 8; e += 32) {
                    const uint32_t off = (uint32_t)(e >> 3) * 128u + (uint32_t)(e & 7) * 16u;
#pragma unroll
                    for (int bx = 0; bx < 4; ++bx)
                        sts128(smem_u32(sm.k[s][4 * rank + bx]) + off, make_uint4(0u, 0u, 0u, 0u));
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sm.tail_ready));
        }
    } else if (warp == 1 || warp == 2) {
        // ======================= MMA issue =======================
        // Two threads, one per S buffer: warp 1 takes the even tiles (S buffer
        // 0, ring stage 0), warp 2 the odd ones. Each issues its tile's 36
        // score MMAs, then, once the softmax has written P, the tile's P.V;
        // in one thread's program order the next score MMAs into the same S
        // buffer follow that P.V. The P.V MMAs of both threads accumulate
        // into the same O, so each waits for the previous tile's P.V to
        // complete: pv_done[k & 1], committed only by the thread of tile k,
        // phase k >> 1. A thread at tile j has itself waited for the phase of
        // tile j - 3 on the other barrier, so the phase it waits for next
        // cannot be confused with an older one of the same parity.
        const int par = (int)warp - 1;
        if (lane == 0 && nt > par) {
            const uint32_t idesc_s = umma_idesc_bf16(M, KT, 0, 0);
            const uint32_t idesc_o = umma_idesc_bf16(M, 256, 0, 1);
            bool ok = mbar_wait(smem_u32(&sm.q_full), 0, abort_flag, 0x421) &&
                      mbar_wait(smem_u32(&sm.qt_ready), 0, abort_flag, 0x425);
            const uint64_t qd0 = umma_smem_desc(smem_u32(sm.q[0]), 16, 1024, 2);
            const uint32_t dcol = tmem + (par ? COL_S1 : COL_S0);
            for (int j = par; ok && j < nt; j += 2) {
                const int s = j % NSTAGE;   // == par
                const uint32_t ph = (uint32_t)(j / NSTAGE) & 1u;
                ok = mbar_wait(smem_u32(&sm.kv_full[s][0]), ph, abort_flag, 0x422);
                if (!ok) break;
                tc_fence_after();
                // the 36 score MMAs fully unrolled, each descriptor the tile's (or
                // Q's) base descriptor plus a constant offset in its 16-byte
                // address field (at N = 64 an MMA finishes in fewer cycles than
                // a loop iteration of the issuing thread would take): group A's
                // boxes first, then, once they have landed, group B's. The two
                // CTAs add the nine boxes in different orders, so their scores
                // may differ in the last bits; each normalises its own half of
                // O by its own sums, and the LSE is the first CTA's.
                const uint64_t kd0 = umma_smem_desc(smem_u32(sm.k[s][0]), 16, 1024, 2);
                auto score_box = [&](int bx, bool first) {
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        if (bx < NBT)
                            umma_ts(dcol, tmem + COL_QT + 32 * bx + 8 * k4, kd0 + (uint64_t)((bx * KBOX + 32 * k4) >> 4),
                                    idesc_s, (first && k4 == 0) ? 0u : 1u);
                        else
                            umma_ss(dcol, qd0 + (uint64_t)(((bx - NBT) * QBOX + 32 * k4) >> 4),
                                    kd0 + (uint64_t)((bx * KBOX + 32 * k4) >> 4), idesc_s, (first && k4 == 0) ? 0u : 1u);
                    }
                };
                // group B landed (and, on the last tile, its rows past the
                // length cleared: the clearing writes those boxes)
                auto group_b = [&]() -> bool {
                    if (!mbar_wait(smem_u32(&sm.kv_full[s][1]), ph, abort_flag, 0x429)) return false;
                    if (j == nt - 1 && tail < KT && !mbar_wait(smem_u32(&sm.tail_ready), 0, abort_flag, 0x426))
                        return false;
                    tc_fence_after();
                    return true;
                };
                if (rank == 0) {
#pragma unroll
                    for (int bx = 4; bx < 9; ++bx) score_box(bx, bx == 4);
                    ok = group_b();
                    if (!ok) break;
#pragma unroll
                    for (int bx = 0; bx < 4; ++bx) score_box(bx, false);
                } else {
#pragma unroll
                    for (int bx = 0; bx < 4; ++bx) score_box(bx, bx == 0);
                    score_box(8, false);
                    ok = group_b();
                    if (!ok) break;
#pragma unroll
                    for (int bx = 4; bx < 8; ++bx) score_box(bx, false);
                }
                // group A of this stage is free once these MMAs complete
                umma_commit(smem_u32(&sm.kv_empty[s][0]));
                umma_commit(smem_u32(&sm.s_full[j & 1]));
                // O_r += P(j) V_j, V = this CTA's 256 columns of the tile, after
                // the P.V of tile j - 1 (the other thread's) has completed
                ok = mbar_wait(smem_u32(&sm.p_full[j & 1]), (j >> 1) & 1, abort_flag, 0x423);
                if (ok && j > 0) ok = mbar_wait(smem_u32(&sm.pv_done[par ^ 1]), ((j - 1) >> 1) & 1, abort_flag, 0x427);
                if (!ok) break;
                tc_fence_after();
                const uint64_t vd0 = umma_smem_desc(smem_u32(sm.k[s][4 * rank]), KBOX, 1024, 2);
#pragma unroll
                for (int ks = 0; ks < KT / 16; ++ks)
                    umma_ts(tmem + COL_O, dcol + ks * 8, vd0 + (uint64_t)((ks * 16 * 128) >> 4), idesc_o,
                            (j > 0 || ks > 0) ? 1u : 0u);
                umma_commit(smem_u32(&sm.kv_empty[s][1]));
                umma_commit(smem_u32(&sm.pv_done[par]));
                if (j == nt - 1) umma_commit(smem_u32(&sm.o_done));   // O final (tile nt-2's P.V already done)
            }
            // no MMA of this thread may still run when TMEM is released
            umma_commit(smem_u32(&sm.s_done[par]));
            mbar_wait(smem_u32(&sm.s_done[par]), 0, nullptr, 0x428);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ====================== softmax + epilogue ======================
        const uint32_t quad = warp & 3u;
        const int r = (int)(quad * 32 + lane);                  // head row = TMEM lane
        const uint32_t trow = tmem + ((quad * 32u) << 16);
        const float sl = p.scale_log2;
        const float2 sl2 = make_float2(sl, sl);
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        if (nt > 0) {
            // Q columns 0-255 (staged by TMA as four swizzled 128-row boxes in
            // ring stage 1) into TMEM, one row per thread
            ok = mbar_wait(smem_u32(&sm.q_full), 0, abort_flag, 0x436);
            ok = __all_sync(0xffffffffu, ok);
            const uint32_t stage = smem_u32(sm.k[1][0]);
#pragma unroll 1
            for (int bx = 0; bx < NBT; ++bx) {
                uint32_t qr[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 w = lds128(stage + bx * QBOX + swz<3>((uint32_t)(r * 128 + c * 16)));
                    qr[4 * c] = w.x;
                    qr[4 * c + 1] = w.y;
                    qr[4 * c + 2] = w.z;
                    qr[4 * c + 3] = w.w;
                }
                tmem_st32(trow + COL_QT + 32 * bx, qr);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(smem_u32(&sm.qt_ready));
        }
        for (int j = 0; ok && j < nt; ++j) {
            const uint32_t colS = (j & 1) ? COL_S1 : COL_S0;
            ok = mbar_wait(smem_u32(&sm.s_full[j & 1]), (j >> 1) & 1, abort_flag, 0x431);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            __syncwarp();
            tc_fence_after();
            uint32_t x[KT];
            tmem_ld32(trow + colS, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
            tmem_ld32(trow + colS + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
            tmem_wait_ld();
            // keys beyond the sequence length (last tile only)
            const int rem = nkeys - 1 - j * KT;
            if (rem < KT - 1) {
#pragma unroll
                for (int e = 0; e < KT; ++e)
                    if (e > rem) x[e] = 0xff800000u;   // -inf
            }
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int e = 0; e < KT; e += 4) {
                mx0 = fmax3(mx0, __uint_as_float(x[e]), __uint_as_float(x[e + 1]));
                mx1 = fmax3(mx1, __uint_as_float(x[e + 2]), __uint_as_float(x[e + 3]));
            }
            const float m_new = fmaxf(m_run, fmaxf(mx0, mx1) * sl);
            if (j == 0) {
                m_run = m_new;
            } else if (__any_sync(0xffffffffu, m_new > m_run + kRescaleThreshold)) {
                // O must be stable: wait for the P.V of tile j-1 (barrier
                // (j-1) & 1, phase (j-1) >> 1; the P.V of tile j-2 came before
                // the score MMAs of tile j in the same thread, and that of
                // tile j-3 was waited for by the P.V of tile j-2). The P.V of
                // tile j starts only after p_full below.
                ok = mbar_wait(smem_u32(&sm.pv_done[(j - 1) & 1]), ((j - 1) >> 1) & 1, abort_flag, 0x435);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                __syncwarp();
                tc_fence_after();
                const float alpha = ex2(m_run - m_new);
#pragma unroll 1
                for (int c = 0; c < 256 / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(trow + COL_O + 32 * c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(trow + COL_O + 32 * c, o);
                }
                tmem_wait_st();
                l_run *= alpha;
                m_run = m_new;
            }
            const float2 nm2 = make_float2(-m_run, -m_run);
            float2 rs = make_float2(0.f, 0.f);
            uint32_t pk[KT / 2];
#pragma unroll
            for (int e = 0; e < KT / 2; ++e) {
                const float2 t2 =
                    ffma2(make_float2(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1])), sl2, nm2);
                const float2 pe = make_float2(ex2(t2.x), ex2(t2.y));
                rs = fadd2(rs, pe);
                pk[e] = f2_to_bf2(pe.x, pe.y);
            }
            tmem_st32(trow + colS, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(smem_u32(&sm.p_full[j & 1]));
            l_run += rs.x + rs.y;
        }
        // ---- epilogue: this CTA's 256 output columns, O / l -> bf16; LSE (rank 0)
        if (nt > 0 && ok) ok = mbar_wait(smem_u32(&sm.o_done), 0, abort_flag, 0x434);
        ok = __all_sync(0xffffffffu, ok);
        __syncwarp();
        tc_fence_after();
        const int head = hb * M + r;
        // Each thread owns one head row of 256 output columns. Writing it
        // straight from registers sends each warp store to 32 rows; instead the
        // row goes to the idle ring (all of its reads completed before o_done)
        // at a 16-byte-padded stride, so that a quarter warp's 16-byte stores
        // fall on distinct banks, and one bulk copy per row moves it out.
        const uint32_t stage = smem_u32(&sm.k[0][0][0]);
        if (p.n_splits > 1) {
            // partial output of this chunk for the merge kernel: unnormalised O
            // (this CTA's 256 columns) and, from rank 0, (m, l); a chunk with
            // no key writes nothing (the merge reads only the chunks below the
            // sequence's length)
            if (nt > 0) {
                constexpr uint32_t ROW = 256 * 4 + 16;
                const uint32_t srow = stage + r * ROW;
#pragma unroll 1
                for (int c = 0; c < 256 / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(trow + COL_O + 32 * c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4)
                        sts128(srow + 128 * c + 16 * q4, make_uint4(o[4 * q4], o[4 * q4 + 1], o[4 * q4 + 2], o[4 * q4 + 3]));
                }
                if (head < p.n_q) {
                    const size_t prow = ((size_t)b * p.n_q + head) * p.n_splits + split;
                    fence_proxy_async_smem();
                    bulk_store(p.ws_o + prow * DV + 256 * rank, srow, 256 * 4);
                    tma_store_commit();
                    if (rank == 0) p.ws_ml[prow] = make_float2(m_run, l_run);
                    tma_store_wait_read0();
                }
            }
        } else {
            if (head < p.n_q && nt == 0) {
                uint4 *orow = reinterpret_cast<uint4 *>(p.o + ((size_t)b * p.n_q + head) * DV + 256 * rank);
                for (int c = 0; c < 256 / 8; ++c) orow[c] = make_uint4(0, 0, 0, 0);
            }
            if (nt > 0) {
                constexpr uint32_t ROW = 256 * 2 + 16;
                const uint32_t srow = stage + r * ROW;
                const float inv_l = 1.f / l_run;
#pragma unroll 1
                for (int c = 0; c < 256 / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(trow + COL_O + 32 * c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            w[e] = f2_to_bf2(__uint_as_float(o[8 * q8 + 2 * e]) * inv_l,
                                             __uint_as_float(o[8 * q8 + 2 * e + 1]) * inv_l);
                        sts128(srow + 64 * c + 16 * q8, make_uint4(w[0], w[1], w[2], w[3]));
                    }
                }
                if (head < p.n_q) {
                    // the entry point requires a 16-byte-aligned output
                    fence_proxy_async_smem();
                    bulk_store(p.o + ((size_t)b * p.n_q + head) * DV + 256 * rank, srow, 256 * 2);
                    tma_store_commit();
                    tma_store_wait_read0();
                }
            }
            if (rank == 0 && head < p.n_q && p.lse != nullptr)
                p.lse[(size_t)b * p.n_q + head] = nt > 0 ? (m_run + log2f(l_run)) * 0.6931471805599453f : -INFINITY;
        }
    }

    // ---- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace mla
}  // namespace attn
