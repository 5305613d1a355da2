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
// sequence is handled by a cluster of two CTAs (two SMs):
//   * CTA r computes the partial scores over its part of the latent columns
//     (r = 0: columns 0-255, r = 1: columns 256-575) with tcgen05 MMAs
//     (Q part resident on chip: columns 0-511 in shared memory, the 64 RoPE
//     columns of CTA 1 in TMEM as the A operand of a TMEM-sourced MMA, which
//     leaves room for a 3-stage cache ring and the fp32 exchange buffer;
//     64-key cache tiles streamed by TMA),
//   * the two CTAs exchange their partial scores through distributed shared
//     memory (fp32, one 64-key row per thread) and both form the same full
//     score row, s = s_0 + s_1, and run the same online softmax,
//   * CTA r accumulates its half of the output, O[:, 256r .. 256r+255] +=
//     P V, where V is the first 512 columns of the very tile it loaded.
// Each cache row is read from HBM once (CTA 0 reads 512 B, CTA 1 640 B) and no
// arithmetic is duplicated except the (cheap) softmax. TMA loads are plain
// (no multicast); cluster barriers are only used at start and end.
#pragma once

#include "sm100.cuh"

namespace attn {
namespace mla {

constexpr int M = 128;            // heads per CTA tile
constexpr int KT = 64;            // keys per tile (MMA N of Q K^T)
constexpr int DL = 576;           // latent row: key width
constexpr int DV = 512;           // value width (first 512 columns of the row)
constexpr int NBMAX = 5;          // 64-column boxes of the larger part (CTA 1: 256..575)
constexpr int NBQ = 4;            // Q boxes kept in shared memory (CTA 1's fifth lives in TMEM)
constexpr int QBOX = M * 128;     // one 64-column box of Q: 128 rows x 128 B
constexpr int KBOX = KT * 128;    // one 64-column box of a key tile: 64 rows x 128 B
constexpr int NSTAGE = 3;
constexpr int XSTRIDE = 272;      // bytes per exchanged row: 64 fp32 + 16 pad (bank spread)
constexpr int THREADS = 256;      // warp 0 TMA, warp 1 MMA, warps 4-7 softmax
constexpr float kRescaleThreshold = 8.0f;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_S0 = 0, COL_S1 = 64, COL_O = 256;   // S double buffer, O half
constexpr uint32_t COL_QR = 128;  // CTA 1: Q columns 512-575 as bf16 pairs (32 columns)

struct Smem {
    uint8_t q[NBQ][QBOX];                  // 64 KB
    uint8_t k[NSTAGE][NBMAX][KBOX];        // 120 KB
    uint8_t xbuf[M][XSTRIDE];              // partner's partial scores (fp32); first
                                           // stages CTA 1's RoPE columns of Q
    uint64_t q_full;
    uint64_t kv_full[NSTAGE], kv_empty[NSTAGE];
    uint64_t s_full[2], p_full[2];
    uint64_t xfull;                        // partner wrote its partial into xbuf
    uint64_t xfree;                        // my partial may be written into the partner's xbuf
    uint64_t qr_ready;                     // CTA 1: RoPE columns of Q copied into TMEM
    uint64_t pv_done;                      // one phase per P.V MMA group
    uint64_t o_done;
    uint32_t tmem_base;
    int abort_flag;
};

constexpr size_t smem_bytes() { return sizeof(Smem) + 1024; }

struct Params {
    int B, n_q, S_max;
    const int32_t *seqlens;
    __nv_bfloat16 *o;      // [B, n_q, 512]
    float *lse;            // [B, n_q] or null
    float scale_log2;
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait on a barrier that the partner CTA arrives on.
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                                  uint32_t site) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait_cluster(bar, parity)) return true;
        if (abort_flag != nullptr && *abort_flag) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_status, kStatusTimeout);
            atomicCAS(&g_timeout_site, 0u, site);
            if (abort_flag != nullptr) *abort_flag = 1;
            return false;
        }
    }
}

__global__ void __launch_bounds__(THREADS, 1)
mla_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_c,
                  const Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t warp = warp_id(), lane = lane_id();
    const uint32_t rank = cluster_rank();            // 0 or 1
    const int b = blockIdx.x / 2;
    const int hb = blockIdx.y;                        // block of 128 heads
    const int nb = 4 + (int)rank;                     // 64-column boxes of this CTA's part
    const int col0 = 256 * (int)rank;                 // first latent column of this CTA's part
    int nkeys = p.seqlens[b];
    if (nkeys > p.S_max) {
        if (threadIdx.x == 0 && rank == 0 && hb == 0) atomicOr(&g_status, kStatusRange);
        nkeys = p.S_max;
    }
    if (nkeys < 0) nkeys = 0;
    const int nt = (nkeys + KT - 1) / KT;

    if (warp == 0 && lane == 0) {
        mbar_init(smem_u32(&sm.q_full), 1);
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(smem_u32(&sm.kv_full[s]), 1);
            mbar_init(smem_u32(&sm.kv_empty[s]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&sm.s_full[i]), 1);
            mbar_init(smem_u32(&sm.p_full[i]), 128);
        }
        mbar_init(smem_u32(&sm.xfull), 4);    // one arrival per partner softmax warp
        mbar_init(smem_u32(&sm.xfree), 4);
        mbar_init(smem_u32(&sm.pv_done), 1);
        mbar_init(smem_u32(&sm.qr_ready), 128);
        mbar_init(smem_u32(&sm.o_done), 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&sm.tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    // both CTAs' barriers exist before either arrives remotely
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort_flag = &sm.abort_flag;

    if (warp == 0) {
        // ======================= TMA producer =======================
        if (lane == 0 && nt > 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_c);
            const uint32_t qbar = smem_u32(&sm.q_full);
            mbar_arrive_expect_tx(qbar, (uint32_t)(nb * QBOX));
            for (int bx = 0; bx < nb; ++bx) {
                const uint32_t dst = bx < NBQ ? smem_u32(sm.q[bx]) : smem_u32(&sm.xbuf[0][0]);
                tma_load_3d(dst, &tm_q, qbar, col0 + 64 * bx, hb * M, b);
            }
            int issued = 0;
            for (int j = 0; j < nt; ++j) {
                const int s = j % NSTAGE;
                if (j >= NSTAGE &&
                    !mbar_wait(smem_u32(&sm.kv_empty[s]), ((j / NSTAGE) + 1) & 1, abort_flag, 0x411))
                    break;
                const uint32_t fb = smem_u32(&sm.kv_full[s]);
                mbar_arrive_expect_tx(fb, (uint32_t)(nb * KBOX));
                for (int bx = 0; bx < nb; ++bx)
                    tma_load_3d(smem_u32(sm.k[s][bx]), &tm_c, fb, col0 + 64 * bx, j * KT, b);
                ++issued;
            }
            mbar_wait(qbar, 0, nullptr, 0x412);
            for (int j = issued - 1; j >= 0 && j >= issued - NSTAGE; --j)
                mbar_wait(smem_u32(&sm.kv_full[j % NSTAGE]), (j / NSTAGE) & 1, nullptr, 0x413);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ======================= MMA issuer =======================
        if (lane == 0 && nt > 0) {
            const uint32_t idesc_s = umma_idesc_bf16(M, KT, 0, 0);
            const uint32_t idesc_o = umma_idesc_bf16(M, 256, 0, 1);
            bool ok = mbar_wait(smem_u32(&sm.q_full), 0, abort_flag, 0x421);
            if (ok && nb > NBQ) {
                ok = mbar_wait(smem_u32(&sm.qr_ready), 0, abort_flag, 0x425);
                tc_fence_after();
            }
            auto issue_s = [&](int j) -> bool {
                const int s = j % NSTAGE;
                if (!mbar_wait(smem_u32(&sm.kv_full[s]), (j / NSTAGE) & 1, abort_flag, 0x422)) return false;
                tc_fence_after();
                const uint32_t dcol = tmem + ((j & 1) ? COL_S1 : COL_S0);
#pragma unroll 1
                for (int bx = 0; bx < NBQ; ++bx) {
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const uint64_t ad = umma_smem_desc(smem_u32(sm.q[bx]) + 32 * k4, 16, 1024, 2);
                        const uint64_t bd = umma_smem_desc(smem_u32(sm.k[s][bx]) + 32 * k4, 16, 1024, 2);
                        umma_ss(dcol, ad, bd, idesc_s, (bx > 0 || k4 > 0) ? 1u : 0u);
                    }
                }
                if (nb > NBQ) {   // RoPE columns: A operand from TMEM
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const uint64_t bd = umma_smem_desc(smem_u32(sm.k[s][NBQ]) + 32 * k4, 16, 1024, 2);
                        umma_ts(dcol, tmem + COL_QR + 8 * k4, bd, idesc_s, 1u);
                    }
                }
                umma_commit(smem_u32(&sm.s_full[j & 1]));
                return true;
            };
            auto issue_pv = [&](int i) -> bool {
                const int s = i % NSTAGE;
                if (!mbar_wait(smem_u32(&sm.p_full[i & 1]), (i >> 1) & 1, abort_flag, 0x423)) return false;
                tc_fence_after();
                const uint32_t pcol = tmem + ((i & 1) ? COL_S1 : COL_S0);
                // V = columns 256r .. 256r+255 of the row = this CTA's boxes 0-3
#pragma unroll
                for (int ks = 0; ks < KT / 16; ++ks) {
                    const uint64_t bd = umma_smem_desc(smem_u32(sm.k[s][0]) + ks * 16 * 128, KBOX, 1024, 2);
                    umma_ts(tmem + COL_O, pcol + ks * 8, bd, idesc_o, (i > 0 || ks > 0) ? 1u : 0u);
                }
                umma_commit(smem_u32(&sm.kv_empty[s]));
                umma_commit(smem_u32(&sm.pv_done));
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int j = 1; ok && j < nt; ++j) {
                ok = issue_s(j);
                if (ok) ok = issue_pv(j - 1);
            }
            if (ok) ok = issue_pv(nt - 1);
            umma_commit(smem_u32(&sm.o_done));
            mbar_wait(smem_u32(&sm.o_done), 0, nullptr, 0x424);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // =============== score exchange + softmax + epilogue ===============
        const uint32_t quad = warp & 3u;
        const int r = (int)(quad * 32 + lane);                  // head row = TMEM lane
        const uint32_t trow = tmem + ((quad * 32u) << 16);
        const uint32_t partner = rank ^ 1u;
        const uint32_t my_row = smem_u32(&sm.xbuf[r][0]);
        const uint32_t peer_row = map_to_rank(my_row, partner);
        const uint32_t peer_xfull = map_to_rank(smem_u32(&sm.xfull), partner);
        const uint32_t peer_xfree = map_to_rank(smem_u32(&sm.xfree), partner);
        const float sl = p.scale_log2;
        const float2 sl2 = make_float2(sl, sl);
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        if (nt > 0 && nb > NBQ) {
            // CTA 1: move the RoPE columns of Q (staged by TMA in xbuf as one
            // swizzled 128-row box) into TMEM, one row per thread
            ok = mbar_wait(smem_u32(&sm.q_full), 0, abort_flag, 0x436);
            ok = __all_sync(0xffffffffu, ok);
            uint32_t qr[32];
            const uint32_t stage = smem_u32(&sm.xbuf[0][0]);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 w = lds128(stage + swz<3>((uint32_t)(r * 128 + c * 16)));
                qr[4 * c] = w.x;
                qr[4 * c + 1] = w.y;
                qr[4 * c + 2] = w.z;
                qr[4 * c + 3] = w.w;
            }
            tmem_st32(trow + COL_QR, qr);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(smem_u32(&sm.qr_ready));
        }
        // my xbuf is free: the partner may write its first partial
        // (one release arrival per warp after the warp's threads synchronise:
        // the release is cumulative over the stores the lanes made before it)
        __syncwarp();
        if (nt > 0 && lane == 0) mbar_arrive_remote(peer_xfree);
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
            // my partial scores, sent to the partner (fp32)
            ok = mbar_wait_cluster(smem_u32(&sm.xfree), j & 1, abort_flag, 0x432);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
#pragma unroll
            for (int c = 0; c < KT / 4; ++c)   // 16 bytes = 4 scores per store
                st_cluster_v4(peer_row + 16 * c, make_uint4(x[4 * c], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3]));
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(peer_xfull);
            ok = mbar_wait_cluster(smem_u32(&sm.xfull), j & 1, abort_flag, 0x433);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            // full scores, identical on both CTAs: s_0 + s_1 in that order
            float s[KT];
#pragma unroll
            for (int c = 0; c < KT / 4; ++c) {
                const uint4 w = lds128(my_row + 16 * c);
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float own = __uint_as_float(x[4 * c + e]), peer = __uint_as_float(ws[e]);
                    s[4 * c + e] = rank == 0 ? own + peer : peer + own;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(peer_xfree);   // the partner may overwrite my xbuf
            // keys beyond the sequence length (last tile only)
            const int rem = nkeys - 1 - j * KT;
            if (rem < KT - 1) {
#pragma unroll
                for (int e = 0; e < KT; ++e)
                    if (e > rem) s[e] = -INFINITY;
            }
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int e = 0; e < KT; e += 4) {
                mx0 = fmax3(mx0, s[e], s[e + 1]);
                mx1 = fmax3(mx1, s[e + 2], s[e + 3]);
            }
            const float m_new = fmaxf(m_run, fmaxf(mx0, mx1) * sl);
            if (j == 0) {
                m_run = m_new;
            } else if (__any_sync(0xffffffffu, m_new > m_run + kRescaleThreshold)) {
                // The Q.K MMA of tile j is issued before the P.V of tile j-1, so
                // wait for that P.V (phase j-1 of pv_done) before touching O; the
                // P.V of tile j starts only after p_full below.
                ok = mbar_wait(smem_u32(&sm.pv_done), (j - 1) & 1, abort_flag, 0x435);
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
                const float2 t2 = ffma2(make_float2(s[2 * e], s[2 * e + 1]), sl2, nm2);
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
        if (head < p.n_q) {
            __nv_bfloat16 *orow = p.o + ((size_t)b * p.n_q + head) * DV + 256 * rank;
            if (nt == 0) {
                for (int c = 0; c < 256 / 8; ++c)
                    reinterpret_cast<uint4 *>(orow)[c] = make_uint4(0, 0, 0, 0);
            }
        }
        if (nt > 0) {
            const float inv_l = 1.f / l_run;
#pragma unroll 1
            for (int c = 0; c < 256 / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(trow + COL_O + 32 * c, o);
                tmem_wait_ld();
                if (head < p.n_q) {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.o + ((size_t)b * p.n_q + head) * DV + 256 * rank + 32 * c);
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8) {
                        uint4 w;
                        w.x = f2_to_bf2(__uint_as_float(o[8 * q8 + 0]) * inv_l, __uint_as_float(o[8 * q8 + 1]) * inv_l);
                        w.y = f2_to_bf2(__uint_as_float(o[8 * q8 + 2]) * inv_l, __uint_as_float(o[8 * q8 + 3]) * inv_l);
                        w.z = f2_to_bf2(__uint_as_float(o[8 * q8 + 4]) * inv_l, __uint_as_float(o[8 * q8 + 5]) * inv_l);
                        w.w = f2_to_bf2(__uint_as_float(o[8 * q8 + 6]) * inv_l, __uint_as_float(o[8 * q8 + 7]) * inv_l);
                        dst[q8] = w;
                    }
                }
            }
        }
        if (rank == 0 && head < p.n_q && p.lse != nullptr)
            p.lse[(size_t)b * p.n_q + head] = nt > 0 ? (m_run + log2f(l_run)) * 0.6931471805599453f : -INFINITY;
    }

    // ---- teardown: no remote access may target a CTA that has left
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace mla
}  // namespace attn
