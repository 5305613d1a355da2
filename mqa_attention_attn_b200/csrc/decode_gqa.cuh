// decode_gqa.cuh -- single-token GQA decode against a KV cache, split-KV.
//
// A work unit is (sequence b, KV head g, a block of GT query heads of that
// group, one chunk of ch consecutive cached keys: a multiple of 128 up to
// 2048, or 1024 at 16 heads, chosen at launch from the sizes and the SM
// count so that small batches too spread over every SM). The grid
// is persistent (as many CTAs per SM as shared memory allows: two for the
// bf16 and e4m3 caches at up to 8 heads per block); each CTA walks its share
// of the units.
//
// Per unit, with the group's GT query rows as the narrow operand of the
// 5th-generation tensor core (padded to NH = max(8, GT) columns):
//   S^T[key][h] = K_tile . Q^T        M = 128 keys, N = NH, K = 128 dims
//   (softmax over the chunk on the CUDA cores, reading S^T from TMEM)
//   O^T[d][h]  += V_tile^T . P^T      M = 128 dims, N = NH, K = 128 keys
// K and V tiles (128 keys x 128 dims, two 64-dim boxes with the 128-byte
// swizzle) stream HBM -> shared memory by TMA through a ring that a producer
// warp keeps full across units; one thread issues the MMAs; four warps
// (one TMEM lane quarter each) do the softmax, hand each tile's P^T to the
// MMA thread through one of two shared slots, and write the partial
// (o, m, l) of the chunk to the workspace. A second kernel merges the chunks
// of each (b, h) by their log-sum-exp weights. With rotary tables given, the
// MMA warp first rotates the unit's query rows at position seqlen - 1.
//
// Each K/V element is read from HBM once and used by all GT heads of its
// group (the grouped sharing of "Attention Engineering: From MHA to GQA, MLA
// & FlashAttention", section 2); the chunk merge is the online-softmax
// rescaling of section 4 applied across chunks instead of tiles. Decode
// arithmetic intensity is about n_q / n_kv FLOPs per byte (same page,
// section 0), so the kernel is bound by HBM bandwidth; the tensor core is
// used because it retires the G-fold reuse of every loaded element in a few
// instructions, leaving the issue slots of the SM to the data movement and
// the softmax.
#pragma once

#include "rope.cuh"
#include "sm100.cuh"

#ifndef ATTN_DEC_STAGES
#define ATTN_DEC_STAGES 2
#endif

namespace attn {
namespace dec {

constexpr int D = 128;            // head dim (keys and values)
constexpr int KT = 128;           // keys per tile (the MMA's M for S^T)
// Largest chunk of keys one work unit takes: 2048 while a head block has at
// most 8 heads, 1024 for 16 (the chunk's S^T, 16 or 8 tiles x NH columns,
// then stays within 256 TMEM columns so that two CTAs share an SM). The
// launch may choose a smaller chunk (a multiple of 128 keys) so that small
// batches still spread over every SM.
__host__ __device__ constexpr int chunk_keys(int GT, bool fp8 = false) {
    return (void)fp8, GT <= 8 ? 2048 : 1024;
}
constexpr int NSTAGE = ATTN_DEC_STAGES;
constexpr int BOX_BYTES = KT * 128;         // one 64-dim box: 128 rows x 128 B
constexpr int TILE_BYTES = 2 * BOX_BYTES;   // 32 KB
constexpr int NSW = 4;            // softmax warps (TMEM lane quarters)
constexpr int PRODUCER_WARP = 4;
constexpr int MMA_WARP = 5;
constexpr int THREADS = 6 * 32;
// FP8 (e4m3) cache: TMA brings 128 x 128-byte tiles into an 8-bit ring and
// NCONV more warps (6 ..) widen them to the f16 tiles the MMAs read.
#ifndef ATTN_DEC_NCONV
#define ATTN_DEC_NCONV 4
#endif
constexpr int NCONV = ATTN_DEC_NCONV;
static_assert(NCONV == 2 || NCONV == 4, "converter warps");
constexpr int CONV_WARP0 = 6;
constexpr int THREADS_FP8 = (6 + NCONV) * 32;
constexpr int NSTAGE8 = 2;
constexpr int TILE8_BYTES = KT * D;         // 16 KB: 128 rows x 128 one-byte values

template <int GT, bool FP8 = false>
struct Cfg {
    static constexpr int NH = GT < 8 ? 8 : GT;             // MMA N (query-head columns)
    static constexpr int CH = chunk_keys(GT, FP8);          // most keys per unit
    static constexpr int TPC = CH / KT;                     // tiles per unit
    static constexpr int QBOX = NH * 128;                   // one 64-dim half of the Q rows
    static constexpr int COL_S = 0;                         // S^T: TPC tiles x NH columns
    static constexpr int COL_O = TPC * NH;                  // O^T: NH columns
    static constexpr int NEED = COL_O + NH;
    static constexpr int TMEM_COLS = NEED <= 32 ? 32 : NEED <= 64 ? 64 : NEED <= 128 ? 128 : 256;
    static_assert(GT == 1 || GT == 2 || GT == 4 || GT == 8 || GT == 16 || GT == 32, "head block");
};

template <int GT, bool FP8 = false>
struct Smem {
    using C = Cfg<GT, FP8>;
    uint8_t ring[NSTAGE][TILE_BYTES];       // 1024-byte aligned (swizzle atoms); f16 when FP8
    uint8_t ring8[FP8 ? NSTAGE8 : 1][FP8 ? TILE8_BYTES : 1024];   // e4m3 tiles as loaded
    uint8_t q[2][C::QBOX];                  // Q rows, two 64-dim boxes, 128-byte swizzle
    uint8_t p[2][C::NH / 8][KT * 16];       // P^T of one tile, two slots: [8-head block][key][8 heads]
    float red_m[2][NSW][GT];                // double-buffered by unit parity
    float red_l[2][NSW][GT];
    uint64_t full[NSTAGE];
    uint64_t empty[NSTAGE];
    uint64_t full8[NSTAGE8], empty8[NSTAGE8];
    uint64_t q_full, q_empty, s_full, o_full, mma_done;
    uint64_t p_full[2], p_empty[2];         // per-tile P hand-off, softmax <-> MMA
    uint64_t q_conv;                        // FP8: Q rows converted to f16
    uint32_t tmem_base;
    int abort_flag;
};

template <int GT, bool FP8 = false>
constexpr size_t smem_bytes() {
    return sizeof(Smem<GT, FP8>) + 1024;  // + alignment slack
}
template <bool FP8>
constexpr bool smem_fits() {   // every head block the launches instantiate
    return smem_bytes<1, FP8>() <= kMaxSmemPerCta && smem_bytes<2, FP8>() <= kMaxSmemPerCta &&
           smem_bytes<4, FP8>() <= kMaxSmemPerCta && smem_bytes<8, FP8>() <= kMaxSmemPerCta &&
           smem_bytes<16, FP8>() <= kMaxSmemPerCta;
}
static_assert(smem_fits<false>() && smem_fits<true>(), "decode shared memory exceeds a CTA's");

// FP8 cache scales: element (b, g, j, c) of the cache means
// e4m3(byte) * k_scale[g] (keys) or * v_scale[g] (values).
struct Fp8Scales {
    const float *k_scale, *v_scale;   // null on the bf16 path
    // 0: one scale per KV head ([n_kv]); t > 0: one scale per 128-key tile of
    // each (sequence, KV head), [B][n_kv][t], key j in tile j / 128
    int tile_stride;
};

// Sliding window over the cache (window 0: none): of keys 0 .. L-1 a
// sequence of length L keeps the last `window` and the first `n_sink`.
struct Window {
    int window, n_sink;
};

// The chunks of a sequence of length L that hold a visible key, in order:
// sink chunks 0 .. n_sc-1, then window chunks wc0 .. ceil(L / CH) - 1.
struct ChunkPlan {
    int n, n_sc, wc0;
    __device__ __forceinline__ int split(int c) const { return c < n_sc ? c : wc0 + (c - n_sc); }
};

__device__ __forceinline__ ChunkPlan chunk_plan(int L, int CH, Window w) {
    const int all = (L + CH - 1) / CH;
    if (w.window <= 0) return ChunkPlan{all, all, all};
    const int n_sc = (min(w.n_sink, L) + CH - 1) / CH;
    const int wc0 = max(max(L - w.window, 0) / CH, n_sc);
    return ChunkPlan{n_sc + max(all - wc0, 0), n_sc, wc0};
}

// Is key `key` of a sequence of length L visible under the window?
__device__ __forceinline__ bool window_keeps(int key, int L, Window w) {
    return w.window <= 0 || key >= L - w.window || key < w.n_sink;
}

// Work units are the non-empty (b, kv head, head block, chunk) slots, in order
// b-major, then kv head and head block, then chunk; sequence b contributes
// n_kv * n_hb * ceil(seqlen_b / CH) units (CH = keys per unit). The CTA walks units c, c + G, ...
// (G = gridDim.x) and every role derives the same unit from its index.
struct UnitCursor {
    int b = 0;          // sequence of the current range
    long long base = 0; // first unit index of sequence b
    int ns = 0;         // chunks of sequence b that hold a visible key
    int seqlen = 0;
    ChunkPlan plan{0, 0, 0};
};

struct Unit {
    int b, kvh, hb, split, key0, nkeys, ntiles, seqlen;
};


// Paged cache: logical key t of sequence b sits in row t % page_size of page
// table[b * pages_per_seq + t / page_size] of a page pool; the K and V tensor
// maps then address [page][token][kv head][dim] (any strides). A 128-key tile
// is KT / box_rows TMA boxes, box_rows = min(page_size, KT).
struct PageTable {
    const int32_t *table;   // [B][pages_per_seq]; null: contiguous cache
    int pages_per_seq;
    int page_shift;         // log2(page_size)
    int box_rows;
    int num_pages;
};

__device__ __forceinline__ int clamp_seqlen(const int32_t *seqlens, int b, int S_max) {
    int L = seqlens[b];
    return L < 0 ? 0 : (L > S_max ? S_max : L);
}

// Advance the cursor to the sequence holding unit i (i never decreases) and
// decode the unit. Returns false when i is past the last unit.
__device__ __forceinline__ void start_sequence(UnitCursor &cur, const int32_t *seqlens, int S_max, int CH, Window w) {
    cur.seqlen = clamp_seqlen(seqlens, cur.b, S_max);
    cur.plan = chunk_plan(cur.seqlen, CH, w);
    cur.ns = cur.plan.n;
}

__device__ __forceinline__ bool next_unit(UnitCursor &cur, long long i, const int32_t *seqlens, int B, int S_max,
                                          int CH, int n_hb, int units_per_chunk, Window w, Unit &u) {
    while (cur.b < B) {
        const long long n = (long long)units_per_chunk * cur.ns;
        if (i < cur.base + n) {
            const long long local = i - cur.base;
            const int y = (int)(local / cur.ns);
            u.b = cur.b;
            u.split = cur.plan.split((int)(local % cur.ns));
            u.kvh = y / n_hb;
            u.hb = y % n_hb;
            u.key0 = u.split * CH;
            u.nkeys = min(CH, cur.seqlen - u.key0);
            u.ntiles = (u.nkeys + KT - 1) / KT;
            u.seqlen = cur.seqlen;
            return true;
        }
        cur.base += n;
        ++cur.b;
        if (cur.b < B) start_sequence(cur, seqlens, S_max, CH, w);
    }
    return false;
}


template <int GT, bool PAGED, bool FP8 = false>
__global__ void __launch_bounds__(FP8 ? THREADS_FP8 : THREADS, (FP8 && GT >= 16) ? 1 : 2)
decode_split_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const int32_t *__restrict__ seqlens,
                    float *__restrict__ ws_o, float2 *__restrict__ ws_ml, int B, int n_q, int n_kv, int G, int n_hb,
                    int S_max, int n_splits, int ch, float scale_log2, const PageTable pt, const Window win,
                    const Fp8Scales fs, const rope::Tables rt) {
    using C = Cfg<GT, FP8>;
    constexpr int NH = C::NH;
    // the merge kernel (launched as a programmatic dependent) may be scheduled
    // now; it waits for this grid to complete before it reads the workspace
    griddep_launch_dependents();
    extern __shared__ uint8_t smem_raw[];
    Smem<GT, FP8> &sm =
        *reinterpret_cast<Smem<GT, FP8> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t warp = warp_id(), lane = lane_id();
    const int units_per_chunk = n_kv * n_hb;   // units of one chunk index of one sequence

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(smem_u32(&sm.full[s]), FP8 ? NCONV : 1);   // FP8: one arrive per converter warp
            mbar_init(smem_u32(&sm.empty[s]), 1);
        }
        for (int s = 0; s < NSTAGE8; ++s) {
            mbar_init(smem_u32(&sm.full8[s]), 1);
            mbar_init(smem_u32(&sm.empty8[s]), NCONV);
        }
        mbar_init(smem_u32(&sm.q_conv), NCONV);
        mbar_init(smem_u32(&sm.q_full), 1);
        mbar_init(smem_u32(&sm.q_empty), 1);
        mbar_init(smem_u32(&sm.s_full), 1);
        for (int x = 0; x < 2; ++x) {
            mbar_init(smem_u32(&sm.p_full[x]), NSW * 32);
            mbar_init(smem_u32(&sm.p_empty[x]), 1);
        }
        mbar_init(smem_u32(&sm.o_full), 1);
        mbar_init(smem_u32(&sm.mma_done), 1);
        sm.abort_flag = 0;
        fence_mbar_init();
        if constexpr (!FP8 && !PAGED) {
            // The first unit's Q rows and first ring tiles go out now, before
            // the setup barrier and the TMEM allocation (the producer warp
            // skips them): every stage is free at the start.
            UnitCursor c0;
            Unit u0;
            if (B > 0) start_sequence(c0, seqlens, S_max, ch, win);
            if (B > 0 && next_unit(c0, blockIdx.x, seqlens, B, S_max, ch, n_hb, n_kv * n_hb, win, u0)) {
                tma_prefetch_desc(&tm_q);
                tma_prefetch_desc(&tm_k);
                tma_prefetch_desc(&tm_v);
                const int h0 = u0.kvh * G + u0.hb * GT;
                mbar_arrive_expect_tx(smem_u32(&sm.q_full), 2 * C::QBOX);
                tma_load_3d(smem_u32(sm.q[0]), &tm_q, smem_u32(&sm.q_full), 0, h0, u0.b);
                tma_load_3d(smem_u32(sm.q[1]), &tm_q, smem_u32(&sm.q_full), 64, h0, u0.b);
                const int pre = min(NSTAGE, 2 * u0.ntiles);
                for (int j = 0; j < pre; ++j) {
                    const CUtensorMap *tm = (j < u0.ntiles) ? &tm_k : &tm_v;
                    const int krow = u0.key0 + (j < u0.ntiles ? j : j - u0.ntiles) * KT;
                    const uint32_t full = smem_u32(&sm.full[j]);
                    mbar_arrive_expect_tx(full, TILE_BYTES);
                    tma_load_4d(smem_u32(sm.ring[j]), tm, full, 0, krow, u0.kvh, u0.b);
                    tma_load_4d(smem_u32(sm.ring[j]) + BOX_BYTES, tm, full, 64, krow, u0.kvh, u0.b);
                }
            }
        }
        // values above S_max are clamped; report it once per launch
        if (blockIdx.x == 0)
            for (int b = 0; b < B; ++b)
                if (seqlens[b] > S_max) {
                    atomicOr(&g_status, kStatusRange);
                    break;
                }
    }
    if (warp == MMA_WARP) {
        tmem_alloc(smem_u32(&sm.tmem_base), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort_flag = &sm.abort_flag;

    UnitCursor cur;
    if (B > 0) start_sequence(cur, seqlens, S_max, ch, win);
    Unit u;

    if (warp == PRODUCER_WARP) {
        // ---------------- TMA producer: Q rows, then K tiles, then V tiles ----------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            int t = 0, n = 0;   // ring tiles issued, units started
            bool ok = true;
            for (long long i = blockIdx.x; ok && next_unit(cur, i, seqlens, B, S_max, ch, n_hb, units_per_chunk, win, u);
                 i += gridDim.x, ++n) {
                // the single Q buffer is free once the previous unit's S^T MMAs completed
                if (n > 0 && !mbar_wait(smem_u32(&sm.q_empty), (n - 1) & 1, abort_flag, 0x101)) break;
                const int h0 = u.kvh * G + u.hb * GT;
                // the first unit's Q and first ring tiles were issued during setup
                const int pre = (!FP8 && !PAGED && n == 0) ? min(NSTAGE, 2 * u.ntiles) : 0;
                if (pre == 0) {
                    mbar_arrive_expect_tx(smem_u32(&sm.q_full), 2 * C::QBOX);
                    tma_load_3d(smem_u32(sm.q[0]), &tm_q, smem_u32(&sm.q_full), 0, h0, u.b);
                    tma_load_3d(smem_u32(sm.q[1]), &tm_q, smem_u32(&sm.q_full), 64, h0, u.b);
                }
                t += pre;
                for (int j = pre; j < 2 * u.ntiles; ++j, ++t) {
                    const CUtensorMap *tm = (j < u.ntiles) ? &tm_k : &tm_v;
                    const int krow = u.key0 + (j < u.ntiles ? j : j - u.ntiles) * KT;
                    if constexpr (FP8) {
                        // 8-bit ring, drained by the converter warps
                        const int s8 = t % NSTAGE8;
                        if (!mbar_wait(smem_u32(&sm.empty8[s8]), ((t / NSTAGE8) & 1) ^ 1, abort_flag, 0x105)) {
                            ok = false;
                            break;
                        }
                        const uint32_t full8 = smem_u32(&sm.full8[s8]);
                        mbar_arrive_expect_tx(full8, TILE8_BYTES);
                        tma_load_4d(smem_u32(sm.ring8[s8]), tm, full8, 0, krow, u.kvh, u.b);
                        continue;
                    }
                    const int s = t % NSTAGE;
                    if (!mbar_wait(smem_u32(&sm.empty[s]), ((t / NSTAGE) & 1) ^ 1, abort_flag, 0x102)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full = smem_u32(&sm.full[s]);
                    const uint32_t dst = smem_u32(sm.ring[s]);
                    if constexpr (PAGED) {
                        // boxes holding at least one key below the length; rows of
                        // the tile past them are never read as valid keys (their
                        // scores are masked and their value rows cleared)
                        const int kend = u.key0 + u.nkeys;
                        const int nbox = min(KT / pt.box_rows, (kend - krow + pt.box_rows - 1) / pt.box_rows);
                        const uint32_t box_bytes = (uint32_t)pt.box_rows * 128u;
                        mbar_arrive_expect_tx(full, 2u * box_bytes * (uint32_t)nbox);
                        const int32_t *row_pages = pt.table + (size_t)u.b * pt.pages_per_seq;
                        for (int x = 0; x < nbox; ++x) {
                            const int key = krow + x * pt.box_rows;
                            const int page = row_pages[key >> pt.page_shift];
                            // a page id outside the pool reads zeros (TMA bounds) and is reported
                            if ((unsigned)page >= (unsigned)pt.num_pages) atomicOr(&g_status, kStatusRange);
                            const int prow = key & ((1 << pt.page_shift) - 1);
                            tma_load_4d(dst + x * box_bytes, tm, full, 0, prow, u.kvh, page);
                            tma_load_4d(dst + BOX_BYTES + x * box_bytes, tm, full, 64, prow, u.kvh, page);
                        }
                    } else {
                        mbar_arrive_expect_tx(full, TILE_BYTES);
                        tma_load_4d(dst, tm, full, 0, krow, u.kvh, u.b);
                        tma_load_4d(dst + BOX_BYTES, tm, full, 64, krow, u.kvh, u.b);
                    }
                }
            }
            // Do not leave while copies into this CTA's shared memory are in
            // flight: wait (bounded) for the last issued tile of each stage
            // and the last Q load.
            if constexpr (FP8) {
                for (int j = t - 1; j >= 0 && j >= t - NSTAGE8; --j)
                    mbar_wait(smem_u32(&sm.full8[j % NSTAGE8]), (j / NSTAGE8) & 1, nullptr, 0x106);
            } else {
                for (int j = t - 1; j >= 0 && j >= t - NSTAGE; --j)
                    mbar_wait(smem_u32(&sm.full[j % NSTAGE]), (j / NSTAGE) & 1, nullptr, 0x103);
            }
            if (n > 0) mbar_wait(smem_u32(&sm.q_full), (n - 1) & 1, nullptr, 0x104);
        }
        __syncwarp();
    } else if (warp == MMA_WARP) {
        // ---------------- MMA issue (one thread), ring bookkeeping (whole warp) ----------------
        // K tile (K-major) x Q rows (K-major); V^T (MN-major) x P^T (MN-major);
        // operands bf16, or f16 on the FP8 path (widened tiles)
        constexpr uint32_t idesc_s = FP8 ? umma_idesc_f16(KT, NH, 0, 0) : umma_idesc_bf16(KT, NH, 0, 0);
        constexpr uint32_t idesc_o = FP8 ? umma_idesc_f16(D, NH, 1, 1) : umma_idesc_bf16(D, NH, 1, 1);
        int t = 0, n = 0, pc = 0;   // ring tiles, units, P tiles handed over
        for (long long i = blockIdx.x; next_unit(cur, i, seqlens, B, S_max, ch, n_hb, units_per_chunk, win, u);
             i += gridDim.x, ++n) {
            if (!mbar_wait(smem_u32(FP8 ? &sm.q_conv : &sm.q_full), n & 1, abort_flag, 0x201)) break;
            if (!FP8 && rt.cos != nullptr) {
                // rotary embedding of the unit's query rows (the new token sits at
                // position seqlen - 1; the cached keys are stored rotated): NH rows
                // x 16 chunks of 8 dims, spread over the warp
                int pos = u.seqlen - 1;
                if (pos >= rt.n_pos) {
                    if (lane == 0) atomicOr(&g_status, kStatusRange);
                    pos = rt.n_pos - 1;
                }
                const float *cr = rt.cos + (size_t)pos * (D / 2), *sr = rt.sin + (size_t)pos * (D / 2);
                for (int i = (int)lane; i < NH * 16; i += 32) {
                    const int row = i >> 4, bx = (i >> 3) & 1, c = i & 7;
                    const uint32_t a = smem_u32(sm.q[bx]) + swz<3>((uint32_t)(row * 128 + c * 16));
                    const int j0 = bx * 32 + c * 4;
                    const float4 cc = __ldg(reinterpret_cast<const float4 *>(cr + j0));
                    const float4 ss = __ldg(reinterpret_cast<const float4 *>(sr + j0));
                    sts128(a, rope::rope_chunk(lds128(a), cc, ss));
                }
                fence_proxy_async_smem();
                __syncwarp();
            }
            bool ok = true;
            for (int j = 0; j < u.ntiles; ++j) {
                const int g = t + j, s = g % NSTAGE;
                if (!mbar_wait(smem_u32(&sm.full[s]), (g / NSTAGE) & 1, abort_flag, 0x202)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t koff = (uint32_t)((kk >> 2) * BOX_BYTES + (kk & 3) * 32);
                        const uint32_t qoff = (uint32_t)((kk >> 2) * C::QBOX + (kk & 3) * 32);
                        const uint64_t ad = umma_smem_desc(smem_u32(sm.ring[s]) + koff, 16, 1024, 2);
                        const uint64_t bd = umma_smem_desc(smem_u32(sm.q[0]) + qoff, 16, 1024, 2);
                        umma_ss(tmem + C::COL_S + j * NH, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(smem_u32(&sm.empty[s]));
                }
                __syncwarp();
            }
            if (!ok) break;
            if (lane == 0) {
                umma_commit(smem_u32(&sm.q_empty));
                umma_commit(smem_u32(&sm.s_full));
            }
            __syncwarp();
            t += u.ntiles;
            for (int j = 0; j < u.ntiles; ++j, ++pc) {
                const int g = t + j, s = g % NSTAGE;
                if (!mbar_wait(smem_u32(&sm.full[s]), (g / NSTAGE) & 1, abort_flag, 0x204) ||
                    !mbar_wait(smem_u32(&sm.p_full[pc & 1]), (pc >> 1) & 1, abort_flag, 0x203)) {
                    ok = false;
                    break;
                }
                const int rows = u.nkeys - j * KT;   // valid value rows of this tile
                if (!FP8 && rows < KT) {             // (the converter clears them on the FP8 path)
                    // Rows past the sequence end get weight 0, but 0 * (NaN or
                    // Inf) is not 0: clear them so that whatever the cache holds
                    // beyond the length cannot reach the output.
                    const uint32_t base = smem_u32(sm.ring[s]);
                    for (int e = rows * 8 + (int)lane; e < KT * 8; e += 32) {
                        const uint32_t off = (uint32_t)(e >> 3) * 128u + (uint32_t)(e & 7) * 16u;
                        sts128(base + off, make_uint4(0u, 0u, 0u, 0u));
                        sts128(base + BOX_BYTES + off, make_uint4(0u, 0u, 0u, 0u));
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                tc_fence_after();
                if (lane == 0) {
#pragma unroll
                    for (int ks = 0; ks < KT / 16; ++ks) {
                        // A = V^T: 16 keys x 128 dims of the tile; B = P^T rows of the same 16 keys
                        const uint64_t ad = umma_smem_desc(smem_u32(sm.ring[s]) + ks * 16 * 128, BOX_BYTES, 1024, 2);
                        const uint64_t bd = umma_smem_desc(smem_u32(sm.p[pc & 1][0]) + ks * 16 * 16, 128, KT * 16, 0);
                        umma_ss(tmem + C::COL_O, ad, bd, idesc_o, (j > 0 || ks > 0) ? 1u : 0u);
                    }
                    umma_commit(smem_u32(&sm.empty[s]));
                    umma_commit(smem_u32(&sm.p_empty[pc & 1]));
                }
                __syncwarp();
            }
            if (!ok) break;
            if (lane == 0) umma_commit(smem_u32(&sm.o_full));
            __syncwarp();
            t += u.ntiles;
        }
        // every MMA issued by this warp has completed before TMEM is released
        if (lane == 0) umma_commit(smem_u32(&sm.mma_done));
        __syncwarp();
        mbar_wait(smem_u32(&sm.mma_done), 0, nullptr, 0x205);
    } else if (FP8 && warp >= CONV_WARP0) {
        // ---------------- FP8: widen e4m3 tiles to f16 (NCONV warps, 128 / NCONV rows each) ----------------
        const int cw = (int)warp - CONV_WARP0;
        int t = 0, n = 0;
        bool ok = true;
        for (long long i = blockIdx.x; ok && next_unit(cur, i, seqlens, B, S_max, ch, n_hb, units_per_chunk, win, u);
             i += gridDim.x, ++n) {
            // the unit's Q rows, bf16 -> f16 in place (same byte positions)
            ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.q_full), n & 1, abort_flag, 0x401));
            if (!ok) break;
            for (int c = cw * 32 + (int)lane; c < 2 * C::QBOX / 16; c += NCONV * 32) {
                const uint32_t a = smem_u32(sm.q[0]) + (uint32_t)c * 16u;
                uint4 w = lds128(a);
                float2 f;
                f = bf2_to_f2(w.x), w.x = f2_to_h2_sat(f.x, f.y);
                f = bf2_to_f2(w.y), w.y = f2_to_h2_sat(f.x, f.y);
                f = bf2_to_f2(w.z), w.z = f2_to_h2_sat(f.x, f.y);
                f = bf2_to_f2(w.w), w.w = f2_to_h2_sat(f.x, f.y);
                sts128(a, w);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sm.q_conv));
            for (int j = 0; j < 2 * u.ntiles; ++j, ++t) {
                const int s8 = t % NSTAGE8, s = t % NSTAGE;
                bool w_ok = mbar_wait(smem_u32(&sm.full8[s8]), (t / NSTAGE8) & 1, abort_flag, 0x402);
                w_ok = w_ok && mbar_wait(smem_u32(&sm.empty[s]), ((t / NSTAGE) & 1) ^ 1, abort_flag, 0x403);
                ok = __all_sync(0xffffffffu, w_ok);
                if (!ok) break;
                // rows past the length become 0 (their scores are masked; 0 * NaN would not be 0)
                const int rows = u.nkeys - (j < u.ntiles ? j : j - u.ntiles) * KT;
                const uint32_t src = smem_u32(sm.ring8[s8]), dst = smem_u32(sm.ring[s]);
                // 16-byte source chunks (16 dims each) of this warp's rows, 32 / NCONV
                // per lane, in batches of 8: all loads of a batch, then its stores
                constexpr int CPL = 32 / NCONV;
#pragma unroll
                for (int kb = 0; kb < CPL; kb += 8) {
                    uint4 w[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int idx = (kb + k) * 32 + (int)lane;
                        const int r = cw * (KT / NCONV) + (idx >> 3), c = idx & 7;
                        w[k] = r < rows ? lds128(src + (uint32_t)r * 128u + (uint32_t)((c ^ (r & 7)) << 4))
                                        : make_uint4(0u, 0u, 0u, 0u);
                    }
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int idx = (kb + k) * 32 + (int)lane;
                        const int r = cw * (KT / NCONV) + (idx >> 3), c = idx & 7;
                        // rows past the length stay 0 (0x00 bytes widen to +0)
                        const uint4 o0 = e4m3x8_to_f16x8(w[k].x, w[k].y);
                        const uint4 o1 = e4m3x8_to_f16x8(w[k].z, w[k].w);
                        // dims 16c .. 16c+15 land in 64-dim box c/4, 16-byte chunks 2(c%4), 2(c%4)+1.
                        // The two boxes share banks, so lanes of box 1 store their odd chunk
                        // first: each 8-lane phase of a store then hits 8 distinct bank groups.
                        const int c0 = (c & 3) * 2, sw = c >> 2;
                        const uint32_t row = dst + (uint32_t)sw * BOX_BYTES + (uint32_t)r * 128u;
                        sts128(row + (uint32_t)(((c0 + sw) ^ (r & 7)) << 4), sw ? o1 : o0);
                        sts128(row + (uint32_t)(((c0 + 1 - sw) ^ (r & 7)) << 4), sw ? o0 : o1);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(smem_u32(&sm.full[s]));
                    mbar_arrive(smem_u32(&sm.empty8[s8]));
                }
            }
        }
    } else if (warp < NSW) {
        // ---------------- softmax + partial output (128 threads, thread = TMEM lane) ----------------
        const int tid = threadIdx.x;                       // key row of each tile; dim row of O^T
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        int n = 0, pc = 0;   // units, P tiles handed over
        for (long long i = blockIdx.x; next_unit(cur, i, seqlens, B, S_max, ch, n_hb, units_per_chunk, win, u);
             i += gridDim.x, ++n) {
            const int h0 = u.kvh * G + u.hb * GT;
            // FP8: the key scale of this KV head scales every score
            const bool tiles = FP8 && fs.tile_stride > 0;   // FP8: a scale per 128-key tile
            const float su = (FP8 && !tiles) ? scale_log2 * fs.k_scale[u.kvh] : scale_log2;
            // FP8 per-tile scales of this unit's tiles: (b, kv head) row, first tile
            const size_t trow = tiles ? ((size_t)u.b * n_kv + u.kvh) * fs.tile_stride + u.key0 / KT : 0;
            bool ok = mbar_wait(smem_u32(&sm.s_full), n & 1, abort_flag, 0x301);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            // pass 1: chunk maximum per head, the chunk's S^T read from TMEM four tiles at a time
            float m[GT];
#pragma unroll
            for (int h = 0; h < GT; ++h) m[h] = -INFINITY;
            for (int jg = 0; jg < u.ntiles; jg += 4) {
                uint32_t sv[4][NH];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj)
                    if (jg + jj < u.ntiles) tmem_ld<NH>(lane_base + C::COL_S + (jg + jj) * NH, sv[jj]);
                tmem_wait_ld();
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int key = (jg + jj) * KT + tid;
                    if (jg + jj < u.ntiles && key < u.nkeys && window_keeps(u.key0 + key, u.seqlen, win)) {
                        // per-tile key scales: the maximum of the scaled scores
                        const float kt = tiles ? __ldg(fs.k_scale + trow + jg + jj) : 1.f;
#pragma unroll
                        for (int h = 0; h < GT; ++h) m[h] = fmaxf(m[h], tiles ? __uint_as_float(sv[jj][h]) * kt
                                                                              : __uint_as_float(sv[jj][h]));
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < GT; ++h) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m[h] = fmaxf(m[h], __shfl_xor_sync(0xffffffffu, m[h], o));
                if (lane == 0) sm.red_m[n & 1][warp][h] = m[h];
            }
            if (named_bar_or(1, NSW * 32, !ok)) break;
            float mc[GT], l[GT];
#pragma unroll
            for (int h = 0; h < GT; ++h) {
                float mm = sm.red_m[n & 1][0][h];
#pragma unroll
                for (int w = 1; w < NSW; ++w) mm = fmaxf(mm, sm.red_m[n & 1][w][h]);
                mc[h] = mm * su;             // finite: every unit holds at least one key
                l[h] = 0.f;
            }
            // pass 2: p = 2^(s * scale * log2 e - m) tile by tile, each tile's
            // P^T rows [key][8 heads] (bf16; f16 on the FP8 path) handed to the
            // MMA thread through one of two slots
            for (int j = 0; j < u.ntiles; ++j, ++pc) {
                uint32_t sv[NH];
                tmem_ld<NH>(lane_base + C::COL_S + j * NH, sv);
                tmem_wait_ld();
                const int key = j * KT + tid;
                const bool valid = key < u.nkeys && window_keeps(u.key0 + key, u.seqlen, win);
                // per-tile scales: the key scale joins the exponent's, the value
                // scale multiplies P (the row sums take P unscaled)
                const float sj = tiles ? su * __ldg(fs.k_scale + trow + j) : su;
                const float vj = tiles ? __ldg(fs.v_scale + trow + j) : 1.f;
                uint32_t pk[NH / 2];
#pragma unroll
                for (int h2 = 0; h2 < NH / 2; ++h2) {
                    float p0 = 0.f, p1 = 0.f;
                    if (2 * h2 < GT && valid) p0 = ex2(fmaf(__uint_as_float(sv[2 * h2]), sj, -mc[2 * h2]));
                    if (2 * h2 + 1 < GT && valid) p1 = ex2(fmaf(__uint_as_float(sv[2 * h2 + 1]), sj, -mc[2 * h2 + 1]));
                    if (2 * h2 < GT) l[2 * h2] += p0;
                    if (2 * h2 + 1 < GT) l[2 * h2 + 1] += p1;
                    pk[h2] = FP8 ? (tiles ? f2_to_h2_sat(p0 * vj, p1 * vj) : f2_to_h2_sat(p0, p1)) : f2_to_bf2(p0, p1);
                }
                // the slot is free once the P.V of the tile two before has completed
                ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.p_empty[pc & 1]), ((pc >> 1) & 1) ^ 1,
                                                       abort_flag, 0x303));
#pragma unroll
                for (int hb8 = 0; hb8 < NH / 8; ++hb8)
                    sts128(smem_u32(sm.p[pc & 1][hb8]) + (uint32_t)tid * 16u,
                           make_uint4(pk[hb8 * 4 + 0], pk[hb8 * 4 + 1], pk[hb8 * 4 + 2], pk[hb8 * 4 + 3]));
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(smem_u32(&sm.p_full[pc & 1]));
            }
#pragma unroll
            for (int h = 0; h < GT; ++h) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) l[h] += __shfl_xor_sync(0xffffffffu, l[h], o);
                if (lane == 0) sm.red_l[n & 1][warp][h] = l[h];
            }
            ok = mbar_wait(smem_u32(&sm.o_full), n & 1, abort_flag, 0x302);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            uint32_t ov[NH];
            tmem_ld<NH>(lane_base + C::COL_O, ov);
            tmem_wait_ld();
            tc_fence_before();
            if (named_bar_or(1, NSW * 32, !ok)) break;
            const size_t row0 = (size_t)u.b * n_q + h0;
            const float vsc = (FP8 && !tiles) ? fs.v_scale[u.kvh] : 1.f;   // FP8: the value scale of this KV head
#pragma unroll
            for (int h = 0; h < GT; ++h)
                ws_o[((row0 + h) * n_splits + u.split) * D + tid] = __uint_as_float(ov[h]) * vsc;
#pragma unroll
            for (int h = 0; h < GT; ++h)
                if (tid == h) {
                    float lt = 0.f;
#pragma unroll
                    for (int w = 0; w < NSW; ++w) lt += sm.red_l[n & 1][w][h];
                    ws_ml[(row0 + h) * n_splits + u.split] = make_float2(mc[h], lt);
                }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// Merge the chunks of each (b, h) (value width DV: 128, or the MLA form's 512):
// M = max m_s, w_s = 2^(m_s - M), O = sum w_s o_s / sum w_s l_s,
// LSE = (M + log2 sum w_s l_s) * ln 2.
// Launched as a programmatic dependent of the split kernel, so that its launch
// overlaps that kernel's tail; it waits for the partials before reading them.
// One CTA per (h, b), 256 threads = 8 groups of 32; a group takes the chunks
// s = g (mod 8) and folds them with a running maximum of its own (each
// chunk's (m_s, l_s) and partial output are loaded together, so a group's
// loads all go out at once), a lane 4 consecutive output dims per 128
// (16-byte loads); the eight groups' sums meet in shared memory, rescaled to
// the overall maximum.
constexpr int COMBINE_THREADS = 256;
constexpr int COMBINE_GROUPS = COMBINE_THREADS / 32;

template <int DV>
__global__ void __launch_bounds__(COMBINE_THREADS)
decode_combine_kernel(const float *__restrict__ ws_o, const float2 *__restrict__ ws_ml,
                      const int32_t *__restrict__ seqlens, __nv_bfloat16 *__restrict__ o,
                      float *__restrict__ lse, int n_q, int n_splits, int S_max, int chunk, Window win) {
    static_assert(DV % 128 == 0, "value width");
    constexpr int NQ = DV / 128;   // float4 loads per lane and chunk
    constexpr int NG = COMBINE_GROUPS;
    __shared__ float red[NG][DV];
    __shared__ float part_m[NG], part_l[NG];
    const int h = blockIdx.x, b = blockIdx.y;
    const int tid = threadIdx.x, g = tid >> 5, lane = tid & 31;
    int seqlen = seqlens[b];
    seqlen = seqlen < 0 ? 0 : (seqlen > S_max ? S_max : seqlen);
    const ChunkPlan plan = chunk_plan(seqlen, chunk, win);
    const int ns = plan.n;   // chunks written for this sequence: splits plan.split(0 .. ns-1)
    const size_t row = (size_t)b * n_q + h;
    const float2 *ml = ws_ml + row * n_splits;
    // launched as a programmatic dependent of the split kernel: its partials
    // are complete and visible past this point
    griddep_wait();
    if (ns == 0) {
        for (int d = tid; d < DV; d += COMBINE_THREADS) o[row * DV + d] = __float2bfloat16_rn(0.f);
        if (tid == 0 && lse) lse[row] = -INFINITY;
        return;
    }
    // this group's chunks folded against its own running maximum Mg:
    // acc = sum 2^(m_s - Mg) o_s, L = sum 2^(m_s - Mg) l_s
    float4 acc[NQ];
#pragma unroll
    for (int qi = 0; qi < NQ; ++qi) acc[qi] = make_float4(0.f, 0.f, 0.f, 0.f);
    float Mg = -INFINITY, L = 0.f;
    const float *base = ws_o + row * n_splits * (size_t)DV + lane * 4;
#pragma unroll 8
    for (int c = g; c < ns; c += NG) {
        const int s = plan.split(c);
        const float2 m_l = ml[s];
        float4 v[NQ];
#pragma unroll
        for (int qi = 0; qi < NQ; ++qi) v[qi] = __ldg(reinterpret_cast<const float4 *>(base + (size_t)s * DV + qi * 128));
        const float m_new = fmaxf(Mg, m_l.x);
        const float a = Mg == -INFINITY ? 0.f : ex2(Mg - m_new);   // rescale of what came before
        const float w = ex2(m_l.x - m_new);
#pragma unroll
        for (int qi = 0; qi < NQ; ++qi) {
            acc[qi].x = fmaf(w, v[qi].x, acc[qi].x * a);
            acc[qi].y = fmaf(w, v[qi].y, acc[qi].y * a);
            acc[qi].z = fmaf(w, v[qi].z, acc[qi].z * a);
            acc[qi].w = fmaf(w, v[qi].w, acc[qi].w * a);
        }
        L = fmaf(w, m_l.y, L * a);
        Mg = m_new;
    }
#pragma unroll
    for (int qi = 0; qi < NQ; ++qi) *reinterpret_cast<float4 *>(&red[g][qi * 128 + lane * 4]) = acc[qi];
    if (lane == 0) {
        part_m[g] = Mg;
        part_l[g] = L;
    }
    __syncthreads();
    // the groups' sums rescaled to M = max over all chunks (a group without
    // chunks has Mg = -inf and weight 0)
    float M = -INFINITY;
#pragma unroll
    for (int k = 0; k < NG; ++k) M = fmaxf(M, part_m[k]);
    float sc[NG], Lt = 0.f;
#pragma unroll
    for (int k = 0; k < NG; ++k) {
        sc[k] = part_m[k] == -INFINITY ? 0.f : ex2(part_m[k] - M);
        Lt = fmaf(sc[k], part_l[k], Lt);
    }
    const float inv = 1.f / Lt;
    for (int d = tid; d < DV; d += COMBINE_THREADS) {
        float x = 0.f;
#pragma unroll
        for (int k = 0; k < NG; ++k) x = fmaf(sc[k], red[k][d], x);
        o[row * DV + d] = __float2bfloat16_rn(x * inv);
    }
    if (tid == 0 && lse) lse[row] = (M + log2f(Lt)) * 0.6931471805599453f;
}

}  // namespace dec
}  // namespace attn
