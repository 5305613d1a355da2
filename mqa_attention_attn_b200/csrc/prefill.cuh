// prefill.cuh -- fused tiled online-softmax attention forward (prefill) for
// sm_100a: TMA-staged Q/K/V tiles, tcgen05 MMAs with TMEM accumulators.
//
// Work split. A CTA owns two 128-row query tiles of one (batch b, KV head g):
//   * G = n_q/n_kv >= 2: each tile packs G/2 query heads x 256/G positions of
//     the group, the two tiles being the two halves of the group's heads at
//     the same positions. Every K/V tile is loaded once into shared memory and
//     multiplied against all G heads of the group: the grouped broadcast of
//     "Attention Engineering: From MHA to GQA, MLA & FlashAttention",
//     section 2 (no repeat_interleave, K/V read once per group).
//   * G = 1 (MHA): the two tiles are consecutive blocks of 128 positions.
// Both tiles stream the same K/V tiles (128 keys each): K through a 2-stage
// and V through a 3-stage ring, each fed by its own TMA warp; one MMA commit
// per iteration releases a V tile and the next K tile together.
//
// Per K/V tile j and query tile t the recurrence of the same page, section 4
// (FlashAttention-2 tiled rescaling) runs as:
//   MMA warp:      S_t = Q_t K_j^T        (tcgen05, fp32 in TMEM)
//   softmax WG t:  m' = max(m, rowmax S_t * scale*log2e)  (causal mask and
//                  the key-count bound applied only on tiles that cross them)
//                  P = 2^(S*scale*log2e - m') -> bf16 into TMEM over S_t
//                  l' = l * 2^(m - m') + rowsum P ; O_t *= 2^(m - m')
//   MMA warp:      O_t += P_t V_j         (A operand from TMEM)
// with two refinements that keep the result exact:
//   * the running maximum is only moved (and O rescaled) when the new tile
//     raises it by more than 2^8; otherwise the stale maximum is kept, which
//     bounds P by 256 and leaves O / l unchanged;
//   * key tiles right of a tile's last causal row are never visited
//     (causal tile skipping, "Attention, Worked Out by Hand (Part 2)",
//     section 2).
// The two query tiles ping-pong: while one softmax warpgroup exponentiates,
// the tensor core runs the other tile's MMAs. Epilogue: O / l -> bf16 ->
// swizzled shared memory -> TMA store; LSE = (m + log2 l) * ln 2.
//
// With rotary position embedding (the ROPE kernel), each softmax warpgroup
// first rotates its Q tile in shared memory, one row per thread (position
// Skv - Sq + i of query i), before the first S MMA of that tile; the keys
// arrive already rotated.
//
// Roles (384 threads): warps 0 and 2 TMA producers (Q and K; V), warp 1 MMA
// issuer and TMEM owner, warps 4-7 and 8-11 the softmax / epilogue
// warpgroups of tiles 0 and 1 (warp w reads TMEM lanes 32*(w%4) .. +31, so
// each warpgroup covers 128 rows).
#pragma once

#include "rope.cuh"
#include "sm100.cuh"

namespace attn {
namespace pf {

constexpr int BM = 128;        // query rows per tile (MMA M)
constexpr int BN = 128;        // keys per K/V tile (MMA N of Q K^T)
constexpr int KSTAGE = 2;       // K ring depth
constexpr int VSTAGE = 3;       // V ring depth
// One release barrier per K/V iteration i, completed by a single MMA commit
// once both tiles' P V of tile i and Q K^T of tile i+1 are done (this frees
// V tile i and K tile i+1). NREL >= max(KSTAGE, VSTAGE) keeps every producer
// within one phase of the barrier it waits on.
constexpr int NREL = 3;
static_assert(NREL >= KSTAGE && NREL >= VSTAGE, "release ring too short");
constexpr int THREADS = 384;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale only past a 256x growth
#ifndef ATTN_PF_P_CHUNKS
#define ATTN_PF_P_CHUNKS 1
#endif
#ifndef ATTN_PF_POLY_EVERY
#define ATTN_PF_POLY_EVERY 0
#endif
// P is handed to the MMA warp in kPChunks pieces of the 128 keys; every
// kPolyEvery-th exponential pair runs on the FMA pipe (0: none).
constexpr int kPChunks = ATTN_PF_P_CHUNKS;
constexpr int kPolyEvery = ATTN_PF_POLY_EVERY;
constexpr int kChunkKeys = BN / kPChunks;
static_assert(kPChunks == 1 || kPChunks == 2 || kPChunks == 4, "P hand-off chunks");
#ifndef ATTN_PF_EARLY_LOADS
#define ATTN_PF_EARLY_LOADS 1
#endif
#ifndef ATTN_PF_L2_PREFETCH
#define ATTN_PF_L2_PREFETCH 1
#endif
// kEarlyLoads: the thread that initialises the barriers issues the Q tiles and
// the first K tiles at once, before the block-wide setup barrier and the TMEM
// allocation. kL2Prefetch: it also prefetches into L2 the Q tiles of the CTA
// one wave later (dense batches). Measured on B200 at the Llama-3-8B prefill
// shape, the two take 3 % off the kernel time; storing O straight from
// registers instead of through shared memory and a TMA store was slower.
constexpr bool kEarlyLoads = ATTN_PF_EARLY_LOADS != 0;
constexpr bool kL2Prefetch = ATTN_PF_L2_PREFETCH != 0;
constexpr int kLaunchRegs = 168;            // registers per thread the kernel must be built with
constexpr int kRegsLow = 56;               // producer / MMA warpgroup after setmaxnreg.dec
constexpr int kRegsHigh = 224;              // softmax warpgroups after setmaxnreg.inc
static_assert(kRegsLow * 128 + kRegsHigh * 256 <= kLaunchRegs * THREADS, "register split exceeds the block");

template <int D>
struct Cfg {
    static constexpr int ROWB = (2 * D < 128) ? 2 * D : 128;   // bytes per shared row of one box
    static constexpr int BOXD = ROWB / 2;                        // elements per box row
    static constexpr int NBOX = D / BOXD;
    static constexpr int SWB = ROWB == 128 ? 3 : (ROWB == 64 ? 2 : 1);
    static constexpr uint32_t LAYOUT = ROWB == 128 ? 2u : (ROWB == 64 ? 4u : 6u);
    static constexpr int QBYTES = BM * D * 2;
    static constexpr int KBYTES = BN * D * 2;
    static constexpr int QBOX = BM * ROWB;
    static constexpr int KBOX = BN * ROWB;
    static constexpr int ATOM = 8 * ROWB;                        // 8-row swizzle atom
    static constexpr uint32_t TMEM_COLS = 512;
    // TMEM columns: S (and P over its first half) of tile t, then O of tile t
    __device__ static constexpr uint32_t col_s(int t) { return (uint32_t)t * 128u; }
    __device__ static constexpr uint32_t col_o(int t) { return 256u + (uint32_t)t * (uint32_t)D; }
    static_assert(D == 32 || D == 64 || D == 128, "head dim");
};

template <int D>
struct Smem {
    uint8_t q[2][Cfg<D>::QBYTES];          // Q tiles; reused as O staging in the epilogue
    uint8_t k[KSTAGE][Cfg<D>::KBYTES];
    uint8_t v[VSTAGE][Cfg<D>::KBYTES];
    uint64_t q_full;
    uint64_t k_full[KSTAGE], v_full[VSTAGE];
    uint64_t rel[NREL];
    uint64_t s_full[2];
    uint64_t p_full[2][kPChunks];  // one per hand-off chunk of P
    uint64_t o_done[2];
    uint64_t mma_done;
    uint64_t v_tail;               // PAGED: the copy of the tile holding the last key (cleared past it)
    uint64_t q_rot[2];             // ROPE: Q tile t rotated in place
    uint32_t tmem_base;
    int abort_flag;
};

template <int D>
constexpr size_t smem_bytes() {
    // at least ~116 KB so that one CTA (which takes all 512 TMEM columns)
    // owns an SM
    size_t s = sizeof(Smem<D>) + 1024;
    return s < 118784 ? 118784 : s;
}
static_assert(smem_bytes<32>() <= kMaxSmemPerCta && smem_bytes<64>() <= kMaxSmemPerCta &&
                  smem_bytes<128>() <= kMaxSmemPerCta,
              "prefill shared memory exceeds a CTA's");

struct Params {
    int B, Sq, Skv, n_q, n_kv, G;
    int Ht, Pt;            // heads and positions per query tile (Ht * Pt = 128)
    int pair_by_heads;     // 1: tiles = two head halves at one position block
    int n_pb;              // position blocks per (b, kv head) (varlen: of the longest sequence)
    int causal;
    float scale_log2;      // scale * log2(e)
    float *lse;            // may be null
    // Packed variable-length batch (the VARLEN kernel): q [total_q][n_q][D],
    // k, v [total_k][n_kv][D], o like q, lse [n_q][total_q]; sequence b owns
    // rows cu_q[b] .. cu_q[b+1]-1 (queries) and cu_k[b] .. cu_k[b+1]-1 (keys).
    // A query tile's rows are then position-major (row = position * Ht +
    // head) instead of head-major.
    const int32_t *cu_q, *cu_k;
    int total_q, total_k;
    // Sliding window (the WINDOW kernel, causal): a query at position p sees
    // key j iff j <= p and (p - j < window or j < n_sink).
    int window, n_sink;
    // Rotary tables (the ROPE kernel): cos/sin [n_pos][D/2], n_pos >= Skv.
    rope::Tables rope;
    // Paged cache (the PAGED kernel: queries packed as in VARLEN): sequence b
    // has seqlens_k[b] cached tokens; token j lives in row j % page_size of
    // page block_table[b * pages_per_seq + j / page_size] of the pools the K
    // and V tensor maps address ([page][token][kv head][dim]); a 128-key tile
    // is 128 / box_rows TMA boxes, box_rows = min(page_size, 128).
    const int32_t *block_table, *seqlens_k;
    int pages_per_seq, page_shift, box_rows, num_pages;
    __nv_bfloat16 *o;      // varlen: rows of a tile that ends past its sequence are stored directly
    // Dense batch: the CTA this many launch slots later has its Q tiles
    // prefetched into L2 by this one (0: none). With one CTA per SM and the
    // grid taken in index order, that CTA starts once this wave drains.
    int l2_ahead;
    // FP8 inputs (the FP8 kernel, BHSD as the dense one): the q map reads
    // the e4m3 bytes (one 128-byte box per row), k and v hold the e4m3
    // values widened to bf16 (exact); element (b, h, i, c) means
    // value * scale[b][h][i / 128] with q_scale [B][n_q][q_tiles] and
    // k_scale, v_scale [B][n_kv][k_tiles].
    const float *q_scale, *k_scale, *v_scale;
    int q_tiles, k_tiles;
};

template <bool B>
struct BoolTag {
    static constexpr bool value = B;
};

// All 32 lanes wait; the outcome is made warp-uniform.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          uint32_t site) {
    bool ok = mbar_wait(bar, parity, abort_flag, site);
    ok = __all_sync(0xffffffffu, ok);
    return ok;
}

// MODE: kDense (BHSD batch), kVarlen (packed batch), kWindow (BHSD, causal
// sliding window with sink keys), kRope (BHSD batch, queries rotated here),
// kPaged (packed queries, keys and values in a paged cache), kFp8 (BHSD
// batch of e4m3 values widened to bf16, one scale per 128-row tile: the
// query and key tile scales folded into the exponent's scale, the value
// tile's scale into P).
enum : int { kDense = 0, kVarlen = 1, kWindow = 2, kRope = 3, kPaged = 4, kFp8 = 5 };

// One 128-key tile of a paged K or V pool into shared memory (the PAGED
// kernel): box x of the tile holds keys key0 + x * box_rows .. + box_rows - 1,
// read from their page through the block table. Boxes at or past the
// sequence's length read an out-of-range page, which TMA fills with zeros,
// so every row of the tile holds finite values (rows past the length get
// weight 0, and 0 * NaN would not be 0); a page id outside the pool reads as
// zeros too and is reported. The barrier expects the whole tile.
template <int NBOX, int BOXD, int KBOX, int ROWB>
__device__ __forceinline__ void load_paged_tile(uint32_t dst, const CUtensorMap *tm, uint32_t bar, const Params &p,
                                                int b, int kvh, int key0, int Skv) {
    const int nbox = BN / p.box_rows;
    const uint32_t box_bytes = (uint32_t)p.box_rows * ROWB;
    const int32_t *row_pages = p.block_table + (size_t)b * p.pages_per_seq;
    for (int x = 0; x < nbox; ++x) {
        const int key = key0 + x * p.box_rows;
        int page = p.num_pages;                        // past the length: zeros
        if (key < Skv) {
            page = row_pages[key >> p.page_shift];
            if ((unsigned)page >= (unsigned)p.num_pages) atomicOr(&g_status, kStatusRange);
        }
        const int prow = key & ((1 << p.page_shift) - 1);
#pragma unroll
        for (int bx = 0; bx < NBOX; ++bx)
            tma_load_4d(dst + bx * KBOX + x * box_bytes, tm, bar, bx * BOXD, prow, kvh, page);
    }
}

template <int D, int MODE>
__global__ void __launch_bounds__(THREADS, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
               const Params p) {
    using C = Cfg<D>;
    constexpr bool VARLEN = MODE == kVarlen;
    constexpr bool PAGED = MODE == kPaged;
    constexpr bool PACKED = VARLEN || PAGED;      // queries packed [total_q][n_q][D]
    constexpr bool WINDOW = MODE == kWindow;
    constexpr bool ROPE = MODE == kRope;
    constexpr bool FP8 = MODE == kFp8;
    static_assert(!FP8 || D == 128, "the FP8 mode stages one 128-byte e4m3 row per query row");
    extern __shared__ uint8_t smem_raw[];
    Smem<D> &sm = *reinterpret_cast<Smem<D> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const uint32_t warp = warp_id(), lane = lane_id();

    // ---- work unit: (b, kv head, position block), heaviest causal blocks first
    int b, kvh, pb;
    int Sq = p.Sq, Skv = p.Skv, q0 = 0, k0 = 0;   // this sequence's sizes and first rows (varlen)
    if (PACKED) {
        b = blockIdx.y;
        kvh = blockIdx.x % p.n_kv;
        pb = p.n_pb - 1 - (int)(blockIdx.x / p.n_kv);
        q0 = p.cu_q[b];
        Sq = p.cu_q[b + 1] - q0;
        bool bad = q0 < 0 || Sq < 0 || q0 + Sq > p.total_q || Sq > p.n_pb * (p.pair_by_heads ? p.Pt : 2 * p.Pt);
        if (VARLEN) {
            k0 = p.cu_k[b];
            Skv = p.cu_k[b + 1] - k0;
            bad = bad || k0 < 0 || Skv < 0 || k0 + Skv > p.total_k;
        } else {
            // the cached tokens of the sequence, at most what its pages hold
            Skv = p.seqlens_k[b];
            const int cap = p.pages_per_seq << p.page_shift;
            if (Skv > cap) {
                if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(&g_status, kStatusRange);
                Skv = cap;
            }
            if (Skv < 0) Skv = 0;
        }
        if (bad) {
            if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(&g_status, kStatusRange);
            Sq = 0;   // malformed offsets: this sequence is skipped
        }
    } else {
        const int nbh = p.B * p.n_kv;
        const int bh = blockIdx.x % nbh;
        pb = p.n_pb - 1 - (int)(blockIdx.x / nbh);
        b = bh / p.n_kv;
        kvh = bh % p.n_kv;
    }
    // query tile t of a unit: first head and first position
    auto tile_origin = [&](int kvh_, int pb_, int t, int &h0_, int &p0_) {
        if (p.pair_by_heads) {
            h0_ = kvh_ * p.G + t * p.Ht;
            p0_ = pb_ * p.Pt;
        } else {
            h0_ = kvh_;  // G == 1: query head == KV head
            p0_ = pb_ * 2 * p.Pt + t * p.Pt;
        }
    };
    int h0[2], p0[2], nt[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        tile_origin(kvh, pb, t, h0[t], p0[t]);
        if (p0[t] >= Sq) {
            nt[t] = 0;
        } else {
            const int last = min(p0[t] + p.Pt, Sq) - 1;
            const int keys = p.causal ? min(Skv, last + (Skv - Sq) + 1) : Skv;
            nt[t] = keys > 0 ? (keys + BN - 1) / BN : 0;   // 0: no row of the tile sees a key
        }
    }
    // Key tiles visited, as iterations j = 0, 1, ...: normally key tile j. With
    // a window: the tiles holding sink keys, then the tiles from the first
    // window of the CTA's earliest row (tile 0's first position) up to each
    // tile's last causal key; tiles between sinks and window are skipped.
    int nsk = 0, jw0 = 0;
    if constexpr (WINDOW) {
        nsk = (min(p.n_sink, Skv) + BN - 1) / BN;
        const int lo = max(0, p0[0] + (Skv - Sq) - p.window + 1);   // first key of any row's window
        jw0 = max(lo / BN, nsk);
#pragma unroll
        for (int t = 0; t < 2; ++t)
            if (nt[t] > 0) nt[t] = nsk + max(0, nt[t] - jw0);
    }
    auto key_tile = [&](int j) { return (WINDOW && j >= nsk) ? jw0 + (j - nsk) : j; };
    const int nmax = max(nt[0], nt[1]);

    // Q tiles of this unit, all on q_full
    auto load_q = [&]() {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_o);
        uint32_t qbytes = 0;
        for (int t = 0; t < 2; ++t)
            if (nt[t] > 0) qbytes += FP8 ? BM * D : C::QBYTES;
        const uint32_t qbar = smem_u32(&sm.q_full);
        mbar_arrive_expect_tx(qbar, qbytes);
        for (int t = 0; t < 2; ++t) {
            if (nt[t] == 0) continue;
            if constexpr (FP8) {
                // the tile's e4m3 rows (128 one-byte dims, 128-byte swizzled)
                // into its second box, widened in place by its warpgroup
                tma_load_3d(smem_u32(sm.q[t]) + C::QBOX, &tm_q, qbar, 0, p0[t], b * p.n_q + h0[t]);
                continue;
            }
            for (int bx = 0; bx < C::NBOX; ++bx)
                if (PACKED)
                    tma_load_3d(smem_u32(sm.q[t]) + bx * C::QBOX, &tm_q, qbar, bx * C::BOXD, h0[t], q0 + p0[t]);
                else
                    tma_load_3d(smem_u32(sm.q[t]) + bx * C::QBOX, &tm_q, qbar, bx * C::BOXD, p0[t],
                                b * p.n_q + h0[t]);
        }
    };
    // K tile of iteration j into its stage (the stage must be free)
    auto load_k = [&](int j) {
        const int s = j % KSTAGE;
        const uint32_t fb = smem_u32(&sm.k_full[s]);
        mbar_arrive_expect_tx(fb, C::KBYTES);
        if (PAGED)
            load_paged_tile<C::NBOX, C::BOXD, C::KBOX, C::ROWB>(smem_u32(sm.k[s]), &tm_k, fb, p, b, kvh, j * BN, Skv);
        else
            for (int bx = 0; bx < C::NBOX; ++bx)
                if (VARLEN)
                    tma_load_3d(smem_u32(sm.k[s]) + bx * C::KBOX, &tm_k, fb, bx * C::BOXD, kvh, k0 + j * BN);
                else
                    tma_load_3d(smem_u32(sm.k[s]) + bx * C::KBOX, &tm_k, fb, bx * C::BOXD, key_tile(j) * BN,
                                b * p.n_kv + kvh);
    };
    // K tiles issued during setup (ROPE: the rotated keys come from the grid
    // launched just before this one, so its K tiles wait in the producer;
    // PAGED: the page lookups issued here spill in the producer's registers)
    const int k_early = (kEarlyLoads && !ROPE && !PAGED && !FP8) ? min(KSTAGE, nmax) : 0;

    // ---- setup: barriers (warp 0), TMEM (warp 1)
    if (warp == 0 && lane == 0) {
        mbar_init(smem_u32(&sm.q_full), 1);
        for (int s = 0; s < KSTAGE; ++s) mbar_init(smem_u32(&sm.k_full[s]), 1);
        for (int s = 0; s < VSTAGE; ++s) mbar_init(smem_u32(&sm.v_full[s]), 1);
        for (int s = 0; s < NREL; ++s) {
            mbar_init(smem_u32(&sm.rel[s]), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(smem_u32(&sm.s_full[t]), 1);
            for (int c = 0; c < kPChunks; ++c) mbar_init(smem_u32(&sm.p_full[t][c]), 128);
            mbar_init(smem_u32(&sm.o_done[t]), 1);
        }
        mbar_init(smem_u32(&sm.mma_done), 1);
        mbar_init(smem_u32(&sm.v_tail), 1);
        for (int t = 0; t < 2; ++t) mbar_init(smem_u32(&sm.q_rot[t]), 128);
        sm.abort_flag = 0;
        fence_mbar_init();
        if constexpr (kEarlyLoads) {
            load_q();
            for (int j = 0; j < k_early; ++j) load_k(j);
        }
        if (kL2Prefetch && !PACKED && p.l2_ahead > 0 && blockIdx.x + (unsigned)p.l2_ahead < gridDim.x) {
            // Q tiles of a unit that starts later, into L2
            const unsigned f = blockIdx.x + (unsigned)p.l2_ahead;
            const int nbh = p.B * p.n_kv;
            const int fbh = (int)(f % (unsigned)nbh);
            const int fpb = p.n_pb - 1 - (int)(f / (unsigned)nbh);
            for (int t = 0; t < 2; ++t) {
                int fh0, fp0;
                tile_origin(fbh % p.n_kv, fpb, t, fh0, fp0);
                if (fp0 >= Sq) continue;
                for (int bx = 0; bx < (FP8 ? 1 : C::NBOX); ++bx)
                    tma_prefetch_l2_3d(&tm_q, bx * C::BOXD, fp0, (fbh / p.n_kv) * p.n_q + fh0);
            }
        }
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&sm.tmem_base), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort_flag = &sm.abort_flag;

    // Register split: the producer / MMA warpgroup needs few registers, the
    // softmax warpgroups hold a 128-key row of S each. 56*128 + 224*256 =
    // 168*384, the block's registers at launch (the host refuses to launch
    // unless the kernel was built with exactly kLaunchRegs per thread).
    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
    if (warp == 0) {
        // ======================= TMA producer =======================
        if (lane == 0) {
            const uint32_t qbar = smem_u32(&sm.q_full);
            if constexpr (!kEarlyLoads) load_q();
            // K tiles (V tiles are loaded by warp 2). ROPE: the rotated keys come
            // from the grid launched just before this one
            // FP8: the widened keys come from the grid launched just before
            if (ROPE || FP8) griddep_wait();
            int issued = k_early;
            for (int j = k_early; j < nmax; ++j) {
                // K tile j - KSTAGE is free once iteration j - KSTAGE - 1 is released
                // (K tile 0 with iteration 0)
                const int it = j - KSTAGE - 1 < 0 ? 0 : j - KSTAGE - 1;
                if (j >= KSTAGE &&
                    !mbar_wait(smem_u32(&sm.rel[it % NREL]), (it / NREL) & 1, abort_flag, 0x11))
                    break;
                load_k(j);
                ++issued;
            }
            // never leave copies in flight into this CTA's shared memory
            mbar_wait(qbar, 0, nullptr, 0x12);
            for (int j = issued - 1; j >= 0 && j >= issued - KSTAGE; --j)
                mbar_wait(smem_u32(&sm.k_full[j % KSTAGE]), (j / KSTAGE) & 1, nullptr, 0x13);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ======================= TMA producer (V tiles) =======================
        // PAGED: the visited tile that ends past the last cached key (-1: none)
        const int tail_tile = (PAGED && Skv % BN != 0 && (Skv - 1) / BN < nmax) ? (Skv - 1) / BN : -1;
        int issued = 0;
        if (lane == 0) {
            if (FP8) griddep_wait();   // the widened values, likewise
            for (int j = 0; j < nmax; ++j) {
                const int s = j % VSTAGE;
                // V tile j - VSTAGE is free once iteration j - VSTAGE is released
                const int it = j - VSTAGE;
                if (j >= VSTAGE &&
                    !mbar_wait(smem_u32(&sm.rel[it % NREL]), (it / NREL) & 1, abort_flag, 0x14))
                    break;
                // PAGED: the tile holding the last key lands on v_tail instead;
                // v_full of its stage is completed below, after the clearing
                const uint32_t fb = smem_u32((PAGED && j == tail_tile) ? &sm.v_tail : &sm.v_full[s]);
                mbar_arrive_expect_tx(fb, C::KBYTES);
                if (PAGED)
                    load_paged_tile<C::NBOX, C::BOXD, C::KBOX, C::ROWB>(smem_u32(sm.v[s]), &tm_v, fb, p, b, kvh, j * BN,
                                                                      Skv);
                else
                for (int bx = 0; bx < C::NBOX; ++bx)
                    if (VARLEN)
                        tma_load_3d(smem_u32(sm.v[s]) + bx * C::KBOX, &tm_v, fb, bx * C::BOXD, kvh, k0 + j * BN);
                    else
                        tma_load_3d(smem_u32(sm.v[s]) + bx * C::KBOX, &tm_v, fb, bx * C::BOXD, key_tile(j) * BN,
                                    b * p.n_kv + kvh);
                ++issued;
            }
        }
        issued = __shfl_sync(0xffffffffu, issued, 0);
        if constexpr (PAGED) {
            // The tile holding the sequence's last key may hold rows past the
            // length (a page's unused slots, whatever they contain): they get
            // weight 0, but 0 * (NaN or Inf) is not 0, so this warp clears
            // them once the tile has landed, then completes the stage's v_full
            // (a plain arrival: the copy's bytes were counted on v_tail).
            const int jt = tail_tile;
            if (jt >= 0 && jt < issued) {
                const int s = jt % VSTAGE;
                const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.v_tail), 0, abort_flag, 0x16));
                if (ok) {
                    const int rows = Skv - jt * BN;             // valid rows of the tile
                    constexpr int CPR = C::ROWB / 16;             // 16-byte chunks per box row
                    for (int e = rows * CPR + (int)lane; e < BN * CPR; e += 32)
#pragma unroll
                        for (int bx = 0; bx < C::NBOX; ++bx)
                            sts128(smem_u32(sm.v[s]) + bx * C::KBOX + (uint32_t)e * 16u, make_uint4(0u, 0u, 0u, 0u));
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0 && ok) mbar_arrive(smem_u32(&sm.v_full[s]));
            }
        }
        if (lane == 0) {
            // never leave copies in flight into this CTA's shared memory
            for (int j = issued - 1; j >= 0 && j >= issued - VSTAGE; --j)
                mbar_wait(smem_u32((PAGED && j == tail_tile) ? &sm.v_tail : &sm.v_full[j % VSTAGE]),
                          (PAGED && j == tail_tile) ? 0 : (j / VSTAGE) & 1, nullptr, 0x15);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ======================= MMA issuer =======================
        if (lane == 0) {
            const uint32_t idesc_s = umma_idesc_bf16(BM, BN, 0, 0);
            const uint32_t idesc_o = umma_idesc_bf16(BM, D, 0, 1);
            bool ok = mbar_wait(smem_u32(&sm.q_full), 0, abort_flag, 0x21);
            // Descriptors are built once per operand tile and stepped by
            // constant offsets in their 16-byte address field: for shared
            // addresses a, o (multiples of 16, a + o < 2^18, so the 14-bit
            // field cannot carry) desc(a + o) = desc(a) + (o >> 4). The base
            // passes through a volatile move so that it is formed where it is
            // used, not hoisted with all its offsets into registers (this
            // warp runs on 56).
            auto issue_s = [&](int t, int j) {
                const int s = j % KSTAGE;
                const uint64_t qd0 = pin_u64(umma_smem_desc(smem_u32(sm.q[t]), 16, C::ATOM, C::LAYOUT));
                const uint64_t kd0 = pin_u64(umma_smem_desc(smem_u32(sm.k[s]), 16, C::ATOM, C::LAYOUT));
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const int kel = ks * 16;
                    const uint32_t off_q = (kel / C::BOXD) * C::QBOX + (kel % C::BOXD) * 2;
                    const uint32_t off_k = (kel / C::BOXD) * C::KBOX + (kel % C::BOXD) * 2;
                    // (the varlen instance builds each descriptor in full: with
                    // the offset form its register allocation spills)
                    if constexpr (PACKED)
                        umma_ss(tmem + C::col_s(t), umma_smem_desc(smem_u32(sm.q[t]) + off_q, 16, C::ATOM, C::LAYOUT),
                                umma_smem_desc(smem_u32(sm.k[s]) + off_k, 16, C::ATOM, C::LAYOUT), idesc_s, ks > 0 ? 1u : 0u);
                    else
                        umma_ss(tmem + C::col_s(t), qd0 + (uint64_t)(off_q >> 4), kd0 + (uint64_t)(off_k >> 4), idesc_s,
                                ks > 0 ? 1u : 0u);
                }
                umma_commit(smem_u32(&sm.s_full[t]));
            };
            // O_t += P_t V_j, 32 keys at a time as soon as the softmax
            // warpgroup has written that chunk of P
            auto issue_pv = [&](int t, int j) -> bool {
                const int s = j % VSTAGE;
                const uint64_t vd0 = pin_u64(umma_smem_desc(smem_u32(sm.v[s]), C::KBOX, C::ATOM, C::LAYOUT));
#pragma unroll
                for (int c = 0; c < kPChunks; ++c) {
                    if (!mbar_wait(smem_u32(&sm.p_full[t][c]), j & 1, abort_flag, 0x23)) return false;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kChunkKeys / 16; ++kk) {
                        const int ks = c * (kChunkKeys / 16) + kk;
                        umma_ts(tmem + C::col_o(t), tmem + C::col_s(t) + ks * 8,
                                vd0 + (uint64_t)((uint32_t)(ks * 16 * C::ROWB) >> 4), idesc_o,
                                (j > 0 || ks > 0) ? 1u : 0u);
                    }
                }
                if (j == nt[t] - 1) umma_commit(smem_u32(&sm.o_done[t]));   // O_t final
                return true;
            };
            if (ok && nmax > 0) {
                ok = mbar_wait(smem_u32(&sm.k_full[0]), 0, abort_flag, 0x22);
                if (ok) {
                    tc_fence_after();
                    for (int t = 0; t < 2 && ok; ++t) {
                        if (nt[t] == 0) continue;
                        // ROPE: this tile's rows have been rotated in place;
                        // FP8: widened to bf16 in place
                        if (ROPE || FP8) ok = mbar_wait(smem_u32(&sm.q_rot[t]), 0, abort_flag, 0x27);
                        if (!ok) break;
                        tc_fence_after();
                        issue_s(t, 0);
                    }
                }
            }
            for (int j = 0; ok && j < nmax; ++j) {
                // operands of this iteration (V tile j, K tile j+1), checked up
                // front so that no wait sits between the MMA groups below
                ok = mbar_wait(smem_u32(&sm.v_full[j % VSTAGE]), (j / VSTAGE) & 1, abort_flag, 0x26);
                if (ok && j + 1 < nmax)
                    ok = mbar_wait(smem_u32(&sm.k_full[(j + 1) % KSTAGE]), ((j + 1) / KSTAGE) & 1, abort_flag,
                                   0x24);
                tc_fence_after();
                for (int t = 0; t < 2 && ok; ++t) {
                    if (j >= nt[t]) continue;
                    ok = issue_pv(t, j);
                    if (!ok) break;
                    if (j + 1 < nt[t]) issue_s(t, j + 1);
                }
                // P V of tile j and Q K^T of tile j+1 issued for both tiles
                umma_commit(smem_u32(&sm.rel[j % NREL]));
            }
            // all MMAs of this CTA done before TMEM can be released
            umma_commit(smem_u32(&sm.mma_done));
            mbar_wait(smem_u32(&sm.mma_done), 0, nullptr, 0x25);
        }
        __syncwarp();
    }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
        // ================== softmax + epilogue warpgroups ==================
        const int t = (int)(warp - 4) / 4;
        const uint32_t quad = warp & 3u;
        const int r = (int)(quad * 32 + lane);          // row of the tile = TMEM lane
        if (p0[t] < Sq) {
            const int hl = PACKED ? r % p.Ht : r / p.Pt;
            const int pl = PACKED ? r / p.Ht : r % p.Pt;
            const int pos = p0[t] + pl;
            const int head = h0[t] + hl;
            if constexpr (ROPE) {
                // rotate the Q tile in place, each row at its absolute position
                // (row's position in the tile: row % Pt, the tile being head-major);
                // the angles are fetched while the tile is still in flight
                rope::RopeTile<D, C::ROWB> rt;
                const int pmask = p.Pt - 1;                 // Pt is a power of two
                const int pbase = p0[t] + (Skv - Sq), last = Skv - 1;
                rt.fetch(p.rope, r, [&](int row) { return min(pbase + (row & pmask), last); });
                if (warp_wait(smem_u32(&sm.q_full), 0, abort_flag, 0x36)) {
                    const int pend = Sq - p0[t];   // rows at positions >= Sq hold no query
                    rt.apply(smem_u32(sm.q[t]), C::QBOX, r, [&](int row) { return (row & pmask) < pend; });
                    fence_proxy_async_smem();
                }
                mbar_arrive(smem_u32(&sm.q_rot[t]));
            }
            if constexpr (FP8) {
                // widen this row's e4m3 query values (staged in the tile's
                // second box) to bf16 in the layout the score MMAs read. A
                // row's 128 staged bytes and its 128 bf16 bytes of the second
                // box are the same 128-byte row (the swizzle permutes chunks
                // within a row), so each thread reads its dims 64-127 before
                // writing them back and no thread touches another's row.
                const uint32_t qt = smem_u32(sm.q[t]);
                if (warp_wait(smem_u32(&sm.q_full), 0, abort_flag, 0x37)) {
                    auto get = [&](int c) { return lds128(qt + C::QBOX + swz<3>((uint32_t)(r * 128 + c * 16))); };
                    auto put = [&](int c, const uint4 &x) {   // e4m3 chunk c = dims 16c .. 16c + 15
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            const int e0 = 16 * c + 8 * hf;
                            const int bx = e0 / C::BOXD, ci = (e0 % C::BOXD) / 8;
                            const uint4 w = hf ? e4m3x8_to_bf16x8(x.z, x.w) : e4m3x8_to_bf16x8(x.x, x.y);
                            sts128(qt + bx * C::QBOX + swz<C::SWB>((uint32_t)(r * C::ROWB + ci * 16)), w);
                        }
                    };
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) put(c, get(c));
                    uint4 hi[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) hi[c] = get(4 + c);
#pragma unroll
                    for (int c = 0; c < 4; ++c) put(4 + c, hi[c]);
                    fence_proxy_async_smem();
                }
                mbar_arrive(smem_u32(&sm.q_rot[t]));
            }
            int lim = p.causal ? pos + (Skv - Sq) : Skv - 1;   // last visible key (< 0: none)
            lim = min(lim, Skv - 1);
            const uint32_t trow = tmem + ((quad * 32u) << 16);
            const uint32_t colS = C::col_s(t), colO = C::col_o(t);
            const float sl = p.scale_log2;
            float m_run = -INFINITY, l_run = 0.f;
            bool ok = true;
            const int ntt = nt[t];
            // FP8: this row's query tile scale (rows past Sq hold no query)
            const float qsr = (FP8 && pos < Sq)
                                  ? __ldg(p.q_scale + ((size_t)b * p.n_q + head) * p.q_tiles + pos / BM) : 1.f;
            const size_t kvsrow = FP8 ? ((size_t)b * p.n_kv + kvh) * p.k_tiles : 0;
            // FP8: key and value tile scales, loaded one tile ahead
            float ks_next = (FP8 && ntt > 0) ? __ldg(p.k_scale + kvsrow) : 1.f;
            float vs_next = (FP8 && ntt > 0) ? __ldg(p.v_scale + kvsrow) : 1.f;
            for (int j = 0; j < ntt; ++j) {
                const float ksj = ks_next, vsj = vs_next;
                if (FP8 && j + 1 < ntt) {
                    ks_next = __ldg(p.k_scale + kvsrow + j + 1);
                    vs_next = __ldg(p.v_scale + kvsrow + j + 1);
                }
                ok = warp_wait(smem_u32(&sm.s_full[t]), j & 1, abort_flag, 0x31);
                if (!ok) break;
                __syncwarp();
                tc_fence_after();
                // the whole 128-key row of S in registers (four loads, one wait)
                uint32_t x[BN];
#pragma unroll
                for (int c = 0; c < BN / 32; ++c)
                    tmem_ld32(trow + colS + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&x[32 * c]));
                tmem_wait_ld();
                const int kbase = key_tile(j) * BN;
                // causal / key-count mask: only on tiles that cross some row's limit
                bool cut = kbase + BN - 1 > lim;
                // window: keys left of the row's window that are not sink keys
                const int wlo = WINDOW ? lim - p.window + 1 : 0;
                if constexpr (WINDOW) cut = cut || (kbase < wlo && kbase + BN > p.n_sink);
                const bool masked = __any_sync(0xffffffffu, cut);
                if (masked) {
                    const int rem = lim - kbase;
#pragma unroll
                    for (int e = 0; e < BN; ++e)
                        if (e > rem) x[e] = 0xff800000u;   // -inf
                    if constexpr (WINDOW) {
                        const int rem_lo = wlo - kbase, rem_sink = p.n_sink - kbase;
#pragma unroll
                        for (int e = 0; e < BN; ++e)
                            if (e < rem_lo && e >= rem_sink) x[e] = 0xff800000u;
                    }
                }
                // row maximum (four independent 3-input max chains)
                float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
                for (int e = 0; e < BN; e += 8) {
                    mx0 = fmax3(mx0, __uint_as_float(x[e + 0]), __uint_as_float(x[e + 1]));
                    mx1 = fmax3(mx1, __uint_as_float(x[e + 2]), __uint_as_float(x[e + 3]));
                    mx2 = fmax3(mx2, __uint_as_float(x[e + 4]), __uint_as_float(x[e + 5]));
                    mx3 = fmax3(mx3, __uint_as_float(x[e + 6]), __uint_as_float(x[e + 7]));
                }
                const float mx = fmaxf(fmax3(mx0, mx1, mx2), mx3);
                // scale * log2(e), times the query and key tile scales (FP8)
                const float slj = FP8 ? sl * qsr * ksj : sl;
                const float2 sl2 = make_float2(slj, slj);
                const float m_new = fmaxf(m_run, mx * slj);
                if (j == 0) {
                    m_run = m_new;
                } else if (__any_sync(0xffffffffu, m_new > m_run + kRescaleThreshold)) {
                    // move the running maximum: rescale this row's O and l
                    // O is stable here: s_full for tile j was committed after
                    // the P.V MMA of tile j-1, and a commit tracks every MMA
                    // issued before it.
                    const float alpha = ex2(m_run - m_new);
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {   // 32 columns at a time: S stays in registers
                        uint32_t o[32];
                        tmem_ld32(trow + colO + 32 * c, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(trow + colO + 32 * c, o);
                    }
                    tmem_wait_st();
                    l_run *= alpha;
                    m_run = m_new;
                }
                // P = 2^(s*scale*log2e - m) -> bf16 pairs over the first half of S,
                // handed to the MMA warp in kPChunks pieces (kPChunks > 1 lets P.V
                // start on the first keys while later ones are still
                // exponentiated; measured on B200 one hand-off is faster, the
                // extra barrier round trips cost more than the overlap gains).
                // Optionally (kPolyEvery > 0) part of the exponentials run on the
                // FMA pipe (ex2_poly2) beside the special-function unit; measured
                // on B200 this is slower for head dim 128 (the softmax is bound
                // by issue and latency, not by the special-function unit), so it
                // is off by default.
                // a row with no visible key yet keeps m = -inf: exponentiate
                // against 0 instead (every p is then 0)
                const float m_use = ((PACKED || WINDOW) && m_run == -INFINITY) ? 0.f : m_run;
                // FP8: the value tile's scale joins the exponent (P is formed
                // already multiplied by it; the row sum divides it out per tile)
                const float lvs = FP8 ? __log2f(vsj) : 0.f;
                const float2 nm2 = make_float2(lvs - m_use, lvs - m_use);
                float2 rs = make_float2(0.f, 0.f);
                // one chunk of exponentials; which pairs take the FMA-pipe
                // polynomial is fixed at compile time (never on masked tiles)
                auto exp_chunk = [&](auto poly_on, int c, uint32_t(&pk)[kChunkKeys / 2]) {
#pragma unroll
                    for (int e = 0; e < kChunkKeys / 2; ++e) {
                        const int i0 = c * kChunkKeys + 2 * e;
                        const float2 t2 = ffma2(make_float2(__uint_as_float(x[i0]), __uint_as_float(x[i0 + 1])),
                                                sl2, nm2);
                        float2 pe;
                        if constexpr (decltype(poly_on)::value && kPolyEvery > 0) {
                            if (e % (kPolyEvery > 0 ? kPolyEvery : 1) == (kPolyEvery > 0 ? kPolyEvery - 1 : 0))
                                pe = ex2_poly2(t2);
                            else
                                pe = make_float2(ex2(t2.x), ex2(t2.y));
                        } else {
                            pe = make_float2(ex2(t2.x), ex2(t2.y));
                        }
                        rs = fadd2(rs, pe);
                        pk[e] = f2_to_bf2(pe.x, pe.y);   // FP8: times the value tile's scale
                    }
                };
#pragma unroll
                for (int c = 0; c < kPChunks; ++c) {
                    uint32_t pk[kChunkKeys / 2];
                    if (masked || kPolyEvery == 0)
                        exp_chunk(BoolTag<false>{}, c, pk);
                    else
                        exp_chunk(BoolTag<true>{}, c, pk);
#pragma unroll
                    for (int q = 0; q < kChunkKeys / 64; ++q)
                        tmem_st32(trow + colS + c * (kChunkKeys / 2) + 32 * q,
                                  *reinterpret_cast<uint32_t(*)[32]>(&pk[32 * q]));
                    if constexpr (kChunkKeys == 32)
                        tmem_st16(trow + colS + c * 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(smem_u32(&sm.p_full[t][c]));
                }
                l_run += FP8 ? (rs.x + rs.y) * __frcp_rn(vsj) : rs.x + rs.y;
            }
            // ---- epilogue: O / l -> bf16 -> swizzled smem -> TMA store; LSE
            if (ok && ntt > 0) ok = warp_wait(smem_u32(&sm.o_done[t]), 0, abort_flag, 0x33);
            __syncwarp();
            tc_fence_after();
            // a row that saw no key: O = 0, LSE = -inf (the empty sum)
            const float inv_l = (!PACKED || l_run > 0.f) ? 1.f / l_run : 0.f;
            const uint32_t stage = smem_u32(sm.q[t]);
            // varlen: a tile reaching past its sequence's last query is stored
            // row by row (TMA would write into the next sequence's rows)
            const bool direct = PACKED && p0[t] + p.Pt > Sq;
            {
                uint32_t o[D];
                if (ntt > 0) {
#pragma unroll
                    for (int c = 0; c < D / 32; ++c)
                        tmem_ld32(trow + colO + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&o[32 * c]));
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < D; ++e) o[e] = 0u;
                }
#pragma unroll
                for (int q8 = 0; q8 < D / 8; ++q8) {     // 16-byte chunks of 8 values
                    const int e0 = 8 * q8;
                    const int bx = e0 / C::BOXD;
                    const int ci = (e0 % C::BOXD) / 8;
                    uint4 w;
                    w.x = f2_to_bf2(__uint_as_float(o[e0 + 0]) * inv_l, __uint_as_float(o[e0 + 1]) * inv_l);
                    w.y = f2_to_bf2(__uint_as_float(o[e0 + 2]) * inv_l, __uint_as_float(o[e0 + 3]) * inv_l);
                    w.z = f2_to_bf2(__uint_as_float(o[e0 + 4]) * inv_l, __uint_as_float(o[e0 + 5]) * inv_l);
                    w.w = f2_to_bf2(__uint_as_float(o[e0 + 6]) * inv_l, __uint_as_float(o[e0 + 7]) * inv_l);
                    if (direct) {
                        if (pos < Sq)
                            *reinterpret_cast<uint4 *>(p.o + ((size_t)(q0 + pos) * p.n_q + head) * D + e0) = w;
                    } else {
                        sts128(stage + bx * C::QBOX + swz<C::SWB>((uint32_t)(r * C::ROWB + ci * 16)), w);
                    }
                }
            }
            if (p.lse != nullptr && pos < Sq) {
                const float lse_v = (!PACKED || l_run > 0.f) ? (m_run + log2f(l_run)) * 0.6931471805599453f : -INFINITY;
                if (PACKED)
                    p.lse[(size_t)head * p.total_q + q0 + pos] = lse_v;
                else
                    p.lse[((size_t)b * p.n_q + head) * p.Sq + pos] = lse_v;
            }
            fence_proxy_async_smem();
            named_bar_sync(2 + t, 128);
            if (r == 0 && ok && !direct) {
                for (int bx = 0; bx < C::NBOX; ++bx) {
                    if (PACKED)
                        tma_store_3d(&tm_o, stage + bx * C::QBOX, bx * C::BOXD, h0[t], q0 + p0[t]);
                    else
                        tma_store_3d(&tm_o, stage + bx * C::QBOX, bx * C::BOXD, p0[t], b * p.n_q + h0[t]);
                }
                tma_store_commit();
                tma_store_wait_read0();
            }
        }
    }

    // ---- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace pf
}  // namespace attn
