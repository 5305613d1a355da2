// attn_api.cu -- the C ABI of libattn_b200.so (declared in include/attn.h):
// argument validation, TMA descriptor encoding and kernel launches.
//
// The library allocates nothing: every buffer (including the decode
// workspace) belongs to the caller. Validation errors return before any
// launch; device-side errors land in the status word that
// attn_device_status() reads.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/attn.h"
#include "decode_gqa.cuh"
#include "decode_mla.cuh"
#include "fp8_widen.cuh"
#include "prefill.cuh"

namespace {

using attn::g_status;

// ---------------------------------------------------------------------------
// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult qres;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

CUtensorMapSwizzle swizzle_for(int row_bytes) {
    return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                            : (row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

// Tensor map of rank `rank` (bf16 elements, or bytes): dims[0] is the
// contiguous one; strides in bytes for dims 1..rank-1.
bool make_map(CUtensorMap *map, const void *base, int rank, const uint64_t *dims, const uint64_t *strides_bytes,
              const uint32_t *box, int row_bytes, CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[5], gstr[4];
    cuuint32_t bdim[5], estr[5];
    for (int i = 0; i < rank; ++i) {
        gdim[i] = dims[i];
        bdim[i] = box[i];
        estr[i] = 1;
    }
    for (int i = 0; i < rank - 1; ++i) gstr[i] = strides_bytes[i];
    CUresult r = fn(map, dtype, (cuuint32_t)rank, const_cast<void *>(base), gdim, gstr,
                    bdim, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_for(row_bytes),
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (kernel, device).
// `done_mask` holds one bit per device; threads that race on the first call
// of a device both set the (same) attributes, which is harmless.
template <typename K>
bool ensure_smem_attr(K kernel, size_t bytes, std::atomic<uint64_t> &done_mask) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const uint64_t bit = 1ull << (dev & 63);
    if (done_mask.load(std::memory_order_acquire) & bit) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
        return false;
    // all of the unified L1 / shared storage as shared memory, so that the
    // occupancy the grid is sized by counts every CTA that fits
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
        return false;
    done_mask.fetch_or(bit, std::memory_order_acq_rel);
    return true;
}
inline bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

// Number of SMs of the current device (cached per device; safe to call from
// several host threads).
int sm_count() {
    static std::atomic<int> counts[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
    int n = counts[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
        counts[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// ---------------------------------------------------------------------------
// prefill
// ---------------------------------------------------------------------------
// Packed variable-length batch of attn_fwd_varlen (null for the dense BHSD layout).
struct VarlenArgs {
    const int32_t *cu_q, *cu_k;
    int max_q, total_q, total_k;
    // paged keys and values (attn_fwd_paged): cu_k is unused, the pools are
    // [page][token][kv head][dim] with these element strides
    const int32_t *block_table = nullptr, *seqlens_k = nullptr;
    int page_size = 0, pages_per_seq = 0, num_pages = 0;
    int64_t ks[3] = {0, 0, 0}, vs[3] = {0, 0, 0};   // page, token, head
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
// Workspace of the FP8 prefill: k and v widened to bf16, each 256-byte aligned.
size_t fp8_prefill_ws_bytes(int B, int Sq, int Skv, int n_q, int n_kv, int d) {
    (void)Sq, (void)n_q;
    return 2 * align256((size_t)B * n_kv * Skv * d * 2);
}

// Per-tile scales of the FP8 prefill (q, k, v then hold the widened values).
struct Fp8Args {
    const float *q_scale, *k_scale, *v_scale;
};

template <int D>
int launch_prefill(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Sq, int Skv,
                   int n_q, int n_kv, int causal, float scale, cudaStream_t stream, const VarlenArgs *vl = nullptr,
                   int window = 0, int n_sink = 0, const attn::rope::Tables *rope = nullptr,
                   const Fp8Args *f8 = nullptr) {
    using attn::pf::kDense;
    using attn::pf::kFp8;
    using attn::pf::kPaged;
    using attn::pf::kRope;
    using attn::pf::kVarlen;
    using attn::pf::kWindow;
    using C = attn::pf::Cfg<D>;
    const int G = n_q / n_kv;
    attn::pf::Params p{};
    p.B = B;
    p.Sq = Sq;
    p.Skv = Skv;
    p.n_q = n_q;
    p.n_kv = n_kv;
    p.G = G;
    p.causal = causal;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634);
    p.lse = lse;
    p.window = window;
    p.n_sink = n_sink;
    if (rope) p.rope = *rope;
    if (f8) {
        if (D != 128 || vl || rope || window > 0) return ATTN_ERR_UNSUPPORTED;
        p.q_scale = f8->q_scale;
        p.k_scale = f8->k_scale;
        p.v_scale = f8->v_scale;
        p.q_tiles = (Sq + attn::pf::BM - 1) / attn::pf::BM;
        p.k_tiles = (Skv + attn::pf::BN - 1) / attn::pf::BN;
    }
    p.o = reinterpret_cast<__nv_bfloat16 *>(o);
    const int Sq_plan = vl ? vl->max_q : Sq;   // position blocks cover the longest sequence
    if (G >= 2) {
        p.Ht = G / 2;
        p.Pt = 256 / G;
        p.pair_by_heads = 1;
        p.n_pb = (Sq_plan + p.Pt - 1) / p.Pt;
    } else {
        p.Ht = 1;
        p.Pt = 128;
        p.pair_by_heads = 0;
        p.n_pb = (Sq_plan + 255) / 256;
    }
    CUtensorMap tq, tk, tv, to;
    if (vl) {
        p.cu_q = vl->cu_q;
        p.cu_k = vl->cu_k;
        p.total_q = vl->total_q;
        p.total_k = vl->total_k;
        p.o = reinterpret_cast<__nv_bfloat16 *>(o);
        // q, o [total_q][n_q][D]: box = BOXD dims x Ht heads x Pt positions
        const uint64_t qd[3] = {(uint64_t)D, (uint64_t)n_q, (uint64_t)vl->total_q};
        const uint64_t qs[2] = {(uint64_t)D * 2, (uint64_t)n_q * D * 2};
        const uint32_t qb[3] = {(uint32_t)C::BOXD, (uint32_t)p.Ht, (uint32_t)p.Pt};
        if (!make_map(&tq, q, 3, qd, qs, qb, C::ROWB)) return ATTN_ERR_CUDA;
        if (!make_map(&to, o, 3, qd, qs, qb, C::ROWB)) return ATTN_ERR_CUDA;
        if (vl->block_table) {
            // page pools [page][token][kv head][D]: box = BOXD dims x box_rows tokens
            p.block_table = vl->block_table;
            p.seqlens_k = vl->seqlens_k;
            p.pages_per_seq = vl->pages_per_seq;
            p.num_pages = vl->num_pages;
            int shift = 0;
            while ((1 << shift) < vl->page_size) ++shift;
            p.page_shift = shift;
            p.box_rows = vl->page_size < attn::pf::BN ? vl->page_size : attn::pf::BN;
            const uint64_t pd[4] = {(uint64_t)D, (uint64_t)vl->page_size, (uint64_t)n_kv, (uint64_t)vl->num_pages};
            const uint32_t pbx[4] = {(uint32_t)C::BOXD, (uint32_t)p.box_rows, 1u, 1u};
            const uint64_t kst[3] = {(uint64_t)vl->ks[1] * 2, (uint64_t)vl->ks[2] * 2, (uint64_t)vl->ks[0] * 2};
            const uint64_t vst[3] = {(uint64_t)vl->vs[1] * 2, (uint64_t)vl->vs[2] * 2, (uint64_t)vl->vs[0] * 2};
            if (!make_map(&tk, k, 4, pd, kst, pbx, C::ROWB)) return ATTN_ERR_CUDA;
            if (!make_map(&tv, v, 4, pd, vst, pbx, C::ROWB)) return ATTN_ERR_CUDA;
        } else {
            // k, v [total_k][n_kv][D]: box = BOXD dims x 1 head x BN keys
            const uint64_t kd[3] = {(uint64_t)D, (uint64_t)n_kv, (uint64_t)vl->total_k};
            const uint64_t ks[2] = {(uint64_t)D * 2, (uint64_t)n_kv * D * 2};
            const uint32_t kb[3] = {(uint32_t)C::BOXD, 1u, (uint32_t)attn::pf::BN};
            if (!make_map(&tk, k, 3, kd, ks, kb, C::ROWB)) return ATTN_ERR_CUDA;
            if (!make_map(&tv, v, 3, kd, ks, kb, C::ROWB)) return ATTN_ERR_CUDA;
        }
    } else {
        {
            const uint64_t dims[3] = {(uint64_t)D, (uint64_t)Sq, (uint64_t)B * n_q};
            const uint64_t str[2] = {(uint64_t)D * 2, (uint64_t)Sq * D * 2};
            const uint32_t box[3] = {(uint32_t)C::BOXD, (uint32_t)p.Pt, (uint32_t)p.Ht};
            if (f8) {
                // FP8: q holds e4m3 bytes, one 128-byte row per query row
                const uint64_t str8[2] = {(uint64_t)D, (uint64_t)Sq * D};
                const uint32_t box8[3] = {(uint32_t)D, (uint32_t)p.Pt, (uint32_t)p.Ht};
                if (!make_map(&tq, q, 3, dims, str8, box8, 128, CU_TENSOR_MAP_DATA_TYPE_UINT8)) return ATTN_ERR_CUDA;
            } else if (!make_map(&tq, q, 3, dims, str, box, C::ROWB)) {
                return ATTN_ERR_CUDA;
            }
            if (!make_map(&to, o, 3, dims, str, box, C::ROWB)) return ATTN_ERR_CUDA;
        }
        {
            const uint64_t dims[3] = {(uint64_t)D, (uint64_t)Skv, (uint64_t)B * n_kv};
            const uint64_t str[2] = {(uint64_t)D * 2, (uint64_t)Skv * D * 2};
            const uint32_t box[3] = {(uint32_t)C::BOXD, (uint32_t)attn::pf::BN, 1u};
            if (!make_map(&tk, k, 3, dims, str, box, C::ROWB)) return ATTN_ERR_CUDA;
            if (!make_map(&tv, v, 3, dims, str, box, C::ROWB)) return ATTN_ERR_CUDA;
        }
    }
    const size_t smem = attn::pf::smem_bytes<D>();
    static std::atomic<uint64_t> attr_done{0};  // per template instance, one bit per device
    if (!ensure_smem_attr(attn::pf::prefill_kernel<D, kDense>, smem, attr_done)) return ATTN_ERR_CUDA;
    static std::atomic<uint64_t> attr_done_v{0}, attr_done_w{0}, attr_done_r{0}, attr_done_p{0};
    if (!ensure_smem_attr(attn::pf::prefill_kernel<D, kVarlen>, smem, attr_done_v)) return ATTN_ERR_CUDA;
    if (!ensure_smem_attr(attn::pf::prefill_kernel<D, kPaged>, smem, attr_done_p)) return ATTN_ERR_CUDA;
    if (!ensure_smem_attr(attn::pf::prefill_kernel<D, kWindow>, smem, attr_done_w)) return ATTN_ERR_CUDA;
    if (!ensure_smem_attr(attn::pf::prefill_kernel<D, kRope>, smem, attr_done_r)) return ATTN_ERR_CUDA;
    if constexpr (D == 128) {
        static std::atomic<uint64_t> attr_done_f{0};
        if (!ensure_smem_attr(attn::pf::prefill_kernel<D, kFp8>, smem, attr_done_f)) return ATTN_ERR_CUDA;
    }
    // The kernel rebalances registers between warpgroups (setmaxnreg); that is
    // only safe if it was built with exactly the register count the split
    // assumes, otherwise the increase could never be granted.
    static std::atomic<int> regs_checked{0};   // 0: not yet checked, 1: ok, -1: mismatch
    if (regs_checked.load(std::memory_order_acquire) == 0) {
        cudaFuncAttributes fa;
        cudaFuncAttributes fv, fw, fr, fp;
        if (cudaFuncGetAttributes(&fa, attn::pf::prefill_kernel<D, kDense>) != cudaSuccess) return ATTN_ERR_CUDA;
        if (cudaFuncGetAttributes(&fv, attn::pf::prefill_kernel<D, kVarlen>) != cudaSuccess) return ATTN_ERR_CUDA;
        if (cudaFuncGetAttributes(&fw, attn::pf::prefill_kernel<D, kWindow>) != cudaSuccess) return ATTN_ERR_CUDA;
        if (cudaFuncGetAttributes(&fr, attn::pf::prefill_kernel<D, kRope>) != cudaSuccess) return ATTN_ERR_CUDA;
        if (cudaFuncGetAttributes(&fp, attn::pf::prefill_kernel<D, kPaged>) != cudaSuccess) return ATTN_ERR_CUDA;
        bool f8_ok = true;
        if constexpr (D == 128) {
            cudaFuncAttributes ff;
            if (cudaFuncGetAttributes(&ff, attn::pf::prefill_kernel<D, kFp8>) != cudaSuccess) return ATTN_ERR_CUDA;
            f8_ok = ff.numRegs == attn::pf::kLaunchRegs;
        }
        regs_checked.store((fa.numRegs == attn::pf::kLaunchRegs && fv.numRegs == attn::pf::kLaunchRegs &&
                            fw.numRegs == attn::pf::kLaunchRegs && fr.numRegs == attn::pf::kLaunchRegs &&
                            fp.numRegs == attn::pf::kLaunchRegs && f8_ok) ? 1 : -1,
                           std::memory_order_release);
    }
    if (regs_checked.load(std::memory_order_acquire) < 0) return ATTN_ERR_UNSUPPORTED;
    if (vl) {
        // x: (position block, kv head), heaviest causal blocks first; y: sequence
        const long long gx = (long long)p.n_pb * n_kv;
        if (gx <= 0 || B <= 0) return ATTN_OK;
        if (gx > 0x7fffffffLL || B > 65535) return ATTN_ERR_UNSUPPORTED;
        if (vl->block_table)
            attn::pf::prefill_kernel<D, kPaged><<<dim3((unsigned)gx, (unsigned)B), attn::pf::THREADS, smem, stream>>>(
                tq, tk, tv, to, p);
        else
            attn::pf::prefill_kernel<D, kVarlen><<<dim3((unsigned)gx, (unsigned)B), attn::pf::THREADS, smem, stream>>>(
                tq, tk, tv, to, p);
    } else {
        const long long grid = (long long)p.n_pb * B * n_kv;
        if (grid <= 0) return ATTN_OK;
        if (grid > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
        // one CTA per SM: the CTA one wave later gets its Q tiles prefetched
        const int n_sm = sm_count();
        p.l2_ahead = (n_sm > 0 && grid > n_sm) ? n_sm : 0;
        if (rope) {
            // launched as a programmatic dependent of the key rotation: the
            // prologue (barriers, TMEM, Q load and rotation) overlaps it and
            // only the K producer waits for it
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)grid);
            cfg.blockDim = dim3(attn::pf::THREADS);
            cfg.dynamicSmemBytes = smem;
            cfg.stream = stream;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[0].val.programmaticStreamSerializationAllowed = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaLaunchKernelEx(&cfg, attn::pf::prefill_kernel<D, kRope>, tq, tk, tv, to, p) != cudaSuccess)
                return ATTN_ERR_CUDA;
        } else if (window > 0) {
            attn::pf::prefill_kernel<D, kWindow><<<(unsigned)grid, attn::pf::THREADS, smem, stream>>>(tq, tk, tv, to,
                                                                                                       p);
        } else if (f8) {
            // a programmatic dependent of the widening pass: the prologue, the
            // e4m3 query tiles and their widening overlap it, and only the K
            // and V producers wait for it
            if constexpr (D == 128) {
                cudaLaunchConfig_t cfg = {};
                cfg.gridDim = dim3((unsigned)grid);
                cfg.blockDim = dim3(attn::pf::THREADS);
                cfg.dynamicSmemBytes = smem;
                cfg.stream = stream;
                cudaLaunchAttribute attr[1];
                attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
                attr[0].val.programmaticStreamSerializationAllowed = 1;
                cfg.attrs = attr;
                cfg.numAttrs = 1;
                if (cudaLaunchKernelEx(&cfg, attn::pf::prefill_kernel<D, kFp8>, tq, tk, tv, to, p) != cudaSuccess)
                    return ATTN_ERR_CUDA;
            }
        } else
            attn::pf::prefill_kernel<D, kDense><<<(unsigned)grid, attn::pf::THREADS, smem, stream>>>(tq, tk, tv, to,
                                                                                                      p);
    }
    return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// decode (GQA, head dim 128)
// ---------------------------------------------------------------------------
// Query heads per decode work unit (a power of two dividing G).
inline int decode_head_block(int G) { return G >= 16 ? 16 : G; }

// CTAs of the persistent decode grid resident at once on the current device:
// two per SM while two fit in the SM's 228 KB of shared memory (with 1 KB
// reserved per CTA; the register budget of two is fixed by the launch
// bounds), else one.
template <int GT, bool FP8>
int decode_slots() {
    const int n_sm = sm_count();
    if (n_sm <= 0) return -1;
    const size_t smem = attn::dec::smem_bytes<GT, FP8>();
    const int per_sm = (int)(233472 / (smem + 1024)) >= 2 ? 2 : 1;
    return per_sm * n_sm;
}

// Keys per decode work unit (the split-KV chunk), planned from the sizes and
// the SM count: with `slots` resident CTAs and B * n_kv * n_hb units per
// chunk index, s = slots / (B * n_kv * n_hb) chunks per (sequence, KV head,
// head block) give every unit of a full-length batch a slot of its own in one
// wave, so a small batch still reaches every SM; the chunk is S_max / s keys
// rounded up to the 128-key tile, at most the kernel's largest chunk (2048,
// or 1024 at 16 heads per unit), which is also what a batch that fills the
// slots by itself gets. The same sizes on the same device always give the
// same chunk (the workspace size follows from it).
template <int GT, bool FP8>
int decode_chunk_t(int B, int n_kv, int G, int S_max) {
    constexpr int CH = attn::dec::Cfg<GT, FP8>::CH, KT = attn::dec::KT;
    const int slots = decode_slots<GT, FP8>();
    const long long per_split = (long long)B * n_kv * (G / GT);
    if (slots <= 0 || per_split <= 0) return CH;
    const long long s = slots / per_split;
    if (s <= 1) return CH;
    long long ch = ((S_max + s - 1) / s + KT - 1) / KT * KT;
    if (ch > CH) ch = CH;
    if (ch < KT) ch = KT;
    return (int)ch;
}
inline int decode_chunk(int B, int n_kv, int G, int S_max, bool fp8) {
    switch (decode_head_block(G)) {
        case 1: return fp8 ? decode_chunk_t<1, true>(B, n_kv, G, S_max) : decode_chunk_t<1, false>(B, n_kv, G, S_max);
        case 2: return fp8 ? decode_chunk_t<2, true>(B, n_kv, G, S_max) : decode_chunk_t<2, false>(B, n_kv, G, S_max);
        case 4: return fp8 ? decode_chunk_t<4, true>(B, n_kv, G, S_max) : decode_chunk_t<4, false>(B, n_kv, G, S_max);
        case 8: return fp8 ? decode_chunk_t<8, true>(B, n_kv, G, S_max) : decode_chunk_t<8, false>(B, n_kv, G, S_max);
        default:
            return fp8 ? decode_chunk_t<16, true>(B, n_kv, G, S_max) : decode_chunk_t<16, false>(B, n_kv, G, S_max);
    }
}
// Number of key chunks of S_max (the workspace's split dimension).
inline int decode_n_splits(int B, int n_kv, int G, int S_max, bool fp8 = false) {
    const int ch = decode_chunk(B, n_kv, G, S_max, fp8);
    return (S_max + ch - 1) / ch;
}

size_t decode_ws_bytes(int B, int n_q, int d_v, int n_splits) {
    const size_t rows = (size_t)B * n_q * n_splits;
    size_t o_bytes = rows * d_v * sizeof(float);
    o_bytes = (o_bytes + 255) & ~size_t(255);
    return o_bytes + rows * sizeof(float2);
}

// Cache addressing of one decode launch: a contiguous cache
// [B][n_kv][S_max][row] (element strides ks/vs = b, head, token) or a page
// pool [num_pages][page_size][n_kv][row] (strides = page, token, head).
struct CacheView {
    const void *k, *v;
    int64_t ks[3], vs[3];              // element strides, outermost first
    attn::dec::PageTable pt;           // pt.table == nullptr: contiguous
    int page_size;
    attn::dec::Window win;             // sliding window (window 0: none)
    attn::dec::Fp8Scales fs;           // FP8 cache: per-KV-head scales
    attn::rope::Tables rt{nullptr, nullptr, 0};   // rotary tables for the query (cos null: none)
};

template <int GT, bool PAGED, bool FP8 = false>
int launch_decode_gqa(const void *q, const CacheView &cv, const int32_t *seqlens, void *o, float *lse, int B,
                      int n_q, int n_kv, int S_max, float scale, void *ws, cudaStream_t stream) {
    using namespace attn::dec;
    using C = Cfg<GT, FP8>;
    const int G = n_q / n_kv;
    const int n_hb = G / GT;
    const int ch = decode_chunk_t<GT, FP8>(B, n_kv, G, S_max);
    const int n_splits = (S_max + ch - 1) / ch;
    CUtensorMap tq, tk, tv;
    {
        // the group's query rows: [B][n_q][128], box = 64 dims x NH heads
        const uint64_t dims[3] = {(uint64_t)D, (uint64_t)n_q, (uint64_t)B};
        const uint64_t str[2] = {(uint64_t)D * 2, (uint64_t)n_q * D * 2};
        const uint32_t box[3] = {64u, (uint32_t)C::NH, 1u};
        if (!make_map(&tq, q, 3, dims, str, box, 128)) return ATTN_ERR_CUDA;
    }
    if (PAGED) {
        // [dim][token in page][kv head][page]
        const uint64_t dims[4] = {(uint64_t)D, (uint64_t)cv.page_size, (uint64_t)n_kv, (uint64_t)cv.pt.num_pages};
        const uint32_t box[4] = {64u, (uint32_t)cv.pt.box_rows, 1u, 1u};
        const uint64_t kstr[3] = {(uint64_t)cv.ks[1] * 2, (uint64_t)cv.ks[2] * 2, (uint64_t)cv.ks[0] * 2};
        const uint64_t vstr[3] = {(uint64_t)cv.vs[1] * 2, (uint64_t)cv.vs[2] * 2, (uint64_t)cv.vs[0] * 2};
        if (!make_map(&tk, cv.k, 4, dims, kstr, box, 128)) return ATTN_ERR_CUDA;
        if (!make_map(&tv, cv.v, 4, dims, vstr, box, 128)) return ATTN_ERR_CUDA;
    } else if (FP8) {
        // one-byte e4m3 elements: [dim][token][kv head][sequence], one 128-byte box per row
        const uint64_t dims[4] = {(uint64_t)D, (uint64_t)S_max, (uint64_t)n_kv, (uint64_t)B};
        const uint32_t box[4] = {128u, (uint32_t)KT, 1u, 1u};
        const uint64_t kstr[3] = {(uint64_t)cv.ks[2], (uint64_t)cv.ks[1], (uint64_t)cv.ks[0]};
        const uint64_t vstr[3] = {(uint64_t)cv.vs[2], (uint64_t)cv.vs[1], (uint64_t)cv.vs[0]};
        if (!make_map(&tk, cv.k, 4, dims, kstr, box, 128, CU_TENSOR_MAP_DATA_TYPE_UINT8)) return ATTN_ERR_CUDA;
        if (!make_map(&tv, cv.v, 4, dims, vstr, box, 128, CU_TENSOR_MAP_DATA_TYPE_UINT8)) return ATTN_ERR_CUDA;
    } else {
        // [dim][token][kv head][sequence]
        const uint64_t dims[4] = {(uint64_t)D, (uint64_t)S_max, (uint64_t)n_kv, (uint64_t)B};
        const uint32_t box[4] = {64u, (uint32_t)KT, 1u, 1u};
        const uint64_t kstr[3] = {(uint64_t)cv.ks[2] * 2, (uint64_t)cv.ks[1] * 2, (uint64_t)cv.ks[0] * 2};
        const uint64_t vstr[3] = {(uint64_t)cv.vs[2] * 2, (uint64_t)cv.vs[1] * 2, (uint64_t)cv.vs[0] * 2};
        if (!make_map(&tk, cv.k, 4, dims, kstr, box, 128)) return ATTN_ERR_CUDA;
        if (!make_map(&tv, cv.v, 4, dims, vstr, box, 128)) return ATTN_ERR_CUDA;
    }
    const size_t smem = smem_bytes<GT, FP8>();
    static std::atomic<uint64_t> attr_done{0};
    if (!ensure_smem_attr(decode_split_kernel<GT, PAGED, FP8>, smem, attr_done)) return ATTN_ERR_CUDA;
    float *ws_o = reinterpret_cast<float *>(ws);
    size_t o_bytes = (size_t)B * n_q * n_splits * D * sizeof(float);
    o_bytes = (o_bytes + 255) & ~size_t(255);
    float2 *ws_ml = reinterpret_cast<float2 *>(reinterpret_cast<uint8_t *>(ws) + o_bytes);
    const float scale_log2 = (float)((double)scale * 1.4426950408889634);
    // persistent: as many CTAs as fit on the SMs at once, never more than the
    // largest possible unit count
    const int slots = decode_slots<GT, FP8>();
    if (slots <= 0) return ATTN_ERR_CUDA;
    constexpr int threads = FP8 ? THREADS_FP8 : THREADS;
    const long long max_units = (long long)B * n_kv * n_hb * n_splits;
    const int grid = (int)(max_units < slots ? max_units : slots);
    decode_split_kernel<GT, PAGED, FP8><<<grid, threads, smem, stream>>>(tq, tk, tv, seqlens, ws_o, ws_ml, B, n_q,
                                                                         n_kv, G, n_hb, S_max, n_splits, ch,
                                                                         scale_log2, cv.pt, cv.win, cv.fs, cv.rt);
    if (cudaPeekAtLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    // the merge, as a programmatic dependent of the split kernel
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(n_q, B);
    cfg.blockDim = dim3(COMBINE_THREADS);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, decode_combine_kernel<D>, (const float *)ws_o, (const float2 *)ws_ml, seqlens,
                           reinterpret_cast<__nv_bfloat16 *>(o), lse, n_q, n_splits, S_max, ch, cv.win) != cudaSuccess)
        return ATTN_ERR_CUDA;
    return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <bool PAGED, bool FP8 = false>
int dispatch_decode_gqa(int G, const void *q, const CacheView &cv, const int32_t *seqlens, void *o, float *lse,
                        int B, int n_q, int n_kv, int S_max, float scale, void *ws, cudaStream_t s) {
    switch (decode_head_block(G)) {
        case 1: return launch_decode_gqa<1, PAGED, FP8>(q, cv, seqlens, o, lse, B, n_q, n_kv, S_max, scale, ws, s);
        case 2: return launch_decode_gqa<2, PAGED, FP8>(q, cv, seqlens, o, lse, B, n_q, n_kv, S_max, scale, ws, s);
        case 4: return launch_decode_gqa<4, PAGED, FP8>(q, cv, seqlens, o, lse, B, n_q, n_kv, S_max, scale, ws, s);
        case 8: return launch_decode_gqa<8, PAGED, FP8>(q, cv, seqlens, o, lse, B, n_q, n_kv, S_max, scale, ws, s);
        default: return launch_decode_gqa<16, PAGED, FP8>(q, cv, seqlens, o, lse, B, n_q, n_kv, S_max, scale, ws, s);
    }
}

// ---------------------------------------------------------------------------
// MLA decode (latent row of 576 = key, its first 512 columns = value)
// ---------------------------------------------------------------------------
// Split-KV plan of the MLA decode: a 2-CTA cluster per (sequence, head
// block, key chunk), one CTA per SM. With c = SMs / 2 clusters resident and
// B * n_hb of them per chunk index, s = c / (B * n_hb) chunks per sequence
// give a full-length batch one wave over every SM; chunks hold at least two
// 64-key tiles (every chunk's cluster loads the whole query block). A batch
// that fills the clusters by itself gets one chunk per sequence, and then no
// workspace: the clusters write O and LSE themselves.
int mla_n_splits(int B, int n_q, int S_max, int *chunk) {
    constexpr int KT = attn::mla::KT, MIN_CHUNK = 2 * KT;
    const int n_sm = sm_count();
    const long long per_split = (long long)B * (n_q / attn::mla::M);
    long long s = (n_sm > 0 && per_split > 0) ? (n_sm / 2) / per_split : 1;
    const long long most = (S_max + MIN_CHUNK - 1) / MIN_CHUNK;
    if (s > most) s = most;
    if (s < 1) s = 1;
    const int ch = (int)(((S_max + s - 1) / s + KT - 1) / KT * KT);
    if (chunk) *chunk = ch;
    return (S_max + ch - 1) / ch;
}
size_t mla_ws_bytes(int B, int n_q, int S_max) {
    const int n_splits = mla_n_splits(B, n_q, S_max, nullptr);
    return n_splits > 1 ? decode_ws_bytes(B, n_q, attn::mla::DV, n_splits) : 0;
}

int launch_decode_mla(const void *q, const void *cache, const int32_t *seqlens, void *o, float *lse, int B, int n_q,
                      int S_max, int64_t stride_b, int64_t stride_s, float scale, void *ws, cudaStream_t stream) {
    using namespace attn::mla;
    CUtensorMap tq, tc;
    {
        const uint64_t dims[3] = {(uint64_t)DL, (uint64_t)n_q, (uint64_t)B};
        const uint64_t str[2] = {(uint64_t)DL * 2, (uint64_t)n_q * DL * 2};
        const uint32_t box[3] = {64u, (uint32_t)M, 1u};
        if (!make_map(&tq, q, 3, dims, str, box, 128)) return ATTN_ERR_CUDA;
    }
    {
        const uint64_t dims[3] = {(uint64_t)DL, (uint64_t)S_max, (uint64_t)B};
        const uint64_t str[2] = {(uint64_t)stride_s * 2, (uint64_t)stride_b * 2};
        const uint32_t box[3] = {64u, (uint32_t)KT, 1u};
        if (!make_map(&tc, cache, 3, dims, str, box, 128)) return ATTN_ERR_CUDA;
    }
    const size_t smem = smem_bytes();
    static std::atomic<uint64_t> attr_done{0};
    if (!ensure_smem_attr(mla_decode_kernel, smem, attr_done)) return ATTN_ERR_CUDA;
    Params p;
    p.B = B;
    p.n_q = n_q;
    p.S_max = S_max;
    p.seqlens = seqlens;
    p.o = reinterpret_cast<__nv_bfloat16 *>(o);
    p.lse = lse;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634);
    p.n_splits = mla_n_splits(B, n_q, S_max, &p.ch);
    p.ws_o = nullptr;
    p.ws_ml = nullptr;
    if (p.n_splits > 1) {
        size_t o_bytes = (size_t)B * n_q * p.n_splits * DV * sizeof(float);
        o_bytes = (o_bytes + 255) & ~size_t(255);
        p.ws_o = reinterpret_cast<float *>(ws);
        p.ws_ml = reinterpret_cast<float2 *>(reinterpret_cast<uint8_t *>(ws) + o_bytes);
    }
    if ((long long)2 * B * p.n_splits > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * B * p.n_splits, n_q / M, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, mla_decode_kernel, tq, tc, p) != cudaSuccess) return ATTN_ERR_CUDA;
    if (p.n_splits == 1) return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
    // the merge of the chunks (as for the GQA decode), a programmatic dependent
    cudaLaunchConfig_t mcfg = {};
    mcfg.gridDim = dim3(n_q, B);
    mcfg.blockDim = dim3(attn::dec::COMBINE_THREADS);
    mcfg.dynamicSmemBytes = 0;
    mcfg.stream = stream;
    cudaLaunchAttribute mattr[1];
    mattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    mattr[0].val.programmaticStreamSerializationAllowed = 1;
    mcfg.attrs = mattr;
    mcfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&mcfg, attn::dec::decode_combine_kernel<DV>, (const float *)p.ws_o, (const float2 *)p.ws_ml,
                           seqlens, reinterpret_cast<__nv_bfloat16 *>(o), lse, n_q, p.n_splits, S_max, p.ch,
                           attn::dec::Window{0, 0}) != cudaSuccess)
        return ATTN_ERR_CUDA;
    return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

__global__ void selftest_timeout_kernel(unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        attn::mbar_init(attn::smem_u32(&bar), 1);
        abort_flag = 0;
        attn::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)  // nothing ever arrives on `bar`
        attn::mbar_wait_slow(attn::smem_u32(&bar), 0, &abort_flag, 0x7e57, limit_ns);
}

__global__ void selftest_ex2_kernel(const float *x, float *y_poly, float *y_sfu, int n) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const float a = x[i], b = (i + 1 < n) ? x[i + 1] : 0.f;
    const float2 p = attn::ex2_poly2(make_float2(a, b));
    y_poly[i] = p.x;
    y_sfu[i] = attn::ex2(a);
    if (i + 1 < n) {
        y_poly[i + 1] = p.y;
        y_sfu[i + 1] = attn::ex2(b);
    }
}

}  // namespace

extern "C" {

int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Sq, int Skv, int n_q,
             int n_kv, int d_qk, int d_v, int causal, float scale, attn_stream_t stream) {
    if (B < 0 || Sq < 0 || Skv < 1 || n_q < 1 || n_kv < 1 || d_qk < 1 || d_v < 1) return ATTN_ERR_INVALID_ARG;
    if (n_q % n_kv != 0) return ATTN_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
    if (B == 0 || Sq == 0) return ATTN_OK;
    if (!q || !k || !v || !o) return ATTN_ERR_INVALID_ARG;
    if (d_qk != d_v || (d_qk != 32 && d_qk != 64 && d_qk != 128)) return ATTN_ERR_UNSUPPORTED;
    const int G = n_q / n_kv;
    if (!is_pow2(G) || G > 256) return ATTN_ERR_UNSUPPORTED;
    if (causal && Sq > Skv) return ATTN_ERR_UNSUPPORTED;
    if ((long long)B * n_q > 0x7fffffffLL || (long long)B * n_kv > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_MISALIGNED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (d_qk) {
        case 32: return launch_prefill<32>(q, k, v, o, lse, B, Sq, Skv, n_q, n_kv, causal, scale, s);
        case 64: return launch_prefill<64>(q, k, v, o, lse, B, Sq, Skv, n_q, n_kv, causal, scale, s);
        default: return launch_prefill<128>(q, k, v, o, lse, B, Sq, Skv, n_q, n_kv, causal, scale, s);
    }
}

int attn_fwd_fp8_workspace_bytes(int B, int Sq, int Skv, int n_q, int n_kv, int d, size_t *bytes) {
    if (!bytes || B < 0 || Sq < 0 || Skv < 1 || n_q < 1 || n_kv < 1 || d < 1) return ATTN_ERR_INVALID_ARG;
    if (d != 128) return ATTN_ERR_UNSUPPORTED;
    *bytes = fp8_prefill_ws_bytes(B, Sq, Skv, n_q, n_kv, d);
    return ATTN_OK;
}

int attn_fwd_fp8(const void *q8, const void *k8, const void *v8, const float *q_scale, const float *k_scale,
                 const float *v_scale, void *o, float *lse, int B, int Sq, int Skv, int n_q, int n_kv, int d,
                 int causal, float scale, void *workspace, size_t workspace_bytes, attn_stream_t stream) {
    if (B < 0 || Sq < 0 || Skv < 1 || n_q < 1 || n_kv < 1 || d < 1) return ATTN_ERR_INVALID_ARG;
    if (n_q % n_kv != 0) return ATTN_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
    if (B == 0 || Sq == 0) return ATTN_OK;
    if (!q8 || !k8 || !v8 || !q_scale || !k_scale || !v_scale || !o) return ATTN_ERR_INVALID_ARG;
    if (d != 128) return ATTN_ERR_UNSUPPORTED;
    const int G = n_q / n_kv;
    if (!is_pow2(G) || G > 256) return ATTN_ERR_UNSUPPORTED;
    if (causal && Sq > Skv) return ATTN_ERR_UNSUPPORTED;
    if ((long long)B * n_q > 0x7fffffffLL || (long long)B * n_kv > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(o)) return ATTN_ERR_MISALIGNED;
    const size_t need = fp8_prefill_ws_bytes(B, Sq, Skv, n_q, n_kv, d);
    if (!workspace || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return ATTN_ERR_MISALIGNED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // keys and values widened into the workspace (bf16, same layouts; every
    // CTA of a KV head reads them); the queries are widened by the attention
    // kernel itself, each tile once, in shared memory
    const size_t nk = (size_t)B * n_kv * Skv * d;
    uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
    uint16_t *k16 = reinterpret_cast<uint16_t *>(ws);
    uint16_t *v16 = reinterpret_cast<uint16_t *>(ws + align256(nk * 2));
    const attn::f8::WidenSeg sk{reinterpret_cast<const uint8_t *>(k8), k16, nk / 16};
    const attn::f8::WidenSeg sv{reinterpret_cast<const uint8_t *>(v8), v16, nk / 16};
    const attn::f8::WidenSeg none{nullptr, nullptr, 0};
    const size_t groups = 2 * nk / 16;
    const int n_sm = sm_count();
    if (n_sm <= 0) return ATTN_ERR_CUDA;
    const size_t want = (groups + attn::f8::WIDEN_THREADS - 1) / attn::f8::WIDEN_THREADS;
    const int grid = (int)(want < (size_t)n_sm * 8 ? want : (size_t)n_sm * 8);
    attn::f8::widen_e4m3_kernel<<<grid, attn::f8::WIDEN_THREADS, 0, s>>>(sk, sv, none);
    if (cudaPeekAtLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    const Fp8Args f8{q_scale, k_scale, v_scale};
    return launch_prefill<128>(q8, k16, v16, o, lse, B, Sq, Skv, n_q, n_kv, causal, scale, s, nullptr, 0, 0,
                               nullptr, &f8);
}

int attn_fwd_window(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Sq, int Skv,
                    int n_q, int n_kv, int d_qk, int d_v, int window, int n_sink, float scale, attn_stream_t stream) {
    if (B < 0 || Sq < 0 || Skv < 1 || n_q < 1 || n_kv < 1 || d_qk < 1 || d_v < 1) return ATTN_ERR_INVALID_ARG;
    if (n_q % n_kv != 0 || window < 1 || n_sink < 0) return ATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
    if (B == 0 || Sq == 0) return ATTN_OK;
    if (!q || !k || !v || !o) return ATTN_ERR_INVALID_ARG;
    if (d_qk != d_v || (d_qk != 32 && d_qk != 64 && d_qk != 128)) return ATTN_ERR_UNSUPPORTED;
    const int G = n_q / n_kv;
    if (!is_pow2(G) || G > 256) return ATTN_ERR_UNSUPPORTED;
    if (Sq > Skv) return ATTN_ERR_UNSUPPORTED;
    if ((long long)B * n_q > 0x7fffffffLL || (long long)B * n_kv > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_MISALIGNED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (d_qk) {
        case 32: return launch_prefill<32>(q, k, v, o, lse, B, Sq, Skv, n_q, n_kv, 1, scale, s, nullptr, window, n_sink);
        case 64: return launch_prefill<64>(q, k, v, o, lse, B, Sq, Skv, n_q, n_kv, 1, scale, s, nullptr, window, n_sink);
        default: return launch_prefill<128>(q, k, v, o, lse, B, Sq, Skv, n_q, n_kv, 1, scale, s, nullptr, window, n_sink);
    }
}

int attn_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse, const int32_t *cu_seqlens_q,
                    const int32_t *cu_seqlens_k, int B, int max_seqlen_q, int total_q, int total_k, int n_q,
                    int n_kv, int d_qk, int d_v, int causal, float scale, attn_stream_t stream) {
    if (B < 0 || max_seqlen_q < 0 || total_q < 0 || total_k < 0 || n_q < 1 || n_kv < 1 || d_qk < 1 || d_v < 1)
        return ATTN_ERR_INVALID_ARG;
    if (n_q % n_kv != 0) return ATTN_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
    if (B == 0 || total_q == 0 || max_seqlen_q == 0) return ATTN_OK;
    if (!q || !o || !cu_seqlens_q || !cu_seqlens_k || (total_k > 0 && (!k || !v))) return ATTN_ERR_INVALID_ARG;
    if (d_qk != d_v || (d_qk != 32 && d_qk != 64 && d_qk != 128)) return ATTN_ERR_UNSUPPORTED;
    const int G = n_q / n_kv;
    if (!is_pow2(G) || G > 256) return ATTN_ERR_UNSUPPORTED;
    if (B > 65535) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(o) || (total_k > 0 && (!aligned16(k) || !aligned16(v))))
        return ATTN_ERR_MISALIGNED;
    // With no key rows at all every query row is empty (O = 0, LSE = -inf) and
    // no K/V tile is ever loaded; the maps are then built over q's memory
    // only because a tensor map needs a non-empty extent.
    VarlenArgs vl{cu_seqlens_q, cu_seqlens_k, max_seqlen_q, total_q, total_k > 0 ? total_k : 1};
    const void *kk = total_k > 0 ? k : static_cast<const void *>(q);
    const void *vv = total_k > 0 ? v : static_cast<const void *>(q);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (d_qk) {
        case 32: return launch_prefill<32>(q, kk, vv, o, lse, B, 0, 0, n_q, n_kv, causal, scale, s, &vl);
        case 64: return launch_prefill<64>(q, kk, vv, o, lse, B, 0, 0, n_q, n_kv, causal, scale, s, &vl);
        default: return launch_prefill<128>(q, kk, vv, o, lse, B, 0, 0, n_q, n_kv, causal, scale, s, &vl);
    }
}

int attn_fwd_paged(const void *q, const void *k_pages, const void *v_pages, const int32_t *block_table,
                   const int32_t *cu_seqlens_q, const int32_t *seqlens_k, void *o, float *lse, int B, int max_seqlen_q,
                   int total_q, int n_q, int n_kv, int d_qk, int d_v, int page_size, int pages_per_seq, int num_pages,
                   int64_t k_stride_page, int64_t k_stride_token, int64_t k_stride_head, int64_t v_stride_page,
                   int64_t v_stride_token, int64_t v_stride_head, int causal, float scale, attn_stream_t stream) {
    if (B < 0 || max_seqlen_q < 0 || total_q < 0 || n_q < 1 || n_kv < 1 || d_qk < 1 || d_v < 1)
        return ATTN_ERR_INVALID_ARG;
    if (n_q % n_kv != 0) return ATTN_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
    if (page_size < 1 || pages_per_seq < 1 || num_pages < 1) return ATTN_ERR_INVALID_ARG;
    if ((long long)page_size * pages_per_seq > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
    if (k_stride_page < 0 || k_stride_token < 0 || k_stride_head < 0 || v_stride_page < 0 || v_stride_token < 0 ||
        v_stride_head < 0)
        return ATTN_ERR_INVALID_ARG;
    if (B == 0 || total_q == 0 || max_seqlen_q == 0) return ATTN_OK;
    if (!q || !o || !k_pages || !v_pages || !block_table || !cu_seqlens_q || !seqlens_k) return ATTN_ERR_INVALID_ARG;
    if (d_qk != d_v || (d_qk != 32 && d_qk != 64 && d_qk != 128)) return ATTN_ERR_UNSUPPORTED;
    const int G = n_q / n_kv;
    if (!is_pow2(G) || G > 256) return ATTN_ERR_UNSUPPORTED;
    if (B > 65535) return ATTN_ERR_UNSUPPORTED;
    // a page is whole TMA boxes of up to 128 rows: 16, 32, 64 or a power of two >= 128 tokens
    if (!(page_size == 16 || page_size == 32 || page_size == 64 || (page_size % 128 == 0 && is_pow2(page_size))))
        return ATTN_ERR_UNSUPPORTED;
    if (k_stride_token < d_qk || v_stride_token < d_v) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(o) || !aligned16(k_pages) || !aligned16(v_pages)) return ATTN_ERR_MISALIGNED;
    if ((k_stride_page | k_stride_token | k_stride_head | v_stride_page | v_stride_token | v_stride_head) & 7)
        return ATTN_ERR_MISALIGNED;
    VarlenArgs vl{cu_seqlens_q, nullptr, max_seqlen_q, total_q, 1};
    vl.block_table = block_table;
    vl.seqlens_k = seqlens_k;
    vl.page_size = page_size;
    vl.pages_per_seq = pages_per_seq;
    vl.num_pages = num_pages;
    vl.ks[0] = k_stride_page, vl.ks[1] = k_stride_token, vl.ks[2] = k_stride_head;
    vl.vs[0] = v_stride_page, vl.vs[1] = v_stride_token, vl.vs[2] = v_stride_head;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (d_qk) {
        case 32: return launch_prefill<32>(q, k_pages, v_pages, o, lse, B, 0, 0, n_q, n_kv, causal, scale, s, &vl);
        case 64: return launch_prefill<64>(q, k_pages, v_pages, o, lse, B, 0, 0, n_q, n_kv, causal, scale, s, &vl);
        default: return launch_prefill<128>(q, k_pages, v_pages, o, lse, B, 0, 0, n_q, n_kv, causal, scale, s, &vl);
    }
}

int attn_decode_workspace_bytes(int B, int n_q, int n_kv, int d_qk, int d_v, int S_max, size_t *bytes) {
    if (!bytes || B < 0 || n_q < 1 || n_kv < 1 || S_max < 1 || n_q % n_kv != 0) return ATTN_ERR_INVALID_ARG;
    if (d_qk == 576 && d_v == 512 && n_kv == 1) {  // 0 when one chunk per sequence is planned
        if (n_q % attn::mla::M != 0) return ATTN_ERR_UNSUPPORTED;
        *bytes = mla_ws_bytes(B, n_q, S_max);
        return ATTN_OK;
    }
    if (!(d_qk == 128 && d_v == 128)) return ATTN_ERR_UNSUPPORTED;
    *bytes = decode_ws_bytes(B, n_q, d_v, decode_n_splits(B, n_kv, n_q / n_kv, S_max));
    return ATTN_OK;
}

}  // extern "C"

namespace {
int decode_entry(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens, void *o, float *lse,
                 int B, int n_q, int n_kv, int d_qk, int d_v, int S_max, int64_t k_stride_b, int64_t k_stride_h,
                 int64_t k_stride_s, int64_t v_stride_b, int64_t v_stride_h, int64_t v_stride_s, float scale,
                 void *workspace, size_t workspace_bytes, attn_stream_t stream, attn::dec::Window win,
                 const attn::rope::Tables *rt = nullptr) {
    if (B < 0 || n_q < 1 || n_kv < 1 || S_max < 1 || n_q % n_kv != 0) return ATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
    if (B == 0) return ATTN_OK;
    if (!q || !kcache || !vcache || !seqlens || !o) return ATTN_ERR_INVALID_ARG;
    if (k_stride_b < 0 || k_stride_h < 0 || k_stride_s < 0 || v_stride_b < 0 || v_stride_h < 0 || v_stride_s < 0)
        return ATTN_ERR_INVALID_ARG;
    if (B > 65535) return ATTN_ERR_UNSUPPORTED;
    const int G = n_q / n_kv;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (d_qk == 128 && d_v == 128) {
        if (!is_pow2(G)) return ATTN_ERR_UNSUPPORTED;
        if (k_stride_s < 128 || v_stride_s < 128) return ATTN_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(o)) return ATTN_ERR_MISALIGNED;
        if ((k_stride_b | k_stride_h | k_stride_s | v_stride_b | v_stride_h | v_stride_s) & 7)
            return ATTN_ERR_MISALIGNED;
        const size_t need = decode_ws_bytes(B, n_q, d_v, decode_n_splits(B, n_kv, G, S_max));
        if (!workspace || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
        if (reinterpret_cast<uintptr_t>(workspace) & 255u) return ATTN_ERR_MISALIGNED;
        CacheView cv{};
        cv.k = kcache;
        cv.v = vcache;
        cv.ks[0] = k_stride_b, cv.ks[1] = k_stride_h, cv.ks[2] = k_stride_s;
        cv.vs[0] = v_stride_b, cv.vs[1] = v_stride_h, cv.vs[2] = v_stride_s;
        cv.win = win;
        if (rt) cv.rt = *rt;
        return dispatch_decode_gqa<false>(G, q, cv, seqlens, o, lse, B, n_q, n_kv, S_max, scale, workspace, s);
    }
    if (win.window > 0 || rt) return ATTN_ERR_UNSUPPORTED;   // the MLA kernel has no window, no rotation
    if (d_qk == 576 && d_v == 512 && n_kv == 1) {
        // the value rows must be the first 512 columns of the key rows
        if (vcache != kcache || v_stride_b != k_stride_b || v_stride_s != k_stride_s) return ATTN_ERR_UNSUPPORTED;
        if (n_q % attn::mla::M != 0 || n_q / attn::mla::M > 65535) return ATTN_ERR_UNSUPPORTED;
        if (k_stride_s < 576) return ATTN_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(kcache) || !aligned16(o)) return ATTN_ERR_MISALIGNED;
        if ((k_stride_b | k_stride_s) & 7) return ATTN_ERR_MISALIGNED;
        if (B > 32767) return ATTN_ERR_UNSUPPORTED;
        const size_t need = mla_ws_bytes(B, n_q, S_max);
        if (need > 0) {
            if (!workspace || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
            if (reinterpret_cast<uintptr_t>(workspace) & 255u) return ATTN_ERR_MISALIGNED;
        }
        return launch_decode_mla(q, kcache, seqlens, o, lse, B, n_q, S_max, k_stride_b, k_stride_s, scale, workspace,
                                 s);
    }
    return ATTN_ERR_UNSUPPORTED;
}
}  // namespace

extern "C" {

int attn_decode(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens, void *o, float *lse,
                int B, int n_q, int n_kv, int d_qk, int d_v, int S_max, int64_t k_stride_b, int64_t k_stride_h,
                int64_t k_stride_s, int64_t v_stride_b, int64_t v_stride_h, int64_t v_stride_s, float scale,
                void *workspace, size_t workspace_bytes, attn_stream_t stream) {
    return decode_entry(q, kcache, vcache, seqlens, o, lse, B, n_q, n_kv, d_qk, d_v, S_max, k_stride_b, k_stride_h,
                        k_stride_s, v_stride_b, v_stride_h, v_stride_s, scale, workspace, workspace_bytes, stream,
                        attn::dec::Window{0, 0});
}

int attn_decode_window(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens, void *o,
                       float *lse, int B, int n_q, int n_kv, int d_qk, int d_v, int S_max, int64_t k_stride_b,
                       int64_t k_stride_h, int64_t k_stride_s, int64_t v_stride_b, int64_t v_stride_h,
                       int64_t v_stride_s, int window, int n_sink, float scale, void *workspace,
                       size_t workspace_bytes, attn_stream_t stream) {
    if (window < 1 || n_sink < 0) return ATTN_ERR_INVALID_ARG;
    if (!(d_qk == 128 && d_v == 128)) return ATTN_ERR_UNSUPPORTED;
    return decode_entry(q, kcache, vcache, seqlens, o, lse, B, n_q, n_kv, d_qk, d_v, S_max, k_stride_b, k_stride_h,
                        k_stride_s, v_stride_b, v_stride_h, v_stride_s, scale, workspace, workspace_bytes, stream,
                        attn::dec::Window{window, n_sink});
}

// ---- rotary position embedding ----
int attn_rope_tables(float *cos_t, float *sin_t, int n_pos, int d, double base, attn_stream_t stream) {
    if (n_pos < 0 || d < 2 || d % 2 != 0 || !std::isfinite(base) || !(base > 0.0)) return ATTN_ERR_INVALID_ARG;
    if (n_pos == 0) return ATTN_OK;
    if (!cos_t || !sin_t) return ATTN_ERR_INVALID_ARG;
    const long long n = (long long)n_pos * (d / 2);
    const int blocks = (int)std::min<long long>((n + 255) / 256, 4LL * 148);
    attn::rope::rope_tables_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(cos_t, sin_t, n_pos,
                                                                                             d / 2, base);
    return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // extern "C"

namespace {
bool rope_tables_ok(const float *cos_t, const float *sin_t, int n_pos) {
    return cos_t && sin_t && n_pos >= 1;
}
// x, y [BH][S][d]: grid x over the 16-byte words of S rows, y over BH.
int launch_rope_apply(const void *x, void *y, long long BH, int S, int d, int pos0, const attn::rope::Tables &t,
                      cudaStream_t stream) {
    const long long words = (long long)S * (d / 8);
    if (BH == 0 || words == 0) return ATTN_OK;
    if (words > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    const unsigned gx = (unsigned)((words + 255) / 256);
    const unsigned gy = (unsigned)std::min<long long>((BH + attn::rope::ROPE_BH - 1) / attn::rope::ROPE_BH, 65535);
    attn::rope::rope_apply_kernel<<<dim3(gx, gy), 256, 0, stream>>>(reinterpret_cast<const __nv_bfloat16 *>(x),
                                                                    reinterpret_cast<__nv_bfloat16 *>(y), BH, S, d,
                                                                    pos0, t);
    return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}
}  // namespace

extern "C" {

int attn_rope_apply(const void *x, void *y, int B, int H, int S, int d, int pos0, const float *cos_t,
                    const float *sin_t, int n_pos, attn_stream_t stream) {
    if (B < 0 || H < 0 || S < 0 || d < 8 || d % 8 != 0 || pos0 < 0) return ATTN_ERR_INVALID_ARG;
    if ((long long)B * H * S == 0) return ATTN_OK;
    if (!x || !y || !rope_tables_ok(cos_t, sin_t, n_pos)) return ATTN_ERR_INVALID_ARG;
    if ((long long)pos0 + S > n_pos) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y) || !aligned16(cos_t) || !aligned16(sin_t)) return ATTN_ERR_MISALIGNED;
    return launch_rope_apply(x, y, (long long)B * H, S, d, pos0, attn::rope::Tables{cos_t, sin_t, n_pos},
                             reinterpret_cast<cudaStream_t>(stream));
}

int attn_fwd_rope(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Sq, int Skv, int n_q,
                  int n_kv, int d_qk, int d_v, int causal, float scale, const float *cos_t, const float *sin_t,
                  int n_pos, void *k_rot, attn_stream_t stream) {
    if (B < 0 || Sq < 0 || Skv < 1 || n_q < 1 || n_kv < 1 || d_qk < 1 || d_v < 1) return ATTN_ERR_INVALID_ARG;
    if (n_q % n_kv != 0) return ATTN_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
    if (B == 0 || Sq == 0) return ATTN_OK;
    if (!q || !k || !v || !o || !k_rot || !rope_tables_ok(cos_t, sin_t, n_pos)) return ATTN_ERR_INVALID_ARG;
    if (n_pos < Skv) return ATTN_ERR_INVALID_ARG;
    if (d_qk != d_v || (d_qk != 32 && d_qk != 64 && d_qk != 128)) return ATTN_ERR_UNSUPPORTED;
    const int G = n_q / n_kv;
    if (!is_pow2(G) || G > 256) return ATTN_ERR_UNSUPPORTED;
    if (Sq > Skv) return ATTN_ERR_UNSUPPORTED;   // queries sit at the last Sq key positions
    if ((long long)B * n_q > 0x7fffffffLL || (long long)B * n_kv > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(k_rot) ||
        !aligned16(cos_t) || !aligned16(sin_t))
        return ATTN_ERR_MISALIGNED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const attn::rope::Tables t{cos_t, sin_t, n_pos};
    // keys: rotated once, into k_rot (many query tiles read each key tile)
    int rc = launch_rope_apply(k, k_rot, (long long)B * n_kv, Skv, d_qk, 0, t, s);
    if (rc != ATTN_OK) return rc;
    // queries: rotated in shared memory by the attention kernel
    switch (d_qk) {
        case 32: return launch_prefill<32>(q, k_rot, v, o, lse, B, Sq, Skv, n_q, n_kv, causal, scale, s, nullptr, 0, 0, &t);
        case 64: return launch_prefill<64>(q, k_rot, v, o, lse, B, Sq, Skv, n_q, n_kv, causal, scale, s, nullptr, 0, 0, &t);
        default: return launch_prefill<128>(q, k_rot, v, o, lse, B, Sq, Skv, n_q, n_kv, causal, scale, s, nullptr, 0, 0, &t);
    }
}

int attn_decode_rope(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens, void *o,
                     float *lse, int B, int n_q, int n_kv, int d_qk, int d_v, int S_max, int64_t k_stride_b,
                     int64_t k_stride_h, int64_t k_stride_s, int64_t v_stride_b, int64_t v_stride_h,
                     int64_t v_stride_s, const float *cos_t, const float *sin_t, int n_pos, float scale,
                     void *workspace, size_t workspace_bytes, attn_stream_t stream) {
    if (!rope_tables_ok(cos_t, sin_t, n_pos)) return ATTN_ERR_INVALID_ARG;
    if (!(d_qk == 128 && d_v == 128)) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(cos_t) || !aligned16(sin_t)) return ATTN_ERR_MISALIGNED;
    const attn::rope::Tables t{cos_t, sin_t, n_pos};
    return decode_entry(q, kcache, vcache, seqlens, o, lse, B, n_q, n_kv, d_qk, d_v, S_max, k_stride_b, k_stride_h,
                        k_stride_s, v_stride_b, v_stride_h, v_stride_s, scale, workspace, workspace_bytes, stream,
                        attn::dec::Window{0, 0}, &t);
}

int attn_decode_fp8_workspace_bytes(int B, int n_q, int n_kv, int S_max, size_t *bytes) {
    if (!bytes || B < 0 || n_q < 1 || n_kv < 1 || S_max < 1 || n_q % n_kv != 0) return ATTN_ERR_INVALID_ARG;
    *bytes = decode_ws_bytes(B, n_q, 128, decode_n_splits(B, n_kv, n_q / n_kv, S_max, true));
    return ATTN_OK;
}

int attn_decode_fp8(const void *q, const void *kcache, const void *vcache, const float *k_scale,
                    const float *v_scale, const int32_t *seqlens, void *o, float *lse, int B, int n_q, int n_kv,
                    int S_max, int64_t k_stride_b, int64_t k_stride_h, int64_t k_stride_s, int64_t v_stride_b,
                    int64_t v_stride_h, int64_t v_stride_s, float scale, void *workspace, size_t workspace_bytes,
                    attn_stream_t stream) {
    if (B < 0 || n_q < 1 || n_kv < 1 || S_max < 1 || n_q % n_kv != 0) return ATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
    if (B == 0) return ATTN_OK;
    if (!q || !kcache || !vcache || !k_scale || !v_scale || !seqlens || !o) return ATTN_ERR_INVALID_ARG;
    if (k_stride_b < 0 || k_stride_h < 0 || k_stride_s < 0 || v_stride_b < 0 || v_stride_h < 0 || v_stride_s < 0)
        return ATTN_ERR_INVALID_ARG;
    if (k_stride_s < 128 || v_stride_s < 128) return ATTN_ERR_INVALID_ARG;
    if (B > 65535) return ATTN_ERR_UNSUPPORTED;
    const int G = n_q / n_kv;
    if (!is_pow2(G)) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(o)) return ATTN_ERR_MISALIGNED;
    if ((k_stride_b | k_stride_h | k_stride_s | v_stride_b | v_stride_h | v_stride_s) & 15)
        return ATTN_ERR_MISALIGNED;   // one-byte elements: strides in multiples of 16 bytes
    size_t need = 0;
    attn_decode_fp8_workspace_bytes(B, n_q, n_kv, S_max, &need);
    if (!workspace || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return ATTN_ERR_MISALIGNED;
    CacheView cv{};
    cv.k = kcache;
    cv.v = vcache;
    cv.ks[0] = k_stride_b, cv.ks[1] = k_stride_h, cv.ks[2] = k_stride_s;
    cv.vs[0] = v_stride_b, cv.vs[1] = v_stride_h, cv.vs[2] = v_stride_s;
    cv.fs.k_scale = k_scale;
    cv.fs.v_scale = v_scale;
    return dispatch_decode_gqa<false, true>(G, q, cv, seqlens, o, lse, B, n_q, n_kv, S_max, scale, workspace,
                                            reinterpret_cast<cudaStream_t>(stream));
}

int attn_decode_fp8_tiles(const void *q, const void *kcache, const void *vcache, const float *k_scales,
                          const float *v_scales, const int32_t *seqlens, void *o, float *lse, int B, int n_q, int n_kv,
                          int S_max, int64_t k_stride_b, int64_t k_stride_h, int64_t k_stride_s,
                          int64_t v_stride_b, int64_t v_stride_h, int64_t v_stride_s, float scale, void *workspace,
                          size_t workspace_bytes, attn_stream_t stream) {
    if (B < 0 || n_q < 1 || n_kv < 1 || S_max < 1 || n_q % n_kv != 0) return ATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
    if (B == 0) return ATTN_OK;
    if (!q || !kcache || !vcache || !k_scales || !v_scales || !seqlens || !o) return ATTN_ERR_INVALID_ARG;
    if (k_stride_b < 0 || k_stride_h < 0 || k_stride_s < 0 || v_stride_b < 0 || v_stride_h < 0 || v_stride_s < 0)
        return ATTN_ERR_INVALID_ARG;
    if (k_stride_s < 128 || v_stride_s < 128) return ATTN_ERR_INVALID_ARG;
    if (B > 65535) return ATTN_ERR_UNSUPPORTED;
    const int G = n_q / n_kv;
    if (!is_pow2(G)) return ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(o)) return ATTN_ERR_MISALIGNED;
    if ((k_stride_b | k_stride_h | k_stride_s | v_stride_b | v_stride_h | v_stride_s) & 15)
        return ATTN_ERR_MISALIGNED;   // one-byte elements: strides in multiples of 16 bytes
    size_t need = 0;
    attn_decode_fp8_workspace_bytes(B, n_q, n_kv, S_max, &need);
    if (!workspace || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return ATTN_ERR_MISALIGNED;
    CacheView cv{};
    cv.k = kcache;
    cv.v = vcache;
    cv.ks[0] = k_stride_b, cv.ks[1] = k_stride_h, cv.ks[2] = k_stride_s;
    cv.vs[0] = v_stride_b, cv.vs[1] = v_stride_h, cv.vs[2] = v_stride_s;
    cv.fs.k_scale = k_scales;
    cv.fs.v_scale = v_scales;
    cv.fs.tile_stride = (S_max + attn::dec::KT - 1) / attn::dec::KT;
    return dispatch_decode_gqa<false, true>(G, q, cv, seqlens, o, lse, B, n_q, n_kv, S_max, scale, workspace,
                                            reinterpret_cast<cudaStream_t>(stream));
}

int attn_decode_paged(const void *q, const void *k_pages, const void *v_pages, const int32_t *block_table,
                      const int32_t *seqlens, void *o, float *lse, int B, int n_q, int n_kv, int d_qk, int d_v,
                      int page_size, int pages_per_seq, int num_pages, int64_t k_stride_page,
                      int64_t k_stride_token, int64_t k_stride_head, int64_t v_stride_page, int64_t v_stride_token,
                      int64_t v_stride_head, float scale, void *workspace, size_t workspace_bytes,
                      attn_stream_t stream) {
    if (B < 0 || n_q < 1 || n_kv < 1 || n_q % n_kv != 0) return ATTN_ERR_INVALID_ARG;
    if (page_size < 1 || pages_per_seq < 1 || num_pages < 1) return ATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
    if ((long long)page_size * pages_per_seq > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
    if (B == 0) return ATTN_OK;
    if (!q || !k_pages || !v_pages || !block_table || !seqlens || !o) return ATTN_ERR_INVALID_ARG;
    if (k_stride_page < 0 || k_stride_token < 0 || k_stride_head < 0 || v_stride_page < 0 || v_stride_token < 0 ||
        v_stride_head < 0)
        return ATTN_ERR_INVALID_ARG;
    if (!(d_qk == 128 && d_v == 128)) return ATTN_ERR_UNSUPPORTED;
    // a page is whole TMA boxes of up to 128 rows: 16, 32, 64 or a multiple of 128 tokens
    if (!(page_size == 16 || page_size == 32 || page_size == 64 || (page_size % 128 == 0 && is_pow2(page_size))))
        return ATTN_ERR_UNSUPPORTED;
    if (B > 65535) return ATTN_ERR_UNSUPPORTED;
    const int G = n_q / n_kv;
    if (!is_pow2(G)) return ATTN_ERR_UNSUPPORTED;
    if (k_stride_token < 128 || v_stride_token < 128) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o)) return ATTN_ERR_MISALIGNED;
    if ((k_stride_page | k_stride_token | k_stride_head | v_stride_page | v_stride_token | v_stride_head) & 7)
        return ATTN_ERR_MISALIGNED;
    const int S_max = page_size * pages_per_seq;
    const size_t need = decode_ws_bytes(B, n_q, d_v, decode_n_splits(B, n_kv, G, S_max));
    if (!workspace || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return ATTN_ERR_MISALIGNED;
    CacheView cv{};
    cv.k = k_pages;
    cv.v = v_pages;
    cv.ks[0] = k_stride_page, cv.ks[1] = k_stride_token, cv.ks[2] = k_stride_head;
    cv.vs[0] = v_stride_page, cv.vs[1] = v_stride_token, cv.vs[2] = v_stride_head;
    cv.page_size = page_size;
    cv.pt.table = block_table;
    cv.pt.pages_per_seq = pages_per_seq;
    int shift = 0;
    while ((1 << shift) < page_size) ++shift;
    cv.pt.page_shift = shift;
    cv.pt.box_rows = page_size < attn::dec::KT ? page_size : attn::dec::KT;
    cv.pt.num_pages = num_pages;
    return dispatch_decode_gqa<true>(G, q, cv, seqlens, o, lse, B, n_q, n_kv, S_max, scale, workspace,
                                     reinterpret_cast<cudaStream_t>(stream));
}

const char *attn_status_string(int status) {
    switch (status) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_INVALID_ARG: return "invalid argument";
        case ATTN_ERR_UNSUPPORTED: return "unsupported configuration";
        case ATTN_ERR_MISALIGNED: return "pointer or stride not 16-byte aligned";
        case ATTN_ERR_WORKSPACE: return "workspace missing or too small";
        case ATTN_ERR_CUDA: return "CUDA error";
        case ATTN_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait expired on the device";
        case ATTN_ERR_DEVICE_RANGE: return "a device-side value was out of range and clamped";
        default: return "unknown status";
    }
}

int attn_device_status(attn_stream_t stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
    unsigned int st = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&st, g_status, sizeof(st)) != cudaSuccess) return ATTN_ERR_CUDA;
    if (st == 0) return ATTN_OK;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return ATTN_ERR_CUDA;
    if (cudaMemcpyToSymbol(attn::g_timeout_site, &zero, sizeof(zero)) != cudaSuccess) return ATTN_ERR_CUDA;
    if (st & attn::kStatusTimeout) return ATTN_ERR_DEVICE_TIMEOUT;
    return ATTN_ERR_DEVICE_RANGE;
}

int attn_selftest_ex2(const float *x, float *y_poly, float *y_sfu, int n, attn_stream_t stream) {
    if (n < 0 || (n > 0 && (!x || !y_poly || !y_sfu))) return ATTN_ERR_INVALID_ARG;
    if (n == 0) return ATTN_OK;
    const int pairs = (n + 1) / 2;
    selftest_ex2_kernel<<<(pairs + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y_poly, y_sfu,
                                                                                                n);
    return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_selftest_timeout(int timeout_us, attn_stream_t stream) {
    if (timeout_us < 1 || timeout_us > 1000000) return ATTN_ERR_INVALID_ARG;
    selftest_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        (unsigned long long)timeout_us * 1000ull);
    return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// attn_decode_noalloc: the decode step for callers that cannot allocate.
//
// Its split-KV scratch (partial outputs and their softmax statistics) lives
// in the file-scope array below instead of a caller-provided workspace. In
// host code `g_noalloc_scratch` names only a host-side stand-in, so the
// device address is looked up once per device with cudaGetSymbolAddress
// (with that device current) and passed to the kernels.
// ---------------------------------------------------------------------------
namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void *g_noalloc_ptr[64] = {};
CUcontext g_noalloc_ctx[64] = {};   // the context each cached address belongs to

// The current CUDA context, through the runtime's driver entry point (the
// library does not link the driver library itself). nullptr if unavailable.
CUcontext current_context() {
    typedef CUresult (*GetCurrentFn)(CUcontext *);
    static GetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult qres;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<GetCurrentFn>(ptr);
    });
    CUcontext ctx = nullptr;
    if (fn == nullptr || fn(&ctx) != CUDA_SUCCESS) return nullptr;
    return ctx;
}

// Device address of the scratch array on the current device. The first call
// on a device does the lookup; so does the first call after the device's
// context changed (cudaDeviceReset loads the module, and the array, anew).
// Returns nullptr on failure.
void *noalloc_scratch_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    // (no context is current on a thread before its first runtime call that
    // needs one: the lookup below makes the device's primary context current)
    const CUcontext ctx = current_context();
    if (g_noalloc_ptr[dev] == nullptr || ctx == nullptr || ctx != g_noalloc_ctx[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_noalloc_ptr[dev] = ptr;
        g_noalloc_ctx[dev] = current_context();
    }
    return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" int attn_decode_noalloc(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens,
                                   void *o, float *lse, int B, int n_q, int n_kv, int d_qk, int d_v, int S_max,
                                   int64_t k_stride_b, int64_t k_stride_h, int64_t k_stride_s,
                                   int64_t v_stride_b, int64_t v_stride_h, int64_t v_stride_s, float scale,
                                   attn_stream_t stream) {
    if (B < 0 || n_q < 1 || n_kv < 1 || S_max < 1 || n_q % n_kv != 0) return ATTN_ERR_INVALID_ARG;
    if (B == 0) return ATTN_OK;
    if (!(d_qk == 128 && d_v == 128)) return ATTN_ERR_UNSUPPORTED;
    const size_t need = decode_ws_bytes(B, n_q, d_v, decode_n_splits(B, n_kv, n_q / n_kv, S_max));
    if (need > (size_t)ATTN_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_WORKSPACE;  // beyond the static maximum
    void *scratch = noalloc_scratch_ptr();
    if (scratch == nullptr) return ATTN_ERR_CUDA;
    return attn_decode(q, kcache, vcache, seqlens, o, lse, B, n_q, n_kv, d_qk, d_v, S_max, k_stride_b, k_stride_h,
                       k_stride_s, v_stride_b, v_stride_h, v_stride_s, scale, scratch, need, stream);
}
