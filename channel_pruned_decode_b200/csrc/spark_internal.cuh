// Internal helpers of the SparK sm_100a library: element access, async bulk
// copies with mbarrier completion, bounded waits, and the launch geometry
// that both the entry points and the workspace-size query must agree on.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "spark.h"

namespace spark {

constexpr int kD = 128;               // head dimension the kernels are built for
constexpr int kMaskWords = kD / 32;   // 128-bit channel mask per token
constexpr int kWsHeader = 256;        // status word + padding at workspace start
constexpr uint32_t kDevTimeout = 1u;  // status bit: a bounded wait ran out
constexpr uint32_t kDevBadArg = 2u;   // status bit: a device-side length or budget was out of range

// ------------------------------------------------------- argument checks
inline int elem_size(int dtype) { return dtype == SPARK_F32 ? 4 : (dtype == SPARK_BF16 ? 2 : 0); }

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape and pointer checks of a cache descriptor shared by every entry point
// that reads or writes one; returns SPARK_OK or the error status.
inline int check_cache(const spark_kcache *kc) {
    if (!kc) return SPARK_ERR_ARG;
    if (kc->B < 0 || kc->Hkv < 0 || kc->S < 0) return SPARK_ERR_ARG;
    if (elem_size(kc->dtype) == 0) return SPARK_ERR_ARG;
    if (kc->D != kD) return SPARK_ERR_UNSUPPORTED;
    if (kc->T < 0 || kc->T > kc->D) return SPARK_ERR_ARG;
    if (kc->lens && (reinterpret_cast<uintptr_t>(kc->lens) & 3u)) return SPARK_ERR_ARG;
    if ((long)kc->B * kc->Hkv == 0) return SPARK_OK;
    if (!kc->qn || !kc->stats || !aligned16(kc->qn) || !aligned16(kc->stats)) return SPARK_ERR_ARG;
    if (kc->S > 0) {
        if (!kc->mask || !aligned16(kc->mask)) return SPARK_ERR_ARG;
        if (kc->T > 0 && (!kc->vals || !aligned16(kc->vals))) return SPARK_ERR_ARG;
    }
    return SPARK_OK;
}

// Every check of spark_prune's arguments except the workspace: the cache
// descriptor, the window sizes and the input pointers.  spark_prune and its
// allocation-free variant differ only in where the scratch comes from.
inline int check_prune_args(const void *k, const void *q_obs, int G, int W, const spark_kcache *out) {
    const int rc = check_cache(out);
    if (rc != SPARK_OK) return rc;
    if (G < 1 || W < 1) return SPARK_ERR_ARG;
    if ((long)out->B * out->Hkv == 0) return SPARK_OK;
    if (!q_obs || !aligned16(q_obs)) return SPARK_ERR_ARG;
    if (out->S > 0 && (!k || !aligned16(k))) return SPARK_ERR_ARG;
    return SPARK_OK;
}

// ----------------------------------------------------------------- prune
constexpr int kPruneThreads = 128;    // 4 lanes per token, 32 tokens per group
constexpr int kPruneGroups = 8;       // fewest 32-token groups per CTA (256 tokens)
constexpr int kPruneGroupsMax = 32;   // most (1024 tokens) for large launches
constexpr int kMaxGroups = 8;         // SparK-g channel groups

// 32-token groups per prune CTA: 8, doubled (up to 32) while the launch still
// has >= 2368 CTAs (16 per SM at 4 resident per SM), which amortises each
// CTA's setup and the cold start of its threshold estimates.
inline int prune_groups_per_cta(long BH, int S) {
    int g = kPruneGroups;
    while (g < kPruneGroupsMax && BH * (long)((S + 64L * g - 1) / (64L * g)) >= 2368) g *= 2;
    return g;
}

inline int prune_chunks(int S, int groups_per_cta = kPruneGroups) {
    const int per = 32 * groups_per_cta;
    return S > 0 ? (S + per - 1) / per : 0;
}

// sized for the smallest chunks, so any groups-per-CTA choice fits
inline size_t prune_workspace(long BH, int S) {
    return kWsHeader + (size_t)BH * (size_t)prune_chunks(S) * 2 * sizeof(double);
}

// SparK-g with four groups also keeps one byte per channel and head (the
// channels' slots in the key exchange) after the partials
inline size_t prune_slots_offset(long BH, int S) { return (prune_workspace(BH, S) + 255) / 256 * 256; }
inline size_t prune_grouped_workspace(long BH, int S) { return prune_slots_offset(BH, S) + (size_t)BH * kD; }

// SparK-p workspace: the prune partials with a third one per chunk (the
// data-dependent pruned count), then per group the largest kept count, then
// per head its rows and its first row (the value layout's scan)
struct ToppWs {
    double *partial;
    uint32_t *tg;
    uint32_t *hrows;
    uint32_t *hbase;
};

inline size_t topp_partials_bytes(long BH, int S) {
    return ((size_t)BH * (size_t)prune_chunks(S) * 3 * sizeof(double) + 255) / 256 * 256;
}

inline size_t topp_groups(long BH, int S) { return (size_t)BH * (((size_t)S + 31) / 32); }

inline size_t topp_workspace(long BH, int S) {
    return kWsHeader + topp_partials_bytes(BH, S) + (topp_groups(BH, S) * 4 + 255) / 256 * 256 +
           2 * (((size_t)BH * 4 + 255) / 256 * 256);
}

inline ToppWs topp_ws_layout(void *ws, long BH, int S) {
    char *p = static_cast<char *>(ws) + kWsHeader;
    ToppWs t;
    t.partial = reinterpret_cast<double *>(p);
    p += topp_partials_bytes(BH, S);
    t.tg = reinterpret_cast<uint32_t *>(p);
    p += (topp_groups(BH, S) * 4 + 255) / 256 * 256;
    t.hrows = reinterpret_cast<uint32_t *>(p);
    p += ((size_t)BH * 4 + 255) / 256 * 256;
    t.hbase = reinterpret_cast<uint32_t *>(p);
    return t;
}

// ---------------------------------------------------------------- decode
// recovery selector of the decode kernel beyond spark_recovery: Degenerate F
// over a SparK-p cache (masks may hold fewer bits than the T value slots)
constexpr int kRecoveryDegVar = 3;
// Degenerate F with the channel-order q.k~ loop (chosen for large T)
constexpr int kRecoveryDegDense = 4;

// Each warp of a persistent CTA is an independent flash-decoding worker.  Its
// ring of shared-memory stages holds the mask and kept values of one 32-token
// tile each; the tile's dense V rows go straight to registers.
constexpr int kWT = 32;               // tokens per warp tile
constexpr int kMaxWarps = 16;         // warps per CTA
constexpr int kMaxStagesW = 4;        // ring depth per warp

struct DecodeGeom {
    int chunk;        // prefix tokens per work item (multiple of kWT)
    int n_pre;        // prefix items per (row, kv head)
    int units;        // n_pre + 1 (the last item of a head is its dense tail)
    int nstage;       // stages per warp
    int nwarp;        // warps per CTA
    int ctas;         // persistent grid size
    size_t warp_bytes;  // shared memory of one warp (tables + ring)
    size_t smem;        // dynamic shared memory per CTA
};

// mask (16 B/token) + one 32-token group of kept values
__host__ __device__ inline size_t dec_stage_bytes(int T, int es) {
    return (size_t)kWT * 16 + (size_t)kWT * T * es;
}

// Per-warp tables: bf16 values add a swizzled V tile [kWT][kD] (8 KB); then
// p as [G][kWT] fp32, q' [kD][G], c [kD], for fp32 values p as duplicated
// pairs [kWT][G][2] (the CUDA-core P.V; bf16 values take p from the first
// table), Qc [16] and the ring's mbarriers; rounded to 128 bytes so that the
// stages start aligned.
__host__ __device__ inline size_t dec_vtile_bytes(int es) { return es == 2 ? (size_t)kWT * kD * 2 : 0; }
__host__ __device__ inline size_t dec_pdup_bytes(int G, int es) { return es == 2 ? 0 : (size_t)kWT * G * 8; }
__host__ __device__ inline size_t dec_table_bytes(int G, int es) {
    const size_t b = dec_vtile_bytes(es) + (size_t)G * kWT * 4 + (size_t)kD * G * 4 + kD * 4 +
                     dec_pdup_bytes(G, es) + 64 + kMaxStagesW * 8;
    return (b + 127) / 128 * 128;
}

// Tv >= 0: the stage also carries a pruned value cache (mask + Tv values per
// token); Tv < 0: values are read dense
DecodeGeom decode_geometry(long BH, int S, int T, int Tv, int es, int G, int num_sms);

// partials: acc [BH][units][G][D] fp32, then (m, l) [BH][units][G][2] fp32
inline size_t decode_workspace(long BH, const DecodeGeom &g, int G) {
    return kWsHeader + (size_t)BH * g.units * G * (kD + 2) * sizeof(float);
}

// ------------------------------------------------------- element access
template <typename E> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float to_f(float x) { return x; }
    static constexpr int size = 4;
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
    static constexpr int size = 2;
};

// Prompt tokens of head bh: S, or the row's entry of a per-row length array
// (row = bh / Hkv), clamped to [0, S]; an out-of-range entry is recorded in
// the status word.
__device__ __forceinline__ int row_len(const int32_t *lens, long bh, int Hkv, int S, uint32_t *status) {
    if (!lens) return S;
    const int n = lens[bh / Hkv];
    if (n < 0 || n > S) {
        if (status) atomicOr(status, kDevBadArg);
        return n < 0 ? 0 : S;
    }
    return n;
}

// ------------------------------------------------------------- PTX glue
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `parity` of an mbarrier, giving up after `limit_ns` of
// device time (and after at most 2^26 polls).  Returns false on timeout (the
// caller records it and winds down).
__device__ __forceinline__ bool mbar_wait_limit(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t it = 0; it < (1u << 26); ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 63u && global_ns() - t0 > limit_ns) return false;
    }
    return false;
}

// the pipeline's waits give up after ~1 s
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
    return mbar_wait_limit(bar, parity, 1000000000ull);
}

// Async bulk copy global -> shared, completion counted on `bar` (bytes).
// Both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// order-preserving float <-> int map for integer warp max reductions
__device__ __forceinline__ int f2ord(float f) {
    int i = __float_as_int(f);
    return i ^ ((i >> 31) & 0x7fffffff);
}
__device__ __forceinline__ float ord2f(int i) {
    return __int_as_float(i ^ ((i >> 31) & 0x7fffffff));
}

}  // namespace spark
