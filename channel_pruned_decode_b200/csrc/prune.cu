// Prefill channel pruning for SparK on sm_100a.
//
// Method: "KV Cache 还能再砍一刀：SparK ..." (paper walkthrough) section 3.1
// (relaxed objective max sum_j w^j z^j with sum_j z^j = T, proxy saliency
// w = ||q^j||_2 * ||k^j||_2, greedy top-T), 3.2 (observation-window queries,
// per-token unstructured mask) and 3.3 step 1 (the cache stores the pruned
// key, the channel mask and the saliency statistics).
//
// Three launches on the caller's stream:
//   qnorm_kernel   one CTA per (row, kv head), one thread per channel: the
//                  fp64 sum of squares over the G*W window rows of the group,
//                  rounded once to fp32.
//   prune_kernel   one CTA per 256-token chunk of one (row, kv head).  Four
//                  lanes own one token (32 channels each, saliency keys kept in
//                  registers); the T-th largest key is found by a quad-level
//                  bisection on the fp32 bit pattern (w >= 0, so the bit
//                  pattern is monotone in w), ties broken toward the lower
//                  channel by an exclusive scan across the quad.  Kept values
//                  are staged in shared memory in the 32-token interleaved
//                  layout and written back with 16-byte stores; fp32 partial
//                  sums of the pruned saliencies go to fp64 per-lane
//                  accumulators and one fp64 partial per CTA.
//   stats_kernel   fixed-order fp64 sum of the CTA partials per head, then
//                  N = S*(D-T) and mu_pruned = sum w / N.
// All reductions have a fixed order, so reruns are bit-identical.
#include "spark_internal.cuh"

#include <cuda_fp16.h>

namespace spark {

template <typename E>
__global__ void __launch_bounds__(kD) qnorm_kernel(const E *__restrict__ q_obs, int G, int W,
                                                   float *__restrict__ qn) {
    const long bh = blockIdx.x;
    const int j = threadIdx.x;
    const E *base = q_obs + (size_t)bh * G * W * kD + j;
    double acc = 0.0;
    for (int g = 0; g < G; ++g)
        for (int t = 0; t < W; ++t) {
            const double x = (double)Elem<E>::to_f(base[((size_t)g * W + t) * kD]);
            acc = __dadd_rn(acc, __dmul_rn(x, x));  // square of an fp32 value is exact in fp64
        }
    qn[bh * kD + j] = __double2float_rn(sqrt(acc));
}

// Per-lane view of 32 consecutive channels of one key row.
template <typename E> struct KSlice;

template <> struct KSlice<__nv_bfloat16> {
    static constexpr int kWords = 16;  // 32 bf16
    uint32_t w[kWords];
    __device__ __forceinline__ void load(const __nv_bfloat16 *row) {
        const uint4 *p = reinterpret_cast<const uint4 *>(row);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 v = __ldcs(p + i);  // streamed once: evict-first
            w[4 * i + 0] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
    }
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int i = 0; i < kWords; ++i) w[i] = 0u;
    }
    // |k| as fp32 bits
    __device__ __forceinline__ uint32_t abs_bits(int i) const {
        const uint32_t x = w[i >> 1];
        return (i & 1) ? (x & 0x7fff0000u) : ((x << 16) & 0x7fffffffu);
    }
    __device__ __forceinline__ uint16_t raw(int i) const {
        const uint32_t x = w[i >> 1];
        return (uint16_t)((i & 1) ? (x >> 16) : (x & 0xffffu));
    }
};

template <> struct KSlice<float> {
    static constexpr int kWords = 32;
    uint32_t w[kWords];
    __device__ __forceinline__ void load(const float *row) {
        const uint4 *p = reinterpret_cast<const uint4 *>(row);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint4 v = __ldcs(p + i);
            w[4 * i + 0] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
    }
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int i = 0; i < kWords; ++i) w[i] = 0u;
    }
    __device__ __forceinline__ uint32_t abs_bits(int i) const { return w[i] & 0x7fffffffu; }
    __device__ __forceinline__ uint32_t raw(int i) const { return w[i]; }
};

template <typename E> struct RawT { using type = uint16_t; };
template <> struct RawT<float> { using type = uint32_t; };

// Exclusive prefix sum of v over the 4 lanes of a quad (lane & 3 = position).
__device__ __forceinline__ int quad_excl_scan(int v, int s) {
    int incl = v;
    int t = __shfl_up_sync(0xffffffffu, incl, 1);
    if (s >= 1) incl += t;
    t = __shfl_up_sync(0xffffffffu, incl, 2);
    if (s >= 2) incl += t;
    return incl - v;
}

__device__ __forceinline__ int quad_sum(int v) {
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    return v;
}

// Count of the quad's keys >= mid over the packed 16-bit keys.  A key16 is
// the upper half of the fp32 saliency (a positive bf16 pattern), clamped to
// 0x7bff: read as fp16 bit patterns these stay in the same order, and fp16
// packed compare + add (one instruction each per two channels) count them.
// `mid` is 0 or >= 0x400 (a normal fp16 pattern); keys below 0x400 sit below
// every probe.  Counts <= 32 per lane are exact in fp16.
__device__ __forceinline__ __half quad_count16(const uint32_t (&kp)[16], uint32_t mid) {
    const uint32_t mm = mid * 0x10001u;
    const __half2 m2 = *reinterpret_cast<const __half2 *>(&mm);
    const __half2 z = __float2half2_rn(0.f);
    __half2 a0 = z, a1 = z, a2 = z, a3 = z;
#pragma unroll
    for (int i = 0; i < 16; i += 4) {
        a0 = __hadd2(a0, __hge2(*reinterpret_cast<const __half2 *>(&kp[i + 0]), m2));
        a1 = __hadd2(a1, __hge2(*reinterpret_cast<const __half2 *>(&kp[i + 1]), m2));
        a2 = __hadd2(a2, __hge2(*reinterpret_cast<const __half2 *>(&kp[i + 2]), m2));
        a3 = __hadd2(a3, __hge2(*reinterpret_cast<const __half2 *>(&kp[i + 3]), m2));
    }
    a0 = __hadd2(__hadd2(a0, a1), __hadd2(a2, a3));
    // both halves -> one count (<= 32, exact), then the quad's sum (<= 128, exact)
    __half c = __hadd(__low2half(a0), __high2half(a0));
    c = __hadd(c, __shfl_xor_sync(0xffffffffu, c, 1));
    c = __hadd(c, __shfl_xor_sync(0xffffffffu, c, 2));
    return c;
}

__device__ __forceinline__ int quad_count32(const uint32_t (&key)[32], uint32_t mid) {
    int c = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) c += (key[i] >= mid) ? 1 : 0;
    return quad_sum(c);
}

// Mask word (32 channels) of this lane's quarter of the token: the T largest
// exact fp32 keys over the quad, ties to the lower channel index.
//
// Phase 1 searches the T-th largest 16-bit key with packed counts, starting
// at the previous token's threshold `tau16` and galloping outward until the
// bracket closes, then bisecting; it ends either with a probe that leaves
// exactly T keys above it (the usual case) or with the 16-bit tie band
// [tau16, tau16+1) holding the boundary.  Phase 2 bisects the exact 32-bit
// keys inside that band.  Both loops have warp-uniform trip counts (quads
// that are done idle), so the quad shuffles always see the full warp.
__device__ __forceinline__ uint32_t select_top_t(const uint32_t (&key)[32], const uint32_t (&kp)[16], int T,
                                                 int s, uint32_t &tau16) {
    if (T <= 0) return 0u;
    if (T >= kD) return 0xffffffffu;

    // ---- phase 1: 16-bit keys.  count(>= lo) >= T > count(>= hi).
    // Probes: the previous token's threshold, then galloping away from an
    // open side of the bracket (step doubling), then bisection.  The bracket
    // update is written with selects so that quads in different states of
    // the search do not diverge.
    constexpr uint32_t kTop = 0x7c00u;  // above the clamp: nothing reaches it
    const __half hT = __int2half_rn(T);
    uint32_t lo = 0u, hi = kTop;
    __half c_hi_h = __int2half_rn(0);
    bool exact = false;
    bool done = false;
    uint32_t step = 64u;
    uint32_t mid = min(max(tau16, 1u), kTop - 1u);
    while (__any_sync(0xffffffffu, !done)) {
        const uint32_t probe = (mid > 0u && mid < 0x400u) ? 0x400u : mid;
        const __half c = quad_count16(kp, probe);
        const bool ge = __hge(c, hT);
        const bool eq = __heq(c, hT);
        const bool act = !done;
        lo = (act && ge) ? mid : lo;
        hi = (act && !ge) ? mid : hi;
        c_hi_h = (act && !ge) ? c : c_hi_h;
        exact = exact || (act && eq);
        done = done || eq || (hi - lo <= 1u);
        const bool up = (hi == kTop), down = (lo == 0u);
        const uint32_t gal_up = min(lo + step, kTop - 1u);
        const uint32_t gal_dn = max(hi > step ? hi - step : hi >> 1, 1u);
        const uint32_t bis = lo + ((hi - lo) >> 1);
        mid = up ? gal_up : (down ? gal_dn : bis);
        step = (up || down) ? step << 1 : step;
    }
    int c_hi = __half2int_rn(c_hi_h);
    tau16 = lo;

    // ---- phase 2: exact keys inside the band of 16-bit key == lo.  Quads
    // whose phase 1 was exact skip it (done2) but stay in the uniform loop.
    // Bands in fp32 key space: [0, 0x400 << 16) for lo == 0 (every probe
    // below 0x400 acts as 0x400), [0x7bff << 16, 2^31) for the clamp value,
    // [lo << 16, (lo + 1) << 16) otherwise.  When exact, exactly T keys have a
    // 16-bit key >= lo, i.e. an fp32 key >= max(lo, 0x400) << 16.
    uint32_t lo32 = exact ? (max(lo, 0x400u) << 16) : ((lo == 0u) ? 0u : (lo << 16));
    uint32_t hi32 = (lo == 0u) ? (0x400u << 16) : ((lo >= 0x7bffu) ? 0x80000000u : ((lo + 1u) << 16));
    bool exact32 = exact;
    bool done2 = exact || (hi32 - lo32 <= 1u);
    while (__any_sync(0xffffffffu, !done2)) {
        const uint32_t mid32 = lo32 + ((hi32 - lo32) >> 1);
        const int c = quad_count32(key, mid32);
        if (!done2) {
            if (c >= T) {
                lo32 = mid32;
                if (c == T) { exact32 = true; done2 = true; }
            } else {
                hi32 = mid32;
                c_hi = c;
            }
            if (hi32 - lo32 <= 1u) done2 = true;
        }
    }
    // exact32: exactly T keys are >= lo32.  Otherwise lo32 is the T-th largest
    // key, c_hi keys are above it, and the first T - c_hi keys equal to it (in
    // channel order over the quad) are kept.
    const uint32_t thr = exact32 ? lo32 : lo32 + 1u;
    uint32_t m = 0u;
#pragma unroll
    for (int i = 0; i < 32; ++i) m |= (key[i] >= thr ? 1u : 0u) << i;
    if (__any_sync(0xffffffffu, !exact32)) {  // warp-uniform: the scan below shuffles
        int e = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) e += (key[i] == lo32) ? 1 : 0;
        int r = quad_excl_scan(e, s);
        if (!exact32) {
            const int need = T - c_hi;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if (key[i] == lo32) {
                    if (r < need) m |= 1u << i;
                    ++r;
                }
            }
        }
    }
    return m;
}
template <typename E>
__global__ void __launch_bounds__(kPruneThreads, 4)
    prune_kernel(const E *__restrict__ k, const float *__restrict__ qn, uint32_t *__restrict__ mask,
                 E *__restrict__ vals, double *__restrict__ partial, int S, int T, int n_chunks) {
    using Raw = typename RawT<E>::type;
    __shared__ __align__(16) Raw vtile[2][kD * 32];  // [kept index][token in group]
    __shared__ double red[2][kPruneThreads / 32];
    // window-query norms of this head, one padded row per quarter (stride 36
    // floats): the 4 quarters' 16-byte reads fall in distinct banks
    __shared__ __align__(16) float qs[4 * 36];

    const long bh = blockIdx.x / n_chunks;
    const int chunk = blockIdx.x % n_chunks;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int s = lane & 3;                 // quarter: channels [32s, 32s+32)
    const int tl = warp * 8 + (lane >> 2);  // token within the 32-token group
    const long S32 = ((long)S + 31) / 32 * 32;

    if (tid < kD) qs[(tid >> 5) * 36 + (tid & 31)] = __ldg(qn + bh * kD + tid);
    __syncthreads();

    uint32_t tau16 = 0x3f80u;  // reset from the first token's keys below
    double acc_w = 0.0, acc_w2 = 0.0;
    const long g_first = (long)chunk * kPruneGroups;
    KSlice<E> ks, ks_next;
    {
        const long t = g_first * 32 + tl;
        if (t < S) ks.load(k + ((size_t)bh * S + t) * kD + 32 * s);
        else ks.zero();
    }
    for (int gi = 0; gi < kPruneGroups; ++gi) {
        const long grp = g_first + gi;
        const long t0 = grp * 32;
        if (t0 >= S) break;  // uniform across the CTA
        const long t = t0 + tl;
        const bool valid = t < S;
        // prefetch the next group's slice while this one is selected
        {
            const long tn = t + 32;
            if (gi + 1 < kPruneGroups && tn < S) ks_next.load(k + ((size_t)bh * S + tn) * kD + 32 * s);
            else ks_next.zero();
        }

        // exact fp32 saliency keys and their packed 16-bit truncations
        uint32_t key[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float4 q4 = *reinterpret_cast<const float4 *>(qs + s * 36 + 4 * c);
            const float qq[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                key[4 * c + e] = __float_as_uint(__fmul_rn(qq[e], __uint_as_float(ks.abs_bits(4 * c + e))));
        }
        uint32_t kp[16];
        {
            const uint32_t cap = 0x7bff7bffu;
            const __half2 cap2 = *reinterpret_cast<const __half2 *>(&cap);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t pr = __byte_perm(key[2 * i], key[2 * i + 1], 0x7632);
                const __half2 c = __hmin2(*reinterpret_cast<const __half2 *>(&pr), cap2);
                kp[i] = *reinterpret_cast<const uint32_t *>(&c);
            }
        }

        if (gi == 0) {
            // first token of this quad: start 1.5 octaves (192 key16 units)
            // below its largest key instead of at a fixed guess
            __half2 mx = *reinterpret_cast<const __half2 *>(&kp[0]);
#pragma unroll
            for (int i = 1; i < 16; ++i) mx = __hmax2(mx, *reinterpret_cast<const __half2 *>(&kp[i]));
            const uint32_t mb = *reinterpret_cast<const uint32_t *>(&mx);
            uint32_t m16 = max(mb & 0xffffu, mb >> 16);
            m16 = max(m16, __shfl_xor_sync(0xffffffffu, m16, 1));
            m16 = max(m16, __shfl_xor_sync(0xffffffffu, m16, 2));
            tau16 = m16 > 192u ? m16 - 192u : 1u;
        }
        const uint32_t m = select_top_t(key, kp, T, s, tau16);
        if (valid) mask[((size_t)bh * S + t) * kMaskWords + s] = m;

        // pruned-saliency sums (fp32 over this lane's 32 channels, fp64 across
        // tokens) and the kept values, in ascending channel order, into the
        // staging tile
        Raw *vt = vtile[gi & 1];
        int pos = quad_excl_scan(__popc(m), s);
        float sw = 0.f, sw2 = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if ((m >> i) & 1u) {
                vt[pos * 32 + tl] = (Raw)ks.raw(i);
                ++pos;
            } else {
                const float w = __uint_as_float(key[i]);
                sw = __fadd_rn(sw, w);
                sw2 = __fmaf_rn(w, w, sw2);
            }
        }
        if (valid) {
            acc_w = __dadd_rn(acc_w, (double)sw);
            acc_w2 = __dadd_rn(acc_w2, (double)sw2);
        }
        __syncthreads();
        // 32 tokens x T values, contiguous in the interleaved layout
        const int nvec = (int)((size_t)32 * T * sizeof(E) / 16);
        uint4 *dst = reinterpret_cast<uint4 *>(vals + (size_t)bh * S32 * T + (size_t)t0 * T);
        const uint4 *src = reinterpret_cast<const uint4 *>(vt);
        for (int vi = tid; vi < nvec; vi += kPruneThreads) __stcs(dst + vi, src[vi]);
        ks = ks_next;
    }

    // fixed-order reduction: xor tree inside each warp, then warps in order
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        acc_w = __dadd_rn(acc_w, __shfl_xor_sync(0xffffffffu, acc_w, o));
        acc_w2 = __dadd_rn(acc_w2, __shfl_xor_sync(0xffffffffu, acc_w2, o));
    }
    if (lane == 0) {
        red[0][warp] = acc_w;
        red[1][warp] = acc_w2;
    }
    __syncthreads();
    if (tid == 0) {
        double a = 0.0, b = 0.0;
        for (int i = 0; i < kPruneThreads / 32; ++i) {
            a = __dadd_rn(a, red[0][i]);
            b = __dadd_rn(b, red[1][i]);
        }
        partial[((size_t)bh * n_chunks + chunk) * 2 + 0] = a;
        partial[((size_t)bh * n_chunks + chunk) * 2 + 1] = b;
    }
}

// One warp per (row, kv head): lanes sum the chunk partials in a fixed order,
// then a fixed xor tree.
__global__ void stats_kernel(const double *__restrict__ partial, int n_chunks, long BH, int S, int T,
                             double *__restrict__ stats) {
    const long bh = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (bh >= BH) return;
    double a = 0.0, b = 0.0;
    for (int c = lane; c < n_chunks; c += 32) {
        a = __dadd_rn(a, partial[((size_t)bh * n_chunks + c) * 2 + 0]);
        b = __dadd_rn(b, partial[((size_t)bh * n_chunks + c) * 2 + 1]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a = __dadd_rn(a, __shfl_xor_sync(0xffffffffu, a, o));
        b = __dadd_rn(b, __shfl_xor_sync(0xffffffffu, b, o));
    }
    if (lane == 0) {
        const double n = (double)S * (double)(kD - T);
        stats[bh * 4 + 0] = n;
        stats[bh * 4 + 1] = a;
        stats[bh * 4 + 2] = b;
        stats[bh * 4 + 3] = n > 0.0 ? a / n : 0.0;
    }
}

template <typename E>
static cudaError_t launch_prune_t(const void *k, const void *q_obs, int G, int W,
                                  const spark_kcache &kc, void *ws, cudaStream_t st) {
    const long BH = (long)kc.B * kc.Hkv;
    if (BH == 0) return cudaSuccess;
    double *partial = reinterpret_cast<double *>(static_cast<char *>(ws) + kWsHeader);
    qnorm_kernel<E><<<(unsigned)BH, kD, 0, st>>>(static_cast<const E *>(q_obs), G, W, kc.qn);
    const int nch = prune_chunks(kc.S);
    if (nch > 0) {
        prune_kernel<E><<<(unsigned)(BH * nch), kPruneThreads, 0, st>>>(
            static_cast<const E *>(k), kc.qn, kc.mask, static_cast<E *>(kc.vals), partial, kc.S, kc.T,
            nch);
    }
    stats_kernel<<<(unsigned)((BH + 3) / 4), 128, 0, st>>>(partial, nch, BH, kc.S, kc.T, kc.stats);
    return cudaGetLastError();
}

cudaError_t launch_prune(const void *k, const void *q_obs, int G, int W, const spark_kcache &kc,
                         void *ws, cudaStream_t st) {
    if (kc.dtype == SPARK_BF16) return launch_prune_t<__nv_bfloat16>(k, q_obs, G, W, kc, ws, st);
    return launch_prune_t<float>(k, q_obs, G, W, kc, ws, st);
}

// ---------------------------------------------------------------------------
// Allocation-free variant of spark_prune (spark_prune_noalloc).
//
// The per-CTA statistics partials normally live in a workspace the caller
// allocates.  Callers that cannot allocate device memory on the pruning path
// get a fixed, file-scope device array instead.  It holds the same layout as
// the workspace (status header + partials), is created when a device loads
// this library, and stays until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB on every device
static __device__ __align__(256) unsigned char g_prune_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
static void *g_prune_scratch_addr[kMaxDevices];  // device address per device id

// Device address of the scratch array on `dev` (the current device).  Host
// code cannot use the symbol itself: in host code it names a host-side
// stand-in.  Looked up once per device; racing first calls store the same
// value.
static void *prune_scratch(int dev) {
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    void *p = __atomic_load_n(&g_prune_scratch_addr[dev], __ATOMIC_ACQUIRE);
    if (p) return p;
    if (cudaGetSymbolAddress(&p, g_prune_scratch) != cudaSuccess || !p) return nullptr;
    __atomic_store_n(&g_prune_scratch_addr[dev], p, __ATOMIC_RELEASE);
    return p;
}

}  // namespace spark

extern "C" SPARK_API int spark_prune_noalloc(const void *k, const void *q_obs, int G, int W,
                                             const spark_kcache *out, void *stream) {
    using namespace spark;
    if (!out) return SPARK_ERR_ARG;
    if (out->B < 0 || out->Hkv < 0 || out->S < 0) return SPARK_ERR_ARG;
    if (out->dtype != SPARK_F32 && out->dtype != SPARK_BF16) return SPARK_ERR_ARG;
    if (out->D != kD) return SPARK_ERR_UNSUPPORTED;
    if (out->T < 0 || out->T > out->D || G < 1 || W < 1) return SPARK_ERR_ARG;
    const long BH = (long)out->B * out->Hkv;
    if (BH == 0) return SPARK_OK;
    auto a16 = [](const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!a16(q_obs) || !a16(out->qn) || !a16(out->stats)) return SPARK_ERR_ARG;
    if (out->S > 0 && (!a16(k) || !a16(out->mask))) return SPARK_ERR_ARG;
    if (out->S > 0 && out->T > 0 && !a16(out->vals)) return SPARK_ERR_ARG;
    if (prune_workspace(BH, out->S) > kNoAllocScratchBytes) return SPARK_ERR_WORKSPACE;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return SPARK_ERR_CUDA;
    void *ws = prune_scratch(dev);
    if (!ws) return SPARK_ERR_CUDA;
    cudaError_t e = launch_prune(k, q_obs, G, W, *out, ws, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SPARK_OK : SPARK_ERR_CUDA;
}

namespace spark {

}  // namespace spark
