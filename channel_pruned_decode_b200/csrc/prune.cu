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

// Mask word (32 channels) of this lane's quarter of the token: the T largest
// keys over the quad, ties to the lower channel index.
__device__ __forceinline__ uint32_t select_top_t(const uint32_t (&key)[32], int T, int s) {
    if (T <= 0) return 0u;
    if (T >= kD) return 0xffffffffu;
    uint32_t kmax = 0u, kmin = 0xffffffffu;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        kmax = max(kmax, key[i]);
        kmin = min(kmin, key[i]);
    }
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, 1));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, 2));
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, 1));
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, 2));

    // invariant: count(key >= lo) >= T > count(key >= hi); keys are < 2^31
    uint32_t lo = kmin, hi = kmax + 1u;
    int c_hi = 0;
    bool exact = false;
    bool done = (hi - lo <= 1u);
    while (__any_sync(0xffffffffu, !done)) {  // warp-uniform trip count
        const uint32_t mid = lo + ((hi - lo) >> 1);
        int c = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) c += (key[i] >= mid) ? 1 : 0;
        c = quad_sum(c);
        if (!done) {
            if (c >= T) {
                lo = mid;
                if (c == T) { exact = true; done = true; }
            } else {
                hi = mid;
                c_hi = c;
            }
            if (hi - lo <= 1u) done = true;
        }
    }
    // exact: exactly T keys are >= lo.  Otherwise lo is the T-th largest key,
    // c_hi keys are above it, and T - c_hi of the keys equal to lo are kept in
    // channel order.
    const uint32_t thr = exact ? lo : lo + 1u;
    uint32_t m = 0u;
    int e = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        m |= (key[i] >= thr ? 1u : 0u) << i;
        e += (key[i] == lo) ? 1 : 0;
    }
    int r = quad_excl_scan(e, s);
    if (!exact) {
        const int need = T - c_hi;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (key[i] == lo) {
                if (r < need) m |= 1u << i;
                ++r;
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
    __shared__ double red[2][kPruneThreads];

    const long bh = blockIdx.x / n_chunks;
    const int chunk = blockIdx.x % n_chunks;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int s = lane & 3;                 // quarter: channels [32s, 32s+32)
    const int tl = warp * 8 + (lane >> 2);  // token within the 32-token group
    const long S32 = ((long)S + 31) / 32 * 32;

    float qv[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) qv[i] = __ldg(qn + bh * kD + 32 * s + i);

    double acc_w = 0.0, acc_w2 = 0.0;
    for (int gi = 0; gi < kPruneGroups; ++gi) {
        const long grp = (long)chunk * kPruneGroups + gi;
        const long t0 = grp * 32;
        if (t0 >= S) break;  // uniform across the CTA
        const long t = t0 + tl;
        const bool valid = t < S;

        KSlice<E> ks;
        if (valid)
            ks.load(k + ((size_t)bh * S + t) * kD + 32 * s);
        else
            ks.zero();

        uint32_t key[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
            key[i] = __float_as_uint(__fmul_rn(qv[i], __uint_as_float(ks.abs_bits(i))));

        const uint32_t m = select_top_t(key, T, s);
        if (valid) mask[((size_t)bh * S + t) * kMaskWords + s] = m;

        // pruned-saliency sums (fp32 over this lane's 32 channels, fp64 across tokens)
        float sw = 0.f, sw2 = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float w = __uint_as_float(key[i]);
            const bool pr = !((m >> i) & 1u);
            sw = __fadd_rn(sw, pr ? w : 0.f);
            sw2 = __fmaf_rn(pr ? w : 0.f, w, sw2);
        }
        if (valid) {
            acc_w = __dadd_rn(acc_w, (double)sw);
            acc_w2 = __dadd_rn(acc_w2, (double)sw2);
        }

        // pack kept values in ascending channel order into the staging tile
        Raw *vt = vtile[gi & 1];
        int pos = quad_excl_scan(__popc(m), s);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if ((m >> i) & 1u) {
                vt[pos * 32 + tl] = (Raw)ks.raw(i);
                ++pos;
            }
        }
        __syncthreads();
        // 32 tokens x T values, contiguous in the interleaved layout
        const int nvec = (int)((size_t)32 * T * sizeof(E) / 16);
        uint4 *dst = reinterpret_cast<uint4 *>(vals + (size_t)bh * S32 * T + (size_t)t0 * T);
        const uint4 *src = reinterpret_cast<const uint4 *>(vt);
        for (int vi = tid; vi < nvec; vi += kPruneThreads) __stcs(dst + vi, src[vi]);
    }

    red[0][tid] = acc_w;
    red[1][tid] = acc_w2;
    __syncthreads();
    if (tid == 0) {
        double a = 0.0, b = 0.0;
        for (int i = 0; i < kPruneThreads; ++i) {
            a = __dadd_rn(a, red[0][i]);
            b = __dadd_rn(b, red[1][i]);
        }
        partial[((size_t)bh * n_chunks + chunk) * 2 + 0] = a;
        partial[((size_t)bh * n_chunks + chunk) * 2 + 1] = b;
    }
}

__global__ void stats_kernel(const double *__restrict__ partial, int n_chunks, long BH, int S, int T,
                             double *__restrict__ stats) {
    const long bh = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (bh >= BH) return;
    double a = 0.0, b = 0.0;
    for (int c = 0; c < n_chunks; ++c) {
        a = __dadd_rn(a, partial[((size_t)bh * n_chunks + c) * 2 + 0]);
        b = __dadd_rn(b, partial[((size_t)bh * n_chunks + c) * 2 + 1]);
    }
    const double n = (double)S * (double)(kD - T);
    stats[bh * 4 + 0] = n;
    stats[bh * 4 + 1] = a;
    stats[bh * 4 + 2] = b;
    stats[bh * 4 + 3] = n > 0.0 ? a / n : 0.0;
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
    stats_kernel<<<(unsigned)((BH + 127) / 128), 128, 0, st>>>(partial, nch, BH, kc.S, kc.T, kc.stats);
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
