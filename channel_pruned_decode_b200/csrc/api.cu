// C ABI entry points of the SparK sm_100a library: argument validation,
// cache layout arithmetic, workspace sizing, the tail-append kernel and the
// device status word.  The compute kernels live in prune.cu and decode.cu.
#include "spark_internal.cuh"

#include <math.h>

namespace spark {
cudaError_t launch_prune(const void *k, const void *q_obs, int G, int W, const spark_kcache &kc,
                         void *ws, cudaStream_t st);
cudaError_t launch_prune_grouped(const void *k, const void *q_obs, int G, int W, int n_groups,
                                 const int *group_T, const spark_kcache &kc, void *ws, cudaStream_t st);
cudaError_t launch_decode(const void *q, const spark_kcache &kc, const void *v, const spark_kcache *vc,
                          const void *k_tail, const void *v_tail, int tail_cap, int n_tail, int G, int recovery,
                          unsigned long long seed, float *out, void *ws, const DecodeGeom &geo, cudaStream_t st,
                          bool topp = false);
cudaError_t launch_prune_values(const void *v, const spark_kcache &vc, void *ws, cudaStream_t st);
cudaError_t launch_prune_topp(const void *k, const void *q_obs, int G, int W, float p, const spark_kcache &kc,
                              void *ws, cudaStream_t st);
cudaError_t launch_think(const void *k, const void *q_obs, int G, int W, const spark_kcache &kc, void *ws,
                         cudaStream_t st);
size_t think_workspace(long BH, int S);
cudaError_t launch_snapkv(const void *k, const void *v, const void *q_obs, long BH, int S, int G, int W, int keep,
                          int pool, void *k_out, void *v_out, int *idx_out, void *ws, cudaStream_t st,
                          const int32_t *keep_rows = nullptr, int Hkv = 1, int keep_cap = 0);

size_t snapkv_partials_bytes(long BH);

// scores (fp32) and pooled keys (u32) per prefix token, then the per-split
// softmax partials
static size_t snapkv_workspace(long BH, int S, int W) {
    return kWsHeader + (size_t)BH * (size_t)(S - W) * 8 + snapkv_partials_bytes(BH);
}


static size_t round256(size_t x) { return (x + 255) / 256 * 256; }

static int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}

// Self-test of the bounded-wait path: one warp waits on an mbarrier that
// nothing ever arrives on, gives up after limit_ns, and records the timeout in
// the status word exactly as the decode pipeline does.
__global__ void wait_selftest_kernel(uint32_t *status, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    const bool ok = mbar_wait_limit(smem_u32(&bar), 0u, limit_ns);
    if (__all_sync(0xffffffffu, !ok) && threadIdx.x == 0) atomicOr(status, kDevTimeout);
}

__global__ void tail_append_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                                   uint4 *__restrict__ k_tail, uint4 *__restrict__ v_tail,
                                   int row_vec, int tail_cap, int slot) {
    const long bh = blockIdx.x;
    const int i = threadIdx.x;
    if (i < row_vec) {
        const size_t dst = ((size_t)bh * tail_cap + slot) * row_vec + i;
        k_tail[dst] = k_new[(size_t)bh * row_vec + i];
        v_tail[dst] = v_new[(size_t)bh * row_vec + i];
    }
}

}  // namespace spark

using namespace spark;

extern "C" {

int spark_lambda_to_T(float lambda, int D) {
    if (!(lambda >= 0.0f && lambda <= 1.0f) || D <= 0) return -1;
    return (int)llround((1.0 - (double)lambda) * (double)D);
}

size_t spark_cache_sizes(int B, int Hkv, int S, int D, int T, int dtype, size_t sizes[4]) {
    const int es = elem_size(dtype);
    if (B < 0 || Hkv < 0 || S < 0 || D != kD || T < 0 || T > D || es == 0) return 0;
    const size_t BH = (size_t)B * Hkv;
    const size_t S32 = ((size_t)S + 31) / 32 * 32;
    size_t sz[4];
    sz[0] = BH * S * kMaskWords * sizeof(uint32_t);
    sz[1] = BH * S32 * T * es;
    sz[2] = BH * D * sizeof(float);
    sz[3] = BH * 4 * sizeof(double);
    size_t total = 0;
    for (int i = 0; i < 4; ++i) {
        if (sizes) sizes[i] = sz[i];
        total += round256(sz[i]);
    }
    return total;
}

size_t spark_cache_bytes(int B, int Hkv, int S, int D, int T, int dtype) {
    return spark_cache_sizes(B, Hkv, S, D, T, dtype, nullptr);
}

size_t spark_workspace_bytes(int op, int B, int Hkv, int G, int S, int D, int T, int n_tail) {
    if (B < 0 || Hkv < 0 || S < 0 || D != kD || T < 0 || T > D || G < 1 || n_tail < 0) return 0;
    const long BH = (long)B * Hkv;
    if (op == SPARK_OP_PRUNE) return round256(prune_grouped_workspace(BH, S));  // also spark_prune_grouped
    if (op == SPARK_OP_SNAPKV) return round256(snapkv_workspace(BH, S, 0));
    if (op == SPARK_OP_THINK) return round256(think_workspace(BH, S));
    if (op == SPARK_OP_TOPP) return round256(topp_workspace(BH, S));
    if (op == SPARK_OP_DECODE) {
        if (G != 1 && G != 2 && G != 4 && G != 8) return 0;
        // the geometry depends on the element size only through the stage
        // size; take the larger of the two so one workspace serves both
        const DecodeGeom g2 = decode_geometry(BH, S, T, -1, 2, G, num_sms());
        const DecodeGeom g4 = decode_geometry(BH, S, T, -1, 4, G, num_sms());
        const size_t a = decode_workspace(BH, g2, G), b = decode_workspace(BH, g4, G);
        return round256(a > b ? a : b);
    }
    return 0;
}

int spark_prune(const void *k, const void *q_obs, int G, int W, const spark_kcache *out,
                void *workspace, size_t ws_bytes, void *stream) {
    const int rc = check_prune_args(k, q_obs, G, W, out);
    if (rc != SPARK_OK) return rc;
    const long BH = (long)out->B * out->Hkv;
    if (BH == 0) return SPARK_OK;
    if (!workspace || !aligned16(workspace)) return SPARK_ERR_WORKSPACE;
    if (ws_bytes < prune_workspace(BH, out->S)) return SPARK_ERR_WORKSPACE;
    cudaError_t e = launch_prune(k, q_obs, G, W, *out, workspace, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SPARK_OK : SPARK_ERR_CUDA;
}

int spark_group_budget(int D, int g, const float *rates, int *Tg) {
    if (!rates || !Tg || D <= 0 || g < 1 || g > kMaxGroups || g > D) return SPARK_ERR_ARG;
    for (int q = 0; q < g; ++q)
        if (!(rates[q] >= 0.0f && rates[q] <= 1.0f)) return SPARK_ERR_ARG;
    for (int q = 0; q < g; ++q) {
        const int size = (q + 1) * D / g - q * D / g;
        Tg[q] = (int)llround((1.0 - (double)rates[q]) * (double)size);
    }
    return SPARK_OK;
}

int spark_prune_grouped(const void *k, const void *q_obs, int G, int W, int n_groups, const int *group_T,
                        const spark_kcache *out, void *workspace, size_t ws_bytes, void *stream) {
    int rc = check_cache(out);
    if (rc != SPARK_OK) return rc;
    if (G < 1 || W < 1) return SPARK_ERR_ARG;
    if (n_groups < 1 || n_groups > kMaxGroups || !group_T) return SPARK_ERR_ARG;
    int sum = 0;
    for (int q = 0; q < n_groups; ++q) {
        const int size = (q + 1) * out->D / n_groups - q * out->D / n_groups;
        if (group_T[q] < 0 || group_T[q] > size) return SPARK_ERR_ARG;
        sum += group_T[q];
    }
    if (sum != out->T) return SPARK_ERR_ARG;
    const long BH = (long)out->B * out->Hkv;
    if (BH == 0) return SPARK_OK;
    if (!q_obs || !aligned16(q_obs)) return SPARK_ERR_ARG;
    if (out->S > 0 && (!k || !aligned16(k))) return SPARK_ERR_ARG;
    if (!workspace || !aligned16(workspace)) return SPARK_ERR_WORKSPACE;
    if (ws_bytes < prune_grouped_workspace(BH, out->S)) return SPARK_ERR_WORKSPACE;
    cudaError_t e = launch_prune_grouped(k, q_obs, G, W, n_groups, group_T, *out, workspace,
                                         static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SPARK_OK : SPARK_ERR_CUDA;
}

int spark_prune_topp(const void *k, const void *q_obs, int G, int W, float p, const spark_kcache *out,
                     void *workspace, size_t ws_bytes, void *stream) {
    int rc = check_cache(out);
    if (rc != SPARK_OK) return rc;
    if (out->lens) return SPARK_ERR_UNSUPPORTED;
    if (G < 1 || W < 1) return SPARK_ERR_ARG;
    if (!(p >= 0.0f && p <= 1.0f)) return SPARK_ERR_ARG;
    const long BH = (long)out->B * out->Hkv;
    if (BH == 0) return SPARK_OK;
    if (!out->goff || (reinterpret_cast<uintptr_t>(out->goff) & 3u)) return SPARK_ERR_ARG;
    // value rows are counted in 32 bits
    if ((double)BH * (double)((out->S + 31) / 32) * (double)out->T >= 4294967295.0) return SPARK_ERR_UNSUPPORTED;
    if (!q_obs || !aligned16(q_obs)) return SPARK_ERR_ARG;
    if (out->S > 0 && (!k || !aligned16(k))) return SPARK_ERR_ARG;
    if (!workspace || !aligned16(workspace)) return SPARK_ERR_WORKSPACE;
    if (ws_bytes < topp_workspace(BH, out->S)) return SPARK_ERR_WORKSPACE;
    cudaError_t e = launch_prune_topp(k, q_obs, G, W, p, *out, workspace, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SPARK_OK : SPARK_ERR_CUDA;
}

size_t spark_topp_offsets_bytes(int B, int Hkv, int S) {
    if (B < 0 || Hkv < 0 || S < 0) return 0;
    return ((size_t)B * Hkv * (((size_t)S + 31) / 32) + 1) * sizeof(uint32_t);
}

int spark_topp_vals_used(const spark_kcache *kc, size_t *bytes, void *stream) {
    if (!kc || !bytes || !kc->goff || kc->B < 0 || kc->Hkv < 0 || kc->S < 0) return SPARK_ERR_ARG;
    const int es = elem_size(kc->dtype);
    if (es == 0) return SPARK_ERR_ARG;
    const size_t n = (size_t)kc->B * kc->Hkv * (((size_t)kc->S + 31) / 32);
    uint32_t rows = 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&rows, kc->goff + n, sizeof(uint32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return SPARK_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SPARK_ERR_CUDA;
    *bytes = (size_t)rows * 32 * (size_t)es;
    return SPARK_OK;
}

// argument checks and launch shared by spark_decode_attn and
// spark_decode_attn_topp; `f` is the kernel's recovery selector
static int decode_entry(const void *q, const spark_kcache *kc, const void *v, const void *k_tail,
                        const void *v_tail, int tail_cap, int n_tail, int G, int recovery, int f,
                        unsigned long long seed, float *out, void *workspace, size_t ws_bytes, void *stream,
                        bool topp = false) {
    int rc = check_cache(kc);
    if (rc != SPARK_OK) return rc;
    if (topp && (!kc->goff || (reinterpret_cast<uintptr_t>(kc->goff) & 3u))) return SPARK_ERR_ARG;
    if (topp && kc->lens) return SPARK_ERR_UNSUPPORTED;
    if (G != 1 && G != 2 && G != 4 && G != 8) return G < 1 ? SPARK_ERR_ARG : SPARK_ERR_UNSUPPORTED;
    if (recovery != SPARK_F_DEGENERATE && recovery != SPARK_F_GAUSSIAN && recovery != SPARK_F_EXPONENTIAL)
        return SPARK_ERR_ARG;
    if (tail_cap < 0 || n_tail < 0 || n_tail > tail_cap) return SPARK_ERR_ARG;
    const long BH = (long)kc->B * kc->Hkv;
    if (BH == 0) return SPARK_OK;
    if (!q || !aligned16(q) || !out || !aligned16(out)) return SPARK_ERR_ARG;
    if (kc->S > 0 && (!v || !aligned16(v))) return SPARK_ERR_ARG;
    if (tail_cap > 0 && (!k_tail || !v_tail || !aligned16(k_tail) || !aligned16(v_tail)))
        return SPARK_ERR_ARG;
    if (!workspace || !aligned16(workspace)) return SPARK_ERR_WORKSPACE;
    const int es = elem_size(kc->dtype);
    const DecodeGeom geo = decode_geometry(BH, kc->S, kc->T, -1, es, G, num_sms());
    if (BH * (long)geo.units >= (1L << 31)) return SPARK_ERR_UNSUPPORTED;  // 32-bit item indices
    if (ws_bytes < decode_workspace(BH, geo, G)) return SPARK_ERR_WORKSPACE;
    cudaError_t e = launch_decode(q, *kc, v, nullptr, k_tail, v_tail, tail_cap, n_tail, G, f, seed, out,
                                  workspace, geo, static_cast<cudaStream_t>(stream), topp);
    return e == cudaSuccess ? SPARK_OK : SPARK_ERR_CUDA;
}

int spark_decode_attn(const void *q, const spark_kcache *kc, const void *v, const void *k_tail,
                      const void *v_tail, int tail_cap, int n_tail, int G, int recovery,
                      unsigned long long seed, float *out, void *workspace, size_t ws_bytes,
                      void *stream) {
    return decode_entry(q, kc, v, k_tail, v_tail, tail_cap, n_tail, G, recovery, recovery, seed, out, workspace,
                        ws_bytes, stream);
}

int spark_decode_attn_topp(const void *q, const spark_kcache *kc, const void *v, const void *k_tail,
                           const void *v_tail, int tail_cap, int n_tail, int G, int recovery,
                           unsigned long long seed, float *out, void *workspace, size_t ws_bytes,
                           void *stream) {
    // Gaussian / Exponential F walk all channels and read the kept values in
    // order, which already handles fewer kept channels than slots
    const int f = recovery == SPARK_F_DEGENERATE ? kRecoveryDegVar : recovery;
    return decode_entry(q, kc, v, k_tail, v_tail, tail_cap, n_tail, G, recovery, f, seed, out, workspace,
                        ws_bytes, stream, true);
}

size_t spark_workspace_bytes_kv(int B, int Hkv, int G, int S, int D, int T, int Tv, int n_tail) {
    if (B < 0 || Hkv < 0 || S < 0 || D != kD || T < 0 || T > D || Tv < 0 || Tv > D || n_tail < 0) return 0;
    if (G != 1 && G != 2 && G != 4 && G != 8) return 0;
    const DecodeGeom g = decode_geometry((long)B * Hkv, S, T, Tv, 2, G, num_sms());
    return round256(decode_workspace((long)B * Hkv, g, G));
}

int spark_prune_think(const void *k, const void *q_obs, int G, int W, const spark_kcache *out, void *workspace,
                      size_t ws_bytes, void *stream) {
    int rc = check_cache(out);
    if (rc != SPARK_OK) return rc;
    if (out->lens) return SPARK_ERR_UNSUPPORTED;
    if (G < 1 || W < 1) return SPARK_ERR_ARG;
    const long BH = (long)out->B * out->Hkv;
    if (BH == 0) return SPARK_OK;
    if (!q_obs || !aligned16(q_obs)) return SPARK_ERR_ARG;
    if (out->S > 0 && (!k || !aligned16(k))) return SPARK_ERR_ARG;
    if (!workspace || !aligned16(workspace)) return SPARK_ERR_WORKSPACE;
    if (ws_bytes < think_workspace(BH, out->S)) return SPARK_ERR_WORKSPACE;
    cudaError_t e = launch_think(k, q_obs, G, W, *out, workspace, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SPARK_OK : SPARK_ERR_CUDA;
}

int spark_prune_values(const void *v, const spark_kcache *out, void *workspace, size_t ws_bytes, void *stream) {
    int rc = check_cache(out);
    if (rc != SPARK_OK) return rc;
    const long BH = (long)out->B * out->Hkv;
    if (BH == 0) return SPARK_OK;
    if (out->S > 0 && (!v || !aligned16(v))) return SPARK_ERR_ARG;
    if (!workspace || !aligned16(workspace)) return SPARK_ERR_WORKSPACE;
    if (ws_bytes < prune_workspace(BH, out->S)) return SPARK_ERR_WORKSPACE;
    cudaError_t e = launch_prune_values(v, *out, workspace, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SPARK_OK : SPARK_ERR_CUDA;
}

int spark_decode_attn_kv(const void *q, const spark_kcache *kc, const spark_kcache *vc, const void *k_tail,
                         const void *v_tail, int tail_cap, int n_tail, int G, float *out, void *workspace,
                         size_t ws_bytes, void *stream) {
    int rc = check_cache(kc);
    if (rc != SPARK_OK) return rc;
    rc = check_cache(vc);
    if (rc != SPARK_OK) return rc;
    if (kc->B != vc->B || kc->Hkv != vc->Hkv || kc->S != vc->S || kc->dtype != vc->dtype) return SPARK_ERR_ARG;
    if (kc->dtype != SPARK_BF16) return SPARK_ERR_UNSUPPORTED;
    if (G != 1 && G != 2 && G != 4 && G != 8) return G < 1 ? SPARK_ERR_ARG : SPARK_ERR_UNSUPPORTED;
    if (tail_cap < 0 || n_tail < 0 || n_tail > tail_cap) return SPARK_ERR_ARG;
    const long BH = (long)kc->B * kc->Hkv;
    if (BH == 0) return SPARK_OK;
    if (!q || !aligned16(q) || !out || !aligned16(out)) return SPARK_ERR_ARG;
    if (tail_cap > 0 && (!k_tail || !v_tail || !aligned16(k_tail) || !aligned16(v_tail)))
        return SPARK_ERR_ARG;
    if (!workspace || !aligned16(workspace)) return SPARK_ERR_WORKSPACE;
    const DecodeGeom geo = decode_geometry(BH, kc->S, kc->T, vc->T, 2, G, num_sms());
    if (BH * (long)geo.units >= (1L << 31)) return SPARK_ERR_UNSUPPORTED;
    if (ws_bytes < decode_workspace(BH, geo, G)) return SPARK_ERR_WORKSPACE;
    cudaError_t e = launch_decode(q, *kc, nullptr, vc, k_tail, v_tail, tail_cap, n_tail, G, SPARK_F_DEGENERATE, 0,
                                  out, workspace, geo, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SPARK_OK : SPARK_ERR_CUDA;
}

int spark_snapkv_evict(const void *k, const void *v, const void *q_obs, int B, int Hkv, int S, int D, int G,
                       int W, int keep, int pool, int dtype, void *k_out, void *v_out, int32_t *idx_out,
                       void *workspace, size_t ws_bytes, void *stream) {
    if (B < 0 || Hkv < 0 || S < 0 || G < 1 || W < 1 || elem_size(dtype) == 0) return SPARK_ERR_ARG;
    if (D != kD || dtype != SPARK_BF16) return SPARK_ERR_UNSUPPORTED;
    if ((G * W) % 16 != 0 || G * W > 128) return SPARK_ERR_UNSUPPORTED;
    if (keep < W || keep > S || pool < 1 || (pool & 1) == 0) return SPARK_ERR_ARG;
    const long BH = (long)B * Hkv;
    if (BH == 0) return SPARK_OK;
    if (!k || !v || !q_obs || !k_out || !v_out || !idx_out) return SPARK_ERR_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(q_obs) || !aligned16(k_out) || !aligned16(v_out) ||
        !aligned16(idx_out))
        return SPARK_ERR_ARG;
    if (!workspace || !aligned16(workspace)) return SPARK_ERR_WORKSPACE;
    if (ws_bytes < snapkv_workspace(BH, S, W)) return SPARK_ERR_WORKSPACE;
    cudaError_t e = launch_snapkv(k, v, q_obs, BH, S, G, W, keep, pool, k_out, v_out, idx_out, workspace,
                                  static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SPARK_OK : SPARK_ERR_CUDA;
}

int spark_snapkv_evict_rows(const void *k, const void *v, const void *q_obs, int B, int Hkv, int S, int D, int G,
                            int W, const int32_t *keep_rows, int keep_cap, int pool, int dtype, void *k_out,
                            void *v_out, int32_t *idx_out, void *workspace, size_t ws_bytes, void *stream) {
    if (B < 0 || Hkv < 0 || S < 0 || G < 1 || W < 1 || elem_size(dtype) == 0) return SPARK_ERR_ARG;
    if (D != kD || dtype != SPARK_BF16) return SPARK_ERR_UNSUPPORTED;
    if ((G * W) % 16 != 0 || G * W > 128) return SPARK_ERR_UNSUPPORTED;
    if (keep_cap < W || W > S || pool < 1 || (pool & 1) == 0) return SPARK_ERR_ARG;
    const long BH = (long)B * Hkv;
    if (BH == 0) return SPARK_OK;
    if (!keep_rows || (reinterpret_cast<uintptr_t>(keep_rows) & 3u)) return SPARK_ERR_ARG;
    if (!k || !v || !q_obs || !k_out || !v_out || !idx_out) return SPARK_ERR_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(q_obs) || !aligned16(k_out) || !aligned16(v_out) ||
        !aligned16(idx_out))
        return SPARK_ERR_ARG;
    if (!workspace || !aligned16(workspace)) return SPARK_ERR_WORKSPACE;
    if (ws_bytes < snapkv_workspace(BH, S, W)) return SPARK_ERR_WORKSPACE;
    cudaError_t e = launch_snapkv(k, v, q_obs, BH, S, G, W, W, pool, k_out, v_out, idx_out, workspace,
                                  static_cast<cudaStream_t>(stream), keep_rows, Hkv, keep_cap);
    return e == cudaSuccess ? SPARK_OK : SPARK_ERR_CUDA;
}

int spark_pyramid_keep(int L, int M, float beta, int W, int S, int *keep) {
    if (L < 1 || W < 1 || M < W || S < M || !(beta >= 0.0f && beta < 1.0f) || !keep) return SPARK_ERR_ARG;
    for (int l = 0; l < L; ++l) {
        const double f = L > 1 ? (double)(L - 1 - 2 * l) / (double)(L - 1) : 0.0;
        long x = llround((double)M * (1.0 + (double)beta * f));
        x = x < W ? W : (x > S ? S : x);
        keep[l] = (int)x;
    }
    return SPARK_OK;
}

int spark_tail_append(const void *k_new, const void *v_new, void *k_tail, void *v_tail, int B, int Hkv,
                      int D, int tail_cap, int slot, int dtype, void *stream) {
    const int es = elem_size(dtype);
    if (es == 0 || B < 0 || Hkv < 0) return SPARK_ERR_ARG;
    if (D != kD) return SPARK_ERR_UNSUPPORTED;
    if (tail_cap < 1 || slot < 0 || slot >= tail_cap) return SPARK_ERR_ARG;
    const long BH = (long)B * Hkv;
    if (BH == 0) return SPARK_OK;
    if (!k_new || !v_new || !k_tail || !v_tail) return SPARK_ERR_ARG;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_tail) || !aligned16(v_tail))
        return SPARK_ERR_ARG;
    const int row_vec = D * es / 16;
    tail_append_kernel<<<(unsigned)BH, 32 * ((row_vec + 31) / 32), 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), static_cast<uint4 *>(k_tail),
        static_cast<uint4 *>(v_tail), row_vec, tail_cap, slot);
    return cudaGetLastError() == cudaSuccess ? SPARK_OK : SPARK_ERR_CUDA;
}

int spark_selftest_wait_timeout(void *workspace, int limit_us, void *stream) {
    if (!workspace || !aligned16(workspace)) return SPARK_ERR_WORKSPACE;
    if (limit_us < 1 || limit_us > 1000000) return SPARK_ERR_ARG;
    wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t *>(workspace),
                                                                          1000ull * (unsigned long long)limit_us);
    return cudaGetLastError() == cudaSuccess ? SPARK_OK : SPARK_ERR_CUDA;
}

int spark_device_status(void *workspace, int *status, int clear, void *stream) {
    if (!workspace || !status) return SPARK_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return SPARK_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SPARK_ERR_CUDA;
    *status = (word & kDevTimeout) ? SPARK_ERR_TIMEOUT : ((word & kDevBadArg) ? SPARK_ERR_ARG : SPARK_OK);
    if (clear && word) {
        if (cudaMemsetAsync(workspace, 0, sizeof(word), st) != cudaSuccess) return SPARK_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return SPARK_ERR_CUDA;
    }
    return SPARK_OK;
}

const char *spark_status_str(int status) {
    switch (status) {
    case SPARK_OK: return "ok";
    case SPARK_ERR_ARG: return "invalid argument";
    case SPARK_ERR_UNSUPPORTED: return "unsupported configuration";
    case SPARK_ERR_CUDA: return "CUDA error";
    case SPARK_ERR_TIMEOUT: return "device-side wait timed out";
    case SPARK_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    default: return "unknown status";
    }
}

}  // extern "C"
