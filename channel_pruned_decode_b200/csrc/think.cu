// ThinK, the structured channel-pruning comparator that the SparK pages set
// SparK against ("KV Cache 还能再砍一刀：SparK ..." section 1 and Fig. 2(c):
// one channel mask shared by all tokens of a head, no recovery; section 4.2
// compares the two at lambda = 0.5 and 0.8).  The pages give no ThinK
// formula; the reading implemented (same as the oracle): the relaxed
// objective of section 3.1 with one mask for the whole key block of a
// (row, kv head) ranks channel j by
//     score_j = qn_j * ||k^j||_2,   ||k^j||_2^2 = sum over the S tokens of k^2
// (fp64), keeps the T channels of largest score (ties -> lower channel) for
// every token, and marks the cache as unrecovered (mu = 0, so a pruned entry
// reads as 0 in decode).
//
// Four launches: qnorm (shared with spark_prune), think_colsum_kernel (per
// 256-token chunk and channel, the fp64 sum of squares), think_select_kernel
// (per head: fixed-order sum of the chunk partials, score, rank-based top-T,
// the head's mask and statistics), think_pack_kernel (per 32-token group:
// the shared mask per token and the kept values in the interleaved layout,
// gathered from a padded shared-memory copy of the tile).
#include "spark_internal.cuh"

namespace spark {

cudaError_t launch_qnorm(const void *q_obs, int G, int W, long BH, int dtype, float *qn, cudaStream_t st);

constexpr int kThinkChunk = 256;    // tokens per colsum CTA
constexpr int kThinkThreads = 256;  // 16 rows x 16 threads (8 channels each) per pass

inline int think_chunks(int S) { return S > 0 ? (S + kThinkChunk - 1) / kThinkChunk : 0; }

size_t think_workspace(long BH, int S) {
    return kWsHeader + (size_t)BH * (size_t)think_chunks(S) * kD * sizeof(double) + (size_t)BH * 16;
}

template <typename E>
__global__ void __launch_bounds__(kThinkThreads) think_colsum_kernel(const E *__restrict__ k, int S, int n_chunks,
                                                                    double *__restrict__ partial) {
    __shared__ double red[16][kD];
    const long bh = blockIdx.x / n_chunks;
    const int chunk = blockIdx.x % n_chunks;
    const int tid = threadIdx.x, rg = tid >> 4, slot = tid & 15;  // row group, 8-channel slot
    double acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.0;
    const long t_begin = (long)chunk * kThinkChunk;
    const long t_end = min((long)S, t_begin + kThinkChunk);
    for (long t = t_begin + rg; t < t_end; t += 16) {
        const E *row = k + ((size_t)bh * S + t) * kD + 8 * slot;
        float x[8];
        if constexpr (sizeof(E) == 2) {
            const uint4 v = __ldcs(reinterpret_cast<const uint4 *>(row));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                x[2 * c] = __uint_as_float(w[c] << 16);
                x[2 * c + 1] = __uint_as_float(w[c] & 0xffff0000u);
            }
        } else {
            const float4 a = __ldcs(reinterpret_cast<const float4 *>(row));
            const float4 b = __ldcs(reinterpret_cast<const float4 *>(row) + 1);
            x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
            x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const double d = (double)x[c];
            acc[c] = __fma_rn(d, d, acc[c]);  // the square of an fp32 value is exact in fp64
        }
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) red[rg][8 * slot + c] = acc[c];
    __syncthreads();
    if (tid < kD) {
        double s = 0.0;
        for (int r = 0; r < 16; ++r) s = __dadd_rn(s, red[r][tid]);  // fixed order
        partial[((size_t)bh * n_chunks + chunk) * kD + tid] = s;
    }
}

// One CTA (128 threads, one per channel) per (row, kv head).
__global__ void __launch_bounds__(kD) think_select_kernel(const double *__restrict__ partial, int n_chunks,
                                                         const float *__restrict__ qn, int S, int T,
                                                         uint32_t *__restrict__ head_mask,
                                                         double *__restrict__ stats) {
    __shared__ double score[kD];
    const long bh = blockIdx.x;
    const int j = threadIdx.x;
    double ss = 0.0;
    for (int c = 0; c < n_chunks; ++c) ss = __dadd_rn(ss, partial[((size_t)bh * n_chunks + c) * kD + j]);
    const double sj = (double)qn[bh * kD + j] * sqrt(ss);
    score[j] = sj;
    __syncthreads();
    int rank = 0;
    for (int i = 0; i < kD; ++i) {
        const double si = score[i];
        rank += (si > sj || (si == sj && i < j)) ? 1 : 0;
    }
    const uint32_t word = __ballot_sync(0xffffffffu, rank < T);
    if ((j & 31) == 0) head_mask[bh * kMaskWords + (j >> 5)] = word;
    if (j == 0) {
        stats[bh * 4 + 0] = (double)S * (double)(kD - T);
        stats[bh * 4 + 1] = 0.0;
        stats[bh * 4 + 2] = 0.0;
        stats[bh * 4 + 3] = 0.0;  // no recovery: a pruned entry reads as 0
    }
}

// One CTA (128 threads) per 32-token group of a (row, kv head).
template <typename E>
__global__ void __launch_bounds__(kD) think_pack_kernel(const E *__restrict__ k, const uint32_t *__restrict__ head_mask,
                                                       int S, int T, int n_groups, uint32_t *__restrict__ mask,
                                                       E *__restrict__ vals) {
    // the tile's 32 key rows, row stride = row bytes + 4 so that a column
    // (fixed channel, 32 tokens) falls in 32 distinct banks
    constexpr int kRowWords = kD * (int)sizeof(E) / 4 + 1;
    __shared__ uint32_t tile[32 * kRowWords];
    __shared__ uint8_t idx[kD];
    const long bh = blockIdx.x / n_groups;
    const int grp = blockIdx.x % n_groups;
    const long t0 = (long)grp * 32;
    const int n = (int)min(32L, (long)S - t0);
    const int tid = threadIdx.x;
    const uint32_t mw = head_mask[bh * kMaskWords + (tid >> 5)];
    if ((mw >> (tid & 31)) & 1u) {
        int pos = __popc(mw & ((1u << (tid & 31)) - 1u));
        for (int w = 0; w < (tid >> 5); ++w) pos += __popc(head_mask[bh * kMaskWords + w]);
        idx[pos] = (uint8_t)tid;
    }
    constexpr int kVec = kD * (int)sizeof(E) / 16;  // 16-byte pieces per row
    for (int e = tid; e < 32 * kVec; e += kD) {
        const int r = e / kVec, c = e % kVec;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < n) v = __ldcs(reinterpret_cast<const uint4 *>(k + ((size_t)bh * S + t0 + r) * kD) + c);
        uint32_t *d = tile + r * kRowWords + 4 * c;
        d[0] = v.x; d[1] = v.y; d[2] = v.z; d[3] = v.w;
    }
    if (tid < n) {
        const uint4 m = make_uint4(head_mask[bh * kMaskWords + 0], head_mask[bh * kMaskWords + 1],
                                   head_mask[bh * kMaskWords + 2], head_mask[bh * kMaskWords + 3]);
        *reinterpret_cast<uint4 *>(mask + ((size_t)bh * S + t0 + tid) * kMaskWords) = m;
    }
    __syncthreads();
    const long S32 = ((long)S + 31) / 32 * 32;
    E *out = vals + (size_t)bh * S32 * T + (size_t)t0 * T;
    const E *tl = reinterpret_cast<const E *>(tile);
    for (int e = tid; e < 32 * T; e += kD) {
        const int i = e >> 5, t = e & 31;
        out[e] = tl[t * kRowWords * (4 / (int)sizeof(E)) + idx[i]];  // value i of token t at (i * 32 + t)
    }
}

template <typename E>
static cudaError_t launch_think_t(const void *k, const void *q_obs, int G, int W, const spark_kcache &kc, void *ws,
                                  cudaStream_t st) {
    const long BH = (long)kc.B * kc.Hkv;
    if (BH == 0) return cudaSuccess;
    cudaError_t e = launch_qnorm(q_obs, G, W, BH, kc.dtype, kc.qn, st);
    if (e != cudaSuccess) return e;
    const int nch = think_chunks(kc.S);
    double *partial = reinterpret_cast<double *>(static_cast<char *>(ws) + kWsHeader);
    uint32_t *hmask = reinterpret_cast<uint32_t *>(partial + (size_t)BH * nch * kD);
    if (nch > 0)
        think_colsum_kernel<E><<<(unsigned)(BH * nch), kThinkThreads, 0, st>>>(static_cast<const E *>(k), kc.S,
                                                                               nch, partial);
    think_select_kernel<<<(unsigned)BH, kD, 0, st>>>(partial, nch, kc.qn, kc.S, kc.T, hmask, kc.stats);
    const int ngr = (kc.S + 31) / 32;
    if (ngr > 0)
        think_pack_kernel<E><<<(unsigned)(BH * ngr), kD, 0, st>>>(static_cast<const E *>(k), hmask, kc.S, kc.T, ngr,
                                                                 kc.mask, static_cast<E *>(kc.vals));
    return cudaGetLastError();
}

cudaError_t launch_think(const void *k, const void *q_obs, int G, int W, const spark_kcache &kc, void *ws,
                         cudaStream_t st) {
    if (kc.dtype == SPARK_BF16) return launch_think_t<__nv_bfloat16>(k, q_obs, G, W, kc, ws, st);
    return launch_think_t<float>(k, q_obs, G, W, kc, ws, st);
}

}  // namespace spark
