// SnapKV-style token eviction pre-pass, the base that SparK stacks on
// ("KV Cache 还能再砍一刀：SparK ..." sections 2 and 4.1: SnapKV / PyramidKV
// bases; 3.2: SparK reuses SnapKV's observation window).  The pages give no
// detail of SnapKV itself; the reading implemented (same as the oracle):
//   - the W window queries are the last W prompt positions p = S-W+w; each of
//     the G*W (query head, window row) rows attends causally over keys 0..p
//     with scale 1/sqrt(D); a prefix token's score (t < P = S-W) is the sum of
//     its probabilities over the G*W rows;
//   - scores are max-pooled along t (odd kernel, stride 1, in-range window);
//   - keep-W prefix tokens with the largest pooled score (ties -> lower t)
//     plus all W window tokens are kept, in original order.
//
// Kernels:
//   snap_scores_kernel  one CTA per (row, kv head): the G*W x S logits are a
//       dense contraction, computed on tensor cores (mma.sync m16n8k16 bf16 ->
//       fp32) from an XOR-swizzled shared-memory copy of the window queries
//       and a double-buffered stream of 64-key tiles (cp.async).  Pass 1 keeps
//       each row's running max and exp-sum (online softmax); pass 2 recomputes
//       the logits and sums the normalised probabilities over the rows, in
//       fp32, in a fixed order.
//   snap_select_kernel  one CTA per head: max-pool, exact radix select of the
//       (keep-W)-th largest pooled score on its fp32 bit pattern (scores are
//       >= 0), and an order-preserving compaction (ties to the lower index).
//   snap_gather_kernel  copies the kept K and V rows (16-byte vectors).
#include "spark_internal.cuh"

#include <algorithm>

namespace spark {

constexpr int kSnapKeys = 64;      // keys per tile
constexpr int kSnapStages = 4;     // key tiles in flight per CTA
constexpr int kSnapMaxSplit = 16;  // CTAs per (row, kv head)
constexpr int kSnapThreads = 256;  // 8 warps x 16 window rows = up to 128 rows
constexpr int kSnapMaxRows = 128;
constexpr int kSelThreads = 1024;

// byte offset of 16-byte chunk c of row r in a [rows][128 bf16] tile, XOR-
// swizzled so that ldmatrix over 8 consecutive rows is bank-conflict free
__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)(r * 256 + ((c ^ (r & 7)) << 4)); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    const int n = valid ? 16 : 0;  // zero-fill when the source row does not exist
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// log2(e) / sqrt(128)
constexpr float kSnapScale = 0.12751743074602467f;

// The keys of a (row, kv head) are split over `nsplit` CTAs.  Mode 0: each
// CTA keeps the running max and exp-sum of every window row over its keys and
// writes them as one partial; mode 1: each CTA merges the partials of its head
// (fixed order), recomputes its keys' logits and writes their summed
// normalised probabilities.  Key tiles stream through a kSnapStages-deep
// cp.async ring.
template <int kMode>
__global__ void __launch_bounds__(kSnapThreads, 2)
    snap_pass_kernel(const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ q_obs, int S, int G,
                     int W, int nsplit, float *__restrict__ ml, float *__restrict__ scores) {
    extern __shared__ __align__(128) unsigned char sm[];
    unsigned char *sq = sm;                               // [128 rows][256 B]
    unsigned char *sk = sm + kSnapMaxRows * 256;          // kSnapStages x [64 keys][256 B]
    float *colp = reinterpret_cast<float *>(sk + kSnapStages * kSnapKeys * 256);  // [8 warps][64]

    const long bh = blockIdx.x / nsplit;
    const int split = blockIdx.x % nsplit;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int R = G * W;                 // window rows (multiple of 16, <= 128)
    const int nwr = R / 16;              // warps with rows
    const long P = (long)S - W;
    const __nv_bfloat16 *kb = k + (size_t)bh * S * kD;
    const __nv_bfloat16 *qb = q_obs + (size_t)bh * R * kD;
    const int ntile = (S + kSnapKeys - 1) / kSnapKeys;
    const int per = (ntile + nsplit - 1) / nsplit;
    const int tile_lo = min(ntile, split * per), tile_hi = min(ntile, tile_lo + per);
    float *mlh = ml + (size_t)bh * nsplit * kSnapMaxRows * 2;  // [split][row][m, l]

    // window queries -> swizzled shared memory (rows past R are zero)
    for (int i = tid; i < kSnapMaxRows * 16; i += kSnapThreads) {
        const int r = i >> 4, c = i & 15;
        cp_async16(smem_u32(sq) + swz(r, c), qb + (size_t)min(r, R - 1) * kD + c * 8, r < R);
    }
    auto load_tile = [&](int tile) {
        unsigned char *dst = sk + (tile % kSnapStages) * kSnapKeys * 256;
        for (int i = tid; i < kSnapKeys * 16; i += kSnapThreads) {
            const int r = i >> 4, c = i & 15;
            const long t = (long)tile * kSnapKeys + r;
            cp_async16(smem_u32(dst) + swz(r, c), kb + (size_t)min(t, (long)S - 1) * kD + c * 8, t < S);
        }
    };

    // per thread: rows g0 = 16*warp + lane/4 and g1 = g0 + 8; columns 2*(lane%4)+{0,1}
    const int g0 = 16 * warp + (lane >> 2), g1 = g0 + 8;
    const long lim0 = P + (g0 % W), lim1 = P + (g1 % W);  // last key each row may see
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    if (kMode == 1 && warp < nwr) {
        // merge the head's partials in split order; split 0 holds key 0,
        // which every row sees, so the merged max is finite
        for (int sp = 0; sp < nsplit; ++sp) {
            const float ma = mlh[((size_t)sp * kSnapMaxRows + g0) * 2], la = mlh[((size_t)sp * kSnapMaxRows + g0) * 2 + 1];
            const float mb = mlh[((size_t)sp * kSnapMaxRows + g1) * 2], lb = mlh[((size_t)sp * kSnapMaxRows + g1) * 2 + 1];
            const float n0 = fmaxf(m0, ma), n1 = fmaxf(m1, mb);
            l0 = (m0 == -INFINITY ? 0.f : l0 * exp2f(m0 - n0)) + (ma == -INFINITY ? 0.f : la * exp2f(ma - n0));
            l1 = (m1 == -INFINITY ? 0.f : l1 * exp2f(m1 - n1)) + (mb == -INFINITY ? 0.f : lb * exp2f(mb - n1));
            m0 = n0;
            m1 = n1;
        }
    }

    // prologue: the first kSnapStages - 1 tiles (with the queries in group 0)
#pragma unroll
    for (int s0 = 0; s0 < kSnapStages - 1; ++s0) {
        if (tile_lo + s0 < tile_hi) load_tile(tile_lo + s0);
        cp_async_commit();
    }
    for (int tile = tile_lo; tile < tile_hi; ++tile) {
        if (tile + kSnapStages - 1 < tile_hi) load_tile(tile + kSnapStages - 1);
        cp_async_commit();
        cp_async_wait<kSnapStages - 1>();
        __syncthreads();
        if (warp < nwr) {
            const unsigned char *kt = sk + (tile % kSnapStages) * kSnapKeys * 256;
            float acc[8][4];
#pragma unroll
            for (int n = 0; n < 8; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                // this warp's 16 rows x 16 dims of the queries (A operand),
                // re-read per tile from the swizzled copy (keeps registers for
                // two CTAs per SM)
                uint32_t af[4];
                {
                    const int r = 16 * warp + (lane & 7) + ((lane >> 3) & 1) * 8;
                    const int c = 2 * ks + (lane >> 4);
                    ldsm_x4(smem_u32(sq) + swz(r, c), af[0], af[1], af[2], af[3]);
                }
#pragma unroll
                for (int n2 = 0; n2 < 4; ++n2) {  // two 8-key n-tiles per ldmatrix.x4
                    const int key = 16 * n2 + (lane & 7) + (lane >> 4) * 8;
                    const int c = 2 * ks + ((lane >> 3) & 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(smem_u32(kt) + swz(key, c), b0, b1, b2, b3);
                    mma_bf16(acc[2 * n2], af, b0, b1);
                    mma_bf16(acc[2 * n2 + 1], af, b2, b3);
                }
            }
            // logits (unscaled: the log2-domain scale is applied inside the
            // exponentials); keys past a row's causal limit become -inf.  A
            // tile whose keys all lie at or before P needs no mask.
            if ((long)(tile + 1) * kSnapKeys - 1 > P) {
                const long t_base = (long)tile * kSnapKeys + 2 * (lane & 3);
#pragma unroll
                for (int n = 0; n < 8; ++n)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const long t = t_base + 8 * n + (e & 1);
                        const long lim = (e < 2) ? lim0 : lim1;
                        acc[n][e] = (t <= lim && t < S) ? acc[n][e] : -INFINITY;
                    }
            }
            if (kMode == 0) {
                float x0 = -INFINITY, x1 = -INFINITY;
#pragma unroll
                for (int n = 0; n < 8; ++n) {
                    x0 = fmaxf(x0, fmaxf(acc[n][0], acc[n][1]));
                    x1 = fmaxf(x1, fmaxf(acc[n][2], acc[n][3]));
                }
                x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, 1));
                x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, 2));
                x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, 1));
                x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, 2));
                const float n0 = fmaxf(m0, x0 * kSnapScale), n1 = fmaxf(m1, x1 * kSnapScale);
                // a split may hold no key of a row yet: keep (m, l) = (-inf, 0)
                const float b0 = n0 == -INFINITY ? 0.f : n0, b1 = n1 == -INFINITY ? 0.f : n1;
                float s0 = 0.f, s1 = 0.f;
#pragma unroll
                for (int n = 0; n < 8; ++n) {
                    s0 += exp2f(fmaf(acc[n][0], kSnapScale, -b0)) + exp2f(fmaf(acc[n][1], kSnapScale, -b0));
                    s1 += exp2f(fmaf(acc[n][2], kSnapScale, -b1)) + exp2f(fmaf(acc[n][3], kSnapScale, -b1));
                }
                l0 = (m0 == -INFINITY ? 0.f : l0 * exp2f(m0 - n0)) + s0;
                l1 = (m1 == -INFINITY ? 0.f : l1 * exp2f(m1 - n1)) + s1;
                m0 = n0;
                m1 = n1;
            } else {
                // column sums of normalised probabilities over this warp's rows
                const float r0 = 1.f / l0, r1 = 1.f / l1;
                float cs[8][2];
#pragma unroll
                for (int n = 0; n < 8; ++n) {
                    cs[n][0] = exp2f(fmaf(acc[n][0], kSnapScale, -m0)) * r0 +
                               exp2f(fmaf(acc[n][2], kSnapScale, -m1)) * r1;
                    cs[n][1] = exp2f(fmaf(acc[n][1], kSnapScale, -m0)) * r0 +
                               exp2f(fmaf(acc[n][3], kSnapScale, -m1)) * r1;
                }
#pragma unroll
                for (int o = 4; o < 32; o <<= 1)
#pragma unroll
                    for (int n = 0; n < 8; ++n) {
                        cs[n][0] += __shfl_xor_sync(0xffffffffu, cs[n][0], o);
                        cs[n][1] += __shfl_xor_sync(0xffffffffu, cs[n][1], o);
                    }
                if (lane < 4) {
#pragma unroll
                    for (int n = 0; n < 8; ++n) {
                        colp[warp * kSnapKeys + 8 * n + 2 * lane] = cs[n][0];
                        colp[warp * kSnapKeys + 8 * n + 2 * lane + 1] = cs[n][1];
                    }
                }
            }
        }
        __syncthreads();
        if (kMode == 1 && tid < kSnapKeys) {
            const long t = (long)tile * kSnapKeys + tid;
            if (t < P) {
                float s = 0.f;
                for (int w = 0; w < nwr; ++w) s += colp[w * kSnapKeys + tid];
                scores[(size_t)bh * (P > 0 ? P : 0) + t] = s;
            }
        }
    }
    cp_async_wait<0>();
    if (kMode == 0 && warp < nwr) {
        // row exp-sums: fold the quad's column shares, then one partial per row
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
        if ((lane & 3) == 0) {
            mlh[((size_t)split * kSnapMaxRows + g0) * 2] = m0;
            mlh[((size_t)split * kSnapMaxRows + g0) * 2 + 1] = l0;
            mlh[((size_t)split * kSnapMaxRows + g1) * 2] = m1;
            mlh[((size_t)split * kSnapMaxRows + g1) * 2 + 1] = l1;
        }
    }
}

// exclusive block-wide prefix sum of one int per thread (kSelThreads threads)
__device__ __forceinline__ int block_excl_scan(int v, int *wsum, int &total) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int s = wsum[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        wsum[lane] = s;
    }
    __syncthreads();
    const int before = (warp > 0 ? wsum[warp - 1] : 0) + x - v;
    total = wsum[31];
    __syncthreads();
    return before;
}

__global__ void __launch_bounds__(kSelThreads)
    snap_select_kernel(const float *__restrict__ scores, uint32_t *__restrict__ pooled, int S, int W, int keep,
                       int pool, int *__restrict__ idx) {
    __shared__ int hist[256];
    __shared__ int wsum[32];
    __shared__ uint32_t sel[3];  // prefix, remaining rank, digit
    const long bh = blockIdx.x;
    const int tid = threadIdx.x;
    const long P = (long)S - W;
    const int kp = keep - W;
    const float *sc = scores + (size_t)bh * P;
    uint32_t *pk = pooled + (size_t)bh * P;
    int *out = idx + (size_t)bh * keep;
    const int h = pool / 2;

    // max-pool; scores are >= 0 so the fp32 bit pattern orders them
    for (long t = tid; t < P; t += kSelThreads) {
        float m = sc[t];
        for (long u = max(0L, t - h); u <= min(P - 1, t + h); ++u) m = fmaxf(m, sc[u]);
        pk[t] = __float_as_uint(m);
    }
    __syncthreads();

    // radix select of the kp-th largest key, 8 bits at a time from the top
    uint32_t prefix = 0u, pmask = 0u;
    int rem = kp;
    for (int shift = 24; shift >= 0 && kp > 0; shift -= 8) {
        for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
        __syncthreads();
        for (long t = tid; t < P; t += kSelThreads) {
            const uint32_t key = pk[t];
            if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
        }
        __syncthreads();
        if (tid == 0) {
            int above = 0;
            int d = 255;
            for (; d > 0; --d) {
                if (above + hist[d] >= rem) break;
                above += hist[d];
            }
            sel[0] = prefix | ((uint32_t)d << shift);
            sel[1] = (uint32_t)(rem - above);
        }
        __syncthreads();
        prefix = sel[0];
        rem = (int)sel[1];
        pmask |= 255u << shift;
        __syncthreads();
    }
    // keep: key > prefix, plus the first `rem` keys == prefix in index order
    int base = 0, eq_base = 0;
    for (long t0 = 0; t0 < P; t0 += kSelThreads) {
        const long t = t0 + tid;
        const uint32_t key = t < P ? pk[t] : 0u;
        const int eq = (kp > 0 && t < P && key == prefix) ? 1 : 0;
        int eq_total;
        const int eq_rank = eq_base + block_excl_scan(eq, wsum, eq_total);
        const int keepf = (kp > 0 && t < P && (key > prefix || (eq && eq_rank < rem))) ? 1 : 0;
        int k_total;
        const int pos = base + block_excl_scan(keepf, wsum, k_total);
        if (keepf) out[pos] = (int)t;
        base += k_total;
        eq_base += eq_total;
    }
    for (int w = tid; w < W; w += kSelThreads) out[kp + w] = (int)(P + w);
}

__global__ void snap_gather_kernel(const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                                   const int *__restrict__ idx, int S, int keep, int row_vec,
                                   uint4 *__restrict__ k_out, uint4 *__restrict__ v_out) {
    const long bh = blockIdx.y;
    const long i = (long)blockIdx.x * (blockDim.x / row_vec) + threadIdx.x / row_vec;
    const int c = threadIdx.x % row_vec;
    if (i >= keep) return;
    const long t = idx[bh * keep + i];
    k_out[((size_t)bh * keep + i) * row_vec + c] = k[((size_t)bh * S + t) * row_vec + c];
    v_out[((size_t)bh * keep + i) * row_vec + c] = v[((size_t)bh * S + t) * row_vec + c];
}

size_t snapkv_smem_bytes() {
    return (size_t)kSnapMaxRows * 256 + (size_t)kSnapStages * kSnapKeys * 256 + 8 * kSnapKeys * 4;
}

// CTAs per head: about six waves of two CTAs per SM over the whole launch,
// at least four 64-key tiles per CTA, at most kSnapMaxSplit
int snapkv_splits(long BH, int S, int num_sms) {
    const int ntile = (S + kSnapKeys - 1) / kSnapKeys;
    long ns = (12L * num_sms + BH - 1) / (BH > 0 ? BH : 1);
    ns = std::min<long>(ns, kSnapMaxSplit);
    ns = std::min<long>(ns, std::max(1, ntile / 4));
    return (int)std::max<long>(ns, 1);
}

size_t snapkv_partials_bytes(long BH) { return (size_t)BH * kSnapMaxSplit * kSnapMaxRows * 2 * sizeof(float); }

cudaError_t launch_snapkv(const void *k, const void *v, const void *q_obs, long BH, int S, int G, int W, int keep,
                          int pool, void *k_out, void *v_out, int *idx_out, void *ws, cudaStream_t st) {
    const long P = (long)S - W;
    float *scores = reinterpret_cast<float *>(static_cast<char *>(ws) + kWsHeader);
    uint32_t *pooled = reinterpret_cast<uint32_t *>(scores + (size_t)BH * P);
    float *ml = reinterpret_cast<float *>(pooled + (size_t)BH * P);
    const size_t smem = snapkv_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(snap_pass_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(snap_pass_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const int ns = snapkv_splits(BH, S, nsm);
    const __nv_bfloat16 *kb = static_cast<const __nv_bfloat16 *>(k);
    const __nv_bfloat16 *qb = static_cast<const __nv_bfloat16 *>(q_obs);
    snap_pass_kernel<0><<<(unsigned)(BH * ns), kSnapThreads, smem, st>>>(kb, qb, S, G, W, ns, ml, scores);
    snap_pass_kernel<1><<<(unsigned)(BH * ns), kSnapThreads, smem, st>>>(kb, qb, S, G, W, ns, ml, scores);
    snap_select_kernel<<<(unsigned)BH, kSelThreads, 0, st>>>(scores, pooled, S, W, keep, pool, idx_out);
    const int row_vec = kD * 2 / 16;  // bf16 rows
    const int rows_per_cta = 256 / row_vec;
    snap_gather_kernel<<<dim3((unsigned)((keep + rows_per_cta - 1) / rows_per_cta), (unsigned)BH), 256, 0, st>>>(
        static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), idx_out, S, keep, row_vec,
        static_cast<uint4 *>(k_out), static_cast<uint4 *>(v_out));
    return cudaGetLastError();
}

}  // namespace spark
