// Recover-then-attend decode attention over the SparK pruned key cache.
//
// Method: "KV Cache 还能再砍一刀：SparK ..." (paper walkthrough) section 3.3
// steps 2-4 and the F table (Degenerate: the sampled score is mu_pruned and
// the key is back-solved as k~_j = mu_pruned / ||q^j||_2), Fig. 3 (decode runs
// standard full attention over the recovered keys); AMD blog "AAAI 2026
// AMD论文Spark方法揭秘" (same).  Flash-decoding split-K with a log-sum-exp
// combine is the standard way to run that attention on one GPU.
//
// Score algebra.  With c_j = mu / qn_j (0 when qn_j = 0) the recovered key is
// k~_j = k_j on kept channels and c_j on pruned ones, so
//     q . k~ = sum_j q_j c_j + sum_{kept j} q_j (k_j - c_j).
// The first term is one constant per query head (Qc); the second touches only
// the T kept values, which is all the cache holds.  Identical to the dense
// recover-then-attend form in real arithmetic; fp32 rounding differs.
//
// decode_kernel: one CTA per (unit, row, kv head).  Units 0..n_pre-1 each own
// a contiguous chunk of prompt tokens; unit n_pre owns the dense tail.  A
// prompt chunk is streamed in 64-token tiles by cp.async.bulk copies
// (mask 16 B/token, interleaved kept values T*es B/token, dense V 256 B/token)
// into an nstage-deep shared-memory ring completed on mbarriers, with bounded
// waits.  Per tile: two threads per token walk the set bits of their 64-bit
// half of the mask and accumulate q'_g (k_j - c_j) for the G heads of the
// group (q' pre-scaled by log2(e)/sqrt(D)); a CTA-wide max updates the running
// max; p = 2^(s - m) goes to shared memory; then 16 channel-groups x 8 token
// subsets accumulate p * V in fp32.  Each unit writes (acc[G][D], m, l).
// combine_kernel merges the units of a (row, head) in a fixed order.
#include "spark_internal.cuh"

#include <algorithm>

namespace spark {

struct DecArgs {
    const void *q;
    const uint32_t *mask;
    const void *vals;
    const float *qn;
    const double *stats;
    const void *v;
    const void *k_tail;
    const void *v_tail;
    float *part;       // [BH][units][G][D + 2]: acc[D], m, l
    uint32_t *status;  // device status word
    int S;
    long S32;
    int T;
    int tail_cap;
    int n_tail;
    int chunk;
    int n_pre;
    int units;
    int nstage;
};

// 8 consecutive channels of a V (or K) row as fp32
template <typename E> struct Row8;
template <> struct Row8<__nv_bfloat16> {
    __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float (&x)[8]) {
        const uint4 u = *reinterpret_cast<const uint4 *>(p);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};
template <> struct Row8<float> {
    __device__ __forceinline__ static void load(const float *p, float (&x)[8]) {
        const float4 a = *reinterpret_cast<const float4 *>(p);
        const float4 b = *reinterpret_cast<const float4 *>(p + 4);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
};

template <int G> struct QVec {
    float v[G];
    __device__ __forceinline__ void load(const float *p) {
        if constexpr (G % 4 == 0) {
#pragma unroll
            for (int i = 0; i < G; i += 4) {
                const float4 a = *reinterpret_cast<const float4 *>(p + i);
                v[i] = a.x; v[i + 1] = a.y; v[i + 2] = a.z; v[i + 3] = a.w;
            }
        } else if constexpr (G == 2) {
            const float2 a = *reinterpret_cast<const float2 *>(p);
            v[0] = a.x; v[1] = a.y;
        } else {
#pragma unroll
            for (int i = 0; i < G; ++i) v[i] = p[i];
        }
    }
};

// log2(e) / sqrt(128): folds the softmax scale and the exp -> exp2 change
// into the query.
constexpr float kQScale = 0.12751743074602467f;

template <typename E, int G>
struct Smem {
    float *tabq;   // [kD][G]
    float *tabc;   // [kD]
    float *qc;     // [G] (16 floats reserved)
    float *pbuf;   // [kNT][G]
    float *wmax;   // [4][G]
    uint64_t *bars;
    unsigned char *stages;
    size_t stage_bytes;
    int T;
    __device__ __forceinline__ uint32_t *smask(int st) const {
        return reinterpret_cast<uint32_t *>(stages + (size_t)st * stage_bytes);
    }
    __device__ __forceinline__ E *svals(int st) const {
        return reinterpret_cast<E *>(stages + (size_t)st * stage_bytes + kNT * 16);
    }
    __device__ __forceinline__ E *sV(int st) const {
        return reinterpret_cast<E *>(stages + (size_t)st * stage_bytes + kNT * 16 +
                                     (size_t)kNT * T * sizeof(E));
    }
};

// One tile's softmax update + P.V accumulation, shared by the prompt and the
// tail paths.  s[] holds this thread's token scores (thread pair per token,
// both halves hold the same sums).  Returns false when the CTA must stop.
template <typename E, int G, typename VRow>
__device__ __forceinline__ void softmax_pv(const Smem<E, G> &sm, const float (&s)[G], int n,
                                           float (&m_run)[G], float (&acc)[G][8], float (&lsum)[G],
                                           VRow vrow) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tt = tid >> 1, h = tid & 1;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const int mx = __reduce_max_sync(0xffffffffu, f2ord(s[g]));
        if (lane == 0) sm.wmax[warp * G + g] = ord2f(mx);
    }
    __syncthreads();
    float alpha[G];
    bool rescale = false;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float mt = sm.wmax[g];
#pragma unroll
        for (int w = 1; w < kDecThreads / 32; ++w) mt = fmaxf(mt, sm.wmax[w * G + g]);
        const float m_new = fmaxf(m_run[g], mt);
        alpha[g] = (m_new == -INFINITY) ? 1.f : exp2f(m_run[g] - m_new);
        rescale |= (alpha[g] != 1.f);
        m_run[g] = m_new;
    }
    if (h == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g)
            sm.pbuf[tt * G + g] = (m_run[g] == -INFINITY) ? 0.f : exp2f(s[g] - m_run[g]);
    }
    __syncthreads();
    if (rescale) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            lsum[g] *= alpha[g];
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[g][c] *= alpha[g];
        }
    }
    const int cg = tid & 15, ts = tid >> 4;
#pragma unroll 2
    for (int kk = 0; kk < kNT / 8; ++kk) {
        const int t2 = ts * (kNT / 8) + kk;
        if (t2 < n) {
            QVec<G> p;
            p.load(sm.pbuf + t2 * G);
            float x[8];
            Row8<E>::load(vrow(t2) + 8 * cg, x);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                lsum[g] += p.v[g];
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[g][c] = fmaf(p.v[g], x[c], acc[g][c]);
            }
        }
    }
}

template <typename E, int G>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(DecArgs a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const int tid = threadIdx.x, lane = tid & 31;
    const int unit = blockIdx.x % a.units;
    const long bh = blockIdx.x / a.units;
    const int es = (int)sizeof(E);

    Smem<E, G> sm;
    sm.T = a.T;
    sm.tabq = reinterpret_cast<float *>(smem_raw);
    sm.tabc = sm.tabq + kD * G;
    sm.qc = sm.tabc + kD;
    sm.pbuf = sm.qc + 16;
    sm.wmax = sm.pbuf + kNT * G;
    {
        uintptr_t p = reinterpret_cast<uintptr_t>(sm.wmax + 4 * G);
        p = (p + 7) & ~uintptr_t(7);
        sm.bars = reinterpret_cast<uint64_t *>(p);
        p = reinterpret_cast<uintptr_t>(sm.bars + kMaxStages);
        p = (p + 127) & ~uintptr_t(127);
        sm.stages = reinterpret_cast<unsigned char *>(p);
    }
    sm.stage_bytes = dec_stage_bytes(a.T, es);

    const bool tail_unit = (unit == a.n_pre);

    // ---- tables: q' (scaled query), c_j = mu / qn_j, Qc = sum_j q'_j c_j
    {
        const int j = tid;
        const E *q = static_cast<const E *>(a.q) + (size_t)bh * G * kD;
        const double mu = a.stats[bh * 4 + 3];
        const float qnj = a.qn[bh * kD + j];
        const float c = (!tail_unit && qnj > 0.f) ? (float)(mu / (double)qnj) : 0.f;
        sm.tabc[j] = c;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float qq = Elem<E>::to_f(q[(size_t)g * kD + j]) * kQScale;
            sm.tabq[j * G + g] = qq;
            float prod = qq * c;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) prod += __shfl_xor_sync(0xffffffffu, prod, o);
            if (lane == 0) sm.wmax[(tid >> 5) * G + g] = prod;
        }
        if (tid == 0) {
            for (int st = 0; st < a.nstage; ++st) mbar_init(smem_u32(sm.bars + st), 1);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        __syncthreads();
        if (tid < G) {
            float s = 0.f;
            for (int w = 0; w < kDecThreads / 32; ++w) s += sm.wmax[w * G + tid];
            sm.qc[tid] = s;
        }
        __syncthreads();
    }

    float m_run[G], lsum[G], acc[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m_run[g] = -INFINITY;
        lsum[g] = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[g][c] = 0.f;
    }
    bool failed = false;
    const int tt = tid >> 1, h = tid & 1;

    if (!tail_unit) {
        const long t_begin = (long)unit * a.chunk;
        const long t_end = min((long)a.S, t_begin + a.chunk);
        const int ntiles = t_end > t_begin ? (int)((t_end - t_begin + kNT - 1) / kNT) : 0;
        const uint32_t *gmask = a.mask + (size_t)bh * a.S * kMaskWords;
        const E *gvals = static_cast<const E *>(a.vals) + (size_t)bh * a.S32 * a.T;
        const E *gv = static_cast<const E *>(a.v) + (size_t)bh * a.S * kD;

        auto issue = [&](int i) {
            const int st = i % a.nstage;
            const long t0 = t_begin + (long)i * kNT;
            const int n = (int)min((long)kNT, t_end - t0);
            const uint32_t mb = (uint32_t)n * 16u;
            const uint32_t vb = (uint32_t)((n + 31) / 32) * 32u * (uint32_t)a.T * (uint32_t)es;
            const uint32_t Vb = (uint32_t)n * kD * (uint32_t)es;
            const uint32_t bar = smem_u32(sm.bars + st);
            mbar_expect_tx(bar, mb + vb + Vb);
            bulk_g2s(smem_u32(sm.smask(st)), gmask + t0 * kMaskWords, mb, bar);
            if (vb) bulk_g2s(smem_u32(sm.svals(st)), gvals + t0 * a.T, vb, bar);
            bulk_g2s(smem_u32(sm.sV(st)), gv + t0 * kD, Vb, bar);
        };
        if (tid == 0)
            for (int i = 0; i < min(a.nstage, ntiles); ++i) issue(i);

        int consumed = 0;
        for (int i = 0; i < ntiles; ++i) {
            const int st = i % a.nstage;
            const long t0 = t_begin + (long)i * kNT;
            const int n = (int)min((long)kNT, t_end - t0);
            bool ok = mbar_wait_bounded(smem_u32(sm.bars + st), (uint32_t)((i / a.nstage) & 1));
            if (!__syncthreads_and(ok)) {
                failed = true;
                break;
            }
            consumed = i + 1;

            // ---- scores: two threads per token, 64 channels each
            float s[G];
#pragma unroll
            for (int g = 0; g < G; ++g) s[g] = 0.f;
            const bool valid = tt < n;
            if (valid && a.T > 0) {
                const uint4 mw = *reinterpret_cast<const uint4 *>(sm.smask(st) + tt * kMaskWords);
                uint32_t wa = h ? mw.z : mw.x;
                uint32_t wb = h ? mw.w : mw.y;
                int pos = h ? (__popc(mw.x) + __popc(mw.y)) : 0;
                const E *vcol = sm.svals(st) + (tt >> 5) * 32 * a.T + (tt & 31);
                const int jb = 64 * h;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t cur = half ? wb : wa;
                    const int jbase = jb + 32 * half;
                    while (cur) {
                        const int b = __ffs(cur) - 1;
                        cur &= cur - 1u;
                        const int j = jbase + b;
                        // a mask with more than T bits (a cache never written by
                        // spark_prune) must not index past this stage
                        const float kv = Elem<E>::to_f(vcol[min(pos, a.T - 1) * 32]);
                        ++pos;
                        const float x = kv - sm.tabc[j];
                        QVec<G> qv;
                        qv.load(sm.tabq + j * G);
#pragma unroll
                        for (int g = 0; g < G; ++g) s[g] = fmaf(qv.v[g], x, s[g]);
                    }
                }
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
                s[g] += __shfl_xor_sync(0xffffffffu, s[g], 1);
                s[g] = valid ? s[g] + sm.qc[g] : -INFINITY;
            }
            const E *sV = sm.sV(st);
            softmax_pv<E, G>(sm, s, n, m_run, acc, lsum, [&](int t2) { return sV + (size_t)t2 * kD; });
            __syncthreads();  // stage and p buffer free
            if (tid == 0 && i + a.nstage < ntiles) {
                fence_proxy_async_smem();
                issue(i + a.nstage);
            }
        }
        if (failed) {
            if (tid == 0) {
                atomicOr(a.status, kDevTimeout);
                // let copies already in flight land before the CTA exits
                const int issued = min(ntiles, consumed + a.nstage);
                for (int i = consumed; i < issued; ++i)
                    (void)mbar_wait_bounded(smem_u32(sm.bars + (i % a.nstage)),
                                            (uint32_t)((i / a.nstage) & 1));
            }
            return;
        }
    } else {
        // ---- dense tail: keys and values read straight from global memory
        const E *kt = static_cast<const E *>(a.k_tail) + (size_t)bh * a.tail_cap * kD;
        const E *vt = static_cast<const E *>(a.v_tail) + (size_t)bh * a.tail_cap * kD;
        for (int t0 = 0; t0 < a.n_tail; t0 += kNT) {
            const int n = min(kNT, a.n_tail - t0);
            float s[G];
#pragma unroll
            for (int g = 0; g < G; ++g) s[g] = 0.f;
            const bool valid = tt < n;
            if (valid) {
                const E *krow = kt + (size_t)(t0 + tt) * kD + 64 * h;
#pragma unroll 2
                for (int c8 = 0; c8 < 8; ++c8) {
                    float x[8];
                    Row8<E>::load(krow + 8 * c8, x);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        QVec<G> qv;
                        qv.load(sm.tabq + (64 * h + 8 * c8 + c) * G);
#pragma unroll
                        for (int g = 0; g < G; ++g) s[g] = fmaf(qv.v[g], x[c], s[g]);
                    }
                }
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
                s[g] += __shfl_xor_sync(0xffffffffu, s[g], 1);
                s[g] = valid ? s[g] : -INFINITY;
            }
            const E *vbase = vt + (size_t)t0 * kD;
            softmax_pv<E, G>(sm, s, n, m_run, acc, lsum, [&](int t2) { return vbase + (size_t)t2 * kD; });
            __syncthreads();
        }
    }

    // ---- epilogue: reduce the 8 token subsets in a fixed order
    float *red = reinterpret_cast<float *>(sm.stages);  // [8][G][kD] then [8][G]
    float *lred = red + 8 * G * kD;
    const int cg = tid & 15, ts = tid >> 4;
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int c = 0; c < 8; ++c) red[(ts * G + g) * kD + 8 * cg + c] = acc[g][c];
        if (cg == 0) lred[ts * G + g] = lsum[g];
    }
    __syncthreads();
    float *out = a.part + ((size_t)bh * a.units + unit) * G * (kD + 2);
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float o = 0.f;
#pragma unroll
        for (int k2 = 0; k2 < 8; ++k2) o += red[(k2 * G + g) * kD + tid];
        out[g * (kD + 2) + tid] = o;
    }
    if (tid < G) {
        float l = 0.f;
        for (int k2 = 0; k2 < 8; ++k2) l += lred[k2 * G + tid];
        out[tid * (kD + 2) + kD] = m_run[tid];
        out[tid * (kD + 2) + kD + 1] = l;
    }
}

template <int G>
__global__ void __launch_bounds__(kD) combine_kernel(const float *__restrict__ part, int units,
                                                     float *__restrict__ out) {
    const long row = blockIdx.x;  // (bh, g)
    const long bh = row / G;
    const int g = (int)(row % G);
    const int d = threadIdx.x;
    const size_t ustride = (size_t)G * (kD + 2);
    const float *base = part + (size_t)bh * units * ustride + (size_t)g * (kD + 2);
    float M = -INFINITY;
    for (int u = 0; u < units; ++u) M = fmaxf(M, base[u * ustride + kD]);
    float L = 0.f, o = 0.f;
    if (M != -INFINITY) {
        for (int u = 0; u < units; ++u) {
            const float mu = base[u * ustride + kD];
            const float lu = base[u * ustride + kD + 1];
            if (lu > 0.f) {
                const float w = exp2f(mu - M);
                L = fmaf(lu, w, L);
                o = fmaf(base[u * ustride + d], w, o);
            }
        }
    }
    out[row * kD + d] = (L > 0.f) ? o / L : 0.f;
}

DecodeGeom decode_geometry(long BH, int S, int T, int es, int G, int num_sms) {
    DecodeGeom g{};
    const size_t stage = dec_stage_bytes(T, es);
    const size_t fixed = dec_fixed_bytes(G);
    const size_t epi = dec_epilogue_bytes(G);
    const size_t per_sm = 228 * 1024, per_cta_max = 227 * 1024;
    g.ctas_per_sm = 1;
    g.nstage = 2;
    for (int cpsm = 3; cpsm >= 1; --cpsm) {
        const size_t lim = std::min(per_cta_max, per_sm / cpsm - 1024);
        if (lim <= fixed) continue;
        const int ns = (int)std::min<size_t>(kMaxStages, (lim - fixed) / stage);
        if (ns >= (cpsm > 1 ? 3 : 2)) {
            g.ctas_per_sm = cpsm;
            g.nstage = ns;
            break;
        }
    }
    g.smem = fixed + std::max((size_t)g.nstage * stage, epi);

    if (S <= 0 || BH <= 0) {
        g.chunk = kNT;
        g.n_pre = 0;
    } else {
        const long slots = (long)num_sms * g.ctas_per_sm;
        const long overhead = 512;  // per-unit fixed cost in token equivalents
        double best = 1e300;
        for (int w = 1; w <= 256; ++w) {
            long n_pre = std::max(1L, (w * slots) / BH);
            long chunk = ((S + n_pre - 1) / n_pre + kNT - 1) / kNT * kNT;
            n_pre = (S + chunk - 1) / chunk;
            const long waves = (BH * n_pre + slots - 1) / slots;
            const double cost = (double)waves * (double)(chunk + overhead);
            if (cost < best) {
                best = cost;
                g.chunk = (int)chunk;
                g.n_pre = (int)n_pre;
            }
            if (chunk == kNT) break;
        }
    }
    g.units = g.n_pre + 1;
    return g;
}

template <typename E, int G>
static cudaError_t launch_decode_t(const DecArgs &a0, long BH, const DecodeGeom &geo, float *out,
                                   cudaStream_t st) {
    DecArgs a = a0;
    a.chunk = geo.chunk;
    a.n_pre = geo.n_pre;
    a.units = geo.units;
    a.nstage = geo.nstage;
    auto kern = decode_kernel<E, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)geo.smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(BH * geo.units), kDecThreads, geo.smem, st>>>(a);
    combine_kernel<G><<<(unsigned)(BH * G), kD, 0, st>>>(a.part, geo.units, out);
    return cudaGetLastError();
}

template <typename E>
static cudaError_t dispatch_g(const DecArgs &a, long BH, const DecodeGeom &geo, int G, float *out,
                              cudaStream_t st) {
    switch (G) {
    case 1: return launch_decode_t<E, 1>(a, BH, geo, out, st);
    case 2: return launch_decode_t<E, 2>(a, BH, geo, out, st);
    case 4: return launch_decode_t<E, 4>(a, BH, geo, out, st);
    case 8: return launch_decode_t<E, 8>(a, BH, geo, out, st);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode(const void *q, const spark_kcache &kc, const void *v, const void *k_tail,
                          const void *v_tail, int tail_cap, int n_tail, int G, float *out, void *ws,
                          const DecodeGeom &geo, cudaStream_t st) {
    const long BH = (long)kc.B * kc.Hkv;
    if (BH == 0) return cudaSuccess;
    DecArgs a{};
    a.q = q;
    a.mask = kc.mask;
    a.vals = kc.vals;
    a.qn = kc.qn;
    a.stats = kc.stats;
    a.v = v;
    a.k_tail = k_tail;
    a.v_tail = v_tail;
    a.status = static_cast<uint32_t *>(ws);
    a.part = reinterpret_cast<float *>(static_cast<char *>(ws) + kWsHeader);
    a.S = kc.S;
    a.S32 = ((long)kc.S + 31) / 32 * 32;
    a.T = kc.T;
    a.tail_cap = tail_cap;
    a.n_tail = n_tail;
    if (kc.dtype == SPARK_BF16) return dispatch_g<__nv_bfloat16>(a, BH, geo, G, out, st);
    return dispatch_g<float>(a, BH, geo, G, out, st);
}

}  // namespace spark
