// Recover-then-attend decode attention over the SparK pruned key cache.
//
// Method: "KV Cache 还能再砍一刀：SparK ..." (paper walkthrough) section 3.3
// steps 2-4 and the F table (Degenerate: the sampled score is mu_pruned and
// the key is back-solved as k~_j = mu_pruned / ||q^j||_2), Fig. 3 (decode runs
// standard full attention over the recovered keys); AMD blog "AAAI 2026
// AMD论文Spark方法揭秘" (same).  Split-K flash decoding with a log-sum-exp
// combine is the standard way to run that attention on one GPU.
//
// Score algebra.  With c_j = mu / qn_j (0 when qn_j = 0) the recovered key is
// k~_j = k_j on kept channels and c_j on pruned ones, so
//     q . k~ = sum_j q_j c_j + sum_{kept j} q_j (k_j - c_j).
// The first term is one constant per query head (Qc); the second touches only
// the T kept values, which is all the cache holds.  Identical to the dense
// recover-then-attend form in real arithmetic; fp32 rounding differs.
//
// decode_kernel: a persistent grid, one CTA per SM, whose warps are
// independent flash-decoding workers.  Work items are (row, kv head, chunk of
// prompt tokens) plus one dense-tail item per head; warp w of the grid takes
// items w, w + #warps, ... (prompt items first, warps numbered CTA-fastest).
// Each warp streams its items' 32-token tiles: the mask (16 B/token) and one
// 32-token group of interleaved kept values (T*es B/token) by cp.async.bulk
// copies, issued by its lane 0 into its own ring of shared-memory stages and
// completed on per-stage mbarriers (bounded waits).  The dense V rows
// (256 B/token) are issued before the tile's q.k~ so that they land under it:
// for bf16 by cp.async into an XOR-swizzled per-warp tile, for fp32 by
// coalesced 8-byte loads into registers.  No CTA-wide barrier is on the path.
// Per tile:
//   q.k~     lane = token; for T < 48 the lane walks exactly T set bits of
//            its 128-bit mask from the top channel down (a queue of the
//            non-empty mask words, one bfind and one bit clear per step, no
//            branch) and accumulates q'_g (k_j - c_j) for the G heads of the
//            group from the q' / c tables (q' = q * log2(e)/sqrt(D)); for
//            larger T (the value-pruned decode included), and for a SparK-p
//            cache (masks with fewer bits than its T value slots), all lanes
//            step through the 128 channels together, so that the table reads
//            are broadcasts, and pruned channels are predicated off -- the
//            same sums in the same order;
//   softmax  warp max (integer REDUX on an order-preserving map) updates the
//            running max; p = 2^(s - m) goes to shared memory;
//   P.V      bf16: tensor cores -- the V tile is the B operand
//            (ldmatrix.trans), p is the A operand split into bf16 hi + lo
//            parts (two mma.sync m16n8k16 per tile, fp32 accumulators), so
//            the products keep ~16 bits of p; fp32: lane = 4 value channels,
//            packed fp32x2 FMAs over the tokens.
// At the end of an item the warp writes (acc[G][D], m, l) for it;
// combine_kernel merges a head's items, eight warps over disjoint item
// slices with loads in flight, then the warp sums in a fixed order.
#include "spark_internal.cuh"

#include <algorithm>

namespace spark {

struct DecArgs {
    const void *q;
    const uint32_t *mask;
    const void *vals;
    const uint32_t *goff;   // SparK-p cache: first value row of each group (else NULL)
    const int32_t *lens;    // prompt tokens per row (else NULL: S for every row)
    int Hkv;
    const uint32_t *vmask;  // pruned value cache (packed-V kernels only)
    const void *vvals;
    int Tv;
    const float *qn;
    const double *stats;
    const void *v;
    const void *k_tail;
    const void *v_tail;
    float *acc;        // [BH][units][G][D]
    float *ml;         // [BH][units][G][2]
    uint32_t *status;  // device status word
    long BH;
    int S;
    long S32;
    int T;
    int tail_cap;
    int n_tail;
    int chunk;
    int n_pre;
    int units;
    int nstage;
    int nwarp;
    size_t warp_bytes;
    unsigned long long seed;  // sampling recoveries only
};

// log2(e) / sqrt(128): folds the softmax scale and the exp -> exp2 change
// into the query.
constexpr float kQScale = 0.12751743074602467f;

// ---- sampling recoveries (F table: Gaussian N(mu, sigma^2), Exponential
// Exp(1/mu)).  One draw per pruned (token, channel) entry, fixed for a given
// seed: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11) with counter
// (t, j, bh low word, bh high word) and key (seed low word, seed high word);
// uniforms from the top 24 bits of the first two output words.
__device__ __forceinline__ void philox4x32_10(uint32_t (&c)[4], uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint32_t hi0 = __umulhi(0xD2511F53u, c[0]), lo0 = 0xD2511F53u * c[0];
        const uint32_t hi1 = __umulhi(0xCD9E8D57u, c[2]), lo1 = 0xCD9E8D57u * c[2];
        const uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
        c[0] = n0;
        c[1] = lo1;
        c[2] = n2;
        c[3] = lo0;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
}

// sampled saliency score of pruned entry (bh, t, j); kF = 1 Gaussian, 2 Exponential
template <int kF>
__device__ __forceinline__ float sample_score(unsigned long long seed, long bh, long t, int j, float mu,
                                              float sigma) {
    uint32_t c[4] = {(uint32_t)t, (uint32_t)j, (uint32_t)((unsigned long long)bh & 0xffffffffu),
                     (uint32_t)((unsigned long long)bh >> 32)};
    philox4x32_10(c, (uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32));
    const float u1 = (float)((c[0] >> 8) + 1u) * (1.0f / 16777216.0f);  // (0, 1], exact
    if constexpr (kF == 2) {
        return -mu * logf(u1);
    } else {
        const float u2 = (float)(c[1] >> 8) * (1.0f / 16777216.0f);    // [0, 1), exact
        return mu + sigma * sqrtf(-2.0f * logf(u1)) * cospif(2.0f * u2);
    }
}

// 4 consecutive channels of a key row (dense tail) as fp32
template <typename E> struct Row4;
template <> struct Row4<__nv_bfloat16> {
    __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float (&x)[4]) {
        const uint2 u = *reinterpret_cast<const uint2 *>(p);
        x[0] = __uint_as_float(u.x << 16);
        x[1] = __uint_as_float(u.x & 0xffff0000u);
        x[2] = __uint_as_float(u.y << 16);
        x[3] = __uint_as_float(u.y & 0xffff0000u);
    }
};
template <> struct Row4<float> {
    __device__ __forceinline__ static void load(const float *p, float (&x)[4]) {
        const float4 a = *reinterpret_cast<const float4 *>(p);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    }
};

// This lane's 4 value channels of a batch of consecutive tokens, in
// registers: 32 tokens for bf16, 16 for fp32 (64 registers either way).
template <typename E> struct VRegs;
template <> struct VRegs<__nv_bfloat16> {
    static constexpr int kTok = 32;
    uint2 v[kTok];
    // row0 points at channel 4*lane of the batch's first token
    __device__ __forceinline__ void load(const __nv_bfloat16 *row0, int n) {
        if (n >= kTok) {
#pragma unroll
            for (int t = 0; t < kTok; ++t) v[t] = __ldcs(reinterpret_cast<const uint2 *>(row0 + (size_t)t * kD));
        } else {
#pragma unroll
            for (int t = 0; t < kTok; ++t)
                v[t] = (t < n) ? __ldcs(reinterpret_cast<const uint2 *>(row0 + (size_t)t * kD)) : make_uint2(0u, 0u);
        }
    }
    __device__ __forceinline__ void get(int t, float2 &x01, float2 &x23) const {
        x01 = make_float2(__uint_as_float(v[t].x << 16), __uint_as_float(v[t].x & 0xffff0000u));
        x23 = make_float2(__uint_as_float(v[t].y << 16), __uint_as_float(v[t].y & 0xffff0000u));
    }
};
template <> struct VRegs<float> {
    static constexpr int kTok = 16;
    float4 v[kTok];
    __device__ __forceinline__ void load(const float *row0, int n) {
        if (n >= kTok) {
#pragma unroll
            for (int t = 0; t < kTok; ++t) v[t] = __ldcs(reinterpret_cast<const float4 *>(row0 + (size_t)t * kD));
        } else {
#pragma unroll
            for (int t = 0; t < kTok; ++t)
                v[t] = (t < n) ? __ldcs(reinterpret_cast<const float4 *>(row0 + (size_t)t * kD))
                               : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    __device__ __forceinline__ void get(int t, float2 &x01, float2 &x23) const {
        x01 = make_float2(v[t].x, v[t].y);
        x23 = make_float2(v[t].z, v[t].w);
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

// Position of the highest set bit, 0xffffffff for zero.
__device__ __forceinline__ uint32_t bit_top(uint32_t x) {
    uint32_t p;
    asm("bfind.u32 %0, %1;" : "=r"(p) : "r"(x));
    return p;
}

// (1 << n) - 1: the bits below position n, all ones for n >= 32 (bmsk with
// clamping), so `x & bit_mask_below(bit_top(x))` clears x's top bit and
// leaves 0 at 0.
__device__ __forceinline__ uint32_t bit_mask_below(uint32_t n) {
    uint32_t m;
    asm("bmsk.clamp.b32 %0, 0, %1;" : "=r"(m) : "r"(n));
    return m;
}

// Stable compaction of the queue (q0, q1, q2, q3) so that its non-empty words
// come first; byte k of bq is the channel base of word k and moves with it.
// Works from the back: after the step for slot k, slots k..3 are compacted.
__device__ __forceinline__ void queue_nonempty(uint32_t &q0, uint32_t &q1, uint32_t &q2, uint32_t &q3,
                                               uint32_t &bq) {
    bool e = q2 == 0u;  // drop slot 2
    q2 = e ? q3 : q2;
    q3 = e ? 0u : q3;
    bq = e ? __byte_perm(bq, 0u, 0x4310) : bq;
    e = q1 == 0u;       // drop slot 1
    q1 = e ? q2 : q1;
    q2 = e ? q3 : q2;
    q3 = e ? 0u : q3;
    bq = e ? __byte_perm(bq, 0u, 0x4320) : bq;
    e = q0 == 0u;       // drop slot 0
    q0 = e ? q1 : q0;
    q1 = e ? q2 : q1;
    q2 = e ? q3 : q2;
    bq = e ? (bq >> 8) : bq;
}

// Per-warp shared memory: tables, p buffers, mbarriers, then the stage ring.
template <typename E, int G>
struct WarpSmem {
    unsigned char *vt;  // bf16 values: swizzled V tile [kWT][kD]
    float *pT;     // [G][kWT] p of the tile, head-major (tensor-core P.V)
    float *tabq;   // [kD][G]   q' per channel
    float *tabc;   // [kD]      c_j = mu / qn_j (1 / qn_j for sampling F)
    float *pdup;   // [kWT][G][2] p duplicated into fp32 pairs (CUDA-core P.V)
    float *qc;     // [G] Qc = sum_j q'_j c_j of the current head
    uint64_t *bars;
    unsigned char *stages;
    uint32_t stage_bytes;
    uint32_t vstage_off;  // offset of the value cache's part of a stage
    __device__ __forceinline__ const uint32_t *svmask(int st) const {
        return reinterpret_cast<const uint32_t *>(stages + (size_t)st * stage_bytes + vstage_off);
    }
    __device__ __forceinline__ const E *svvals(int st) const {
        return reinterpret_cast<const E *>(stages + (size_t)st * stage_bytes + vstage_off + kWT * 16);
    }
    __device__ __forceinline__ const uint32_t *smask(int st) const {
        return reinterpret_cast<const uint32_t *>(stages + (size_t)st * stage_bytes);
    }
    __device__ __forceinline__ const E *svals(int st) const {
        return reinterpret_cast<const E *>(stages + (size_t)st * stage_bytes + kWT * 16);
    }
};

// online-softmax state of one warp for the item in progress
template <int G>
struct Flash {
    float m[G];  // running max (log2 domain), warp-uniform
    float l[G];  // this lane's share of the running sum
    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            m[g] = -INFINITY;
            l[g] = 0.f;
        }
    }
};

// Online-softmax update for one tile: s[] is this lane's token score (-inf
// for lanes past the tile end).  Leaves p in shared memory in the layout the
// P.V engine reads and returns the factor each head's accumulator is scaled
// by (all 1 when no running max moved).
// 2^x in one MUFU instruction (results below 2^-126 flush to 0: such a
// weight is zero next to the tile's maximum, whose weight is 1)
__device__ __forceinline__ float ex2_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <typename E, int G>
__device__ __forceinline__ bool tile_softmax(const WarpSmem<E, G> &ws, Flash<G> &f, const float (&s)[G],
                                             float (&alpha)[G]) {
    const int lane = threadIdx.x & 31;
    float p[G];
    bool rescale = false;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const float mt = ord2f(__reduce_max_sync(0xffffffffu, f2ord(s[g])));
        const float m_new = fmaxf(f.m[g], mt);
        alpha[g] = (m_new == -INFINITY) ? 1.f : ex2_fast(f.m[g] - m_new);
        rescale |= (alpha[g] != 1.f);
        f.m[g] = m_new;
        p[g] = (m_new == -INFINITY) ? 0.f : ex2_fast(s[g] - m_new);
        f.l[g] = fmaf(f.l[g], alpha[g], p[g]);
    }
    if constexpr (sizeof(E) == 2) {
#pragma unroll
        for (int g = 0; g < G; ++g) ws.pT[g * kWT + lane] = p[g];
    } else {
        float *pd = ws.pdup + lane * G * 2;
        if constexpr (G == 1) {
            *reinterpret_cast<float2 *>(pd) = make_float2(p[0], p[0]);
        } else {
#pragma unroll
            for (int g = 0; g < G; g += 2)
                *reinterpret_cast<float4 *>(pd + 2 * g) = make_float4(p[g], p[g], p[g + 1], p[g + 1]);
        }
    }
    __syncwarp();
    return rescale;
}

// P.V accumulator of one warp.  fp32 values: CUDA cores, V rows streamed into
// registers; bf16 values: tensor cores (below).
template <typename E, int G> struct PV;

template <int G> struct PV<float, G> {
    float2 acc[G][2];  // this lane's 4 value channels, as fp32 pairs
    VRegs<float> vr;
    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int g = 0; g < G; ++g) acc[g][0] = acc[g][1] = make_float2(0.f, 0.f);
    }
    // row0: channel 0 of the tile's first value row (global memory)
    __device__ __forceinline__ void begin(const WarpSmem<float, G> &, const float *row0, int n) {
        vr.load(row0 + 4 * (threadIdx.x & 31), n);
    }
    __device__ __forceinline__ void rescale(const float (&alpha)[G]) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float2 a2 = make_float2(alpha[g], alpha[g]);
            acc[g][0] = __fmul2_rn(acc[g][0], a2);
            acc[g][1] = __fmul2_rn(acc[g][1], a2);
        }
    }
    __device__ __forceinline__ void accumulate(const WarpSmem<float, G> &ws, const float *row0, int n) {
        const int lane = threadIdx.x & 31;
        for (int tb = 0; tb < n; tb += VRegs<float>::kTok) {
            if (tb > 0) vr.load(row0 + (size_t)tb * kD + 4 * lane, n - tb);
#pragma unroll
            for (int t = 0; t < VRegs<float>::kTok; ++t) {
                if (tb + t < n) {
                    float2 x01, x23;
                    vr.get(t, x01, x23);
                    const float *pd = ws.pdup + (tb + t) * G * 2;
                    if constexpr (G == 1) {
                        const float2 pp = *reinterpret_cast<const float2 *>(pd);
                        acc[0][0] = __ffma2_rn(pp, x01, acc[0][0]);
                        acc[0][1] = __ffma2_rn(pp, x23, acc[0][1]);
                    } else {
#pragma unroll
                        for (int g = 0; g < G; g += 2) {
                            const float4 pp = *reinterpret_cast<const float4 *>(pd + 2 * g);
                            const float2 pa = make_float2(pp.x, pp.y), pb = make_float2(pp.z, pp.w);
                            acc[g][0] = __ffma2_rn(pa, x01, acc[g][0]);
                            acc[g][1] = __ffma2_rn(pa, x23, acc[g][1]);
                            acc[g + 1][0] = __ffma2_rn(pb, x01, acc[g + 1][0]);
                            acc[g + 1][1] = __ffma2_rn(pb, x23, acc[g + 1][1]);
                        }
                    }
                }
            }
        }
        __syncwarp();  // p buffer free
    }
    __device__ __forceinline__ void store(float *acc_out) const {  // acc_out: [G][kD] of this item
        const int lane = threadIdx.x & 31;
#pragma unroll
        for (int g = 0; g < G; ++g)
            *reinterpret_cast<float4 *>(acc_out + g * kD + 4 * lane) =
                make_float4(acc[g][0].x, acc[g][0].y, acc[g][1].x, acc[g][1].y);
    }
};

// byte offset of 16-byte chunk c of row t in the swizzled V tile: chunks are
// XOR-ed with the row's low 3 bits so that ldmatrix over 8 rows is free of
// bank conflicts
__device__ __forceinline__ uint32_t vswz(int t, int c) { return (uint32_t)(t * 256 + ((c ^ (t & 7)) << 4)); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    const int n = valid ? 16 : 0;  // zero-fill rows past the tile end
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// bf16 values: out^T[d][g] += V^T[d][t] P^T[t][g] on tensor cores
// (mma.sync m16n8k16, fp32 accumulate): A = V^T read by ldmatrix.trans from
// the swizzled V tile, B = P^T from the head-major p buffer, split into a bf16
// high part and a bf16 remainder (two MMAs) so that p keeps ~16 bits.  The
// accumulator fragment holds channel d = 16*mt + lane/4 (+8) and heads
// 2*(lane%4) (+1); heads >= G are padding.
template <int G> struct PV<__nv_bfloat16, G> {
    static_assert(G <= 8, "the MMA n-dimension holds up to 8 heads");
    float c[8][4];
    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) c[mt][e] = 0.f;
    }
    // copy the tile's V rows (channel 0 of row 0 at row0) into the V tile
    __device__ __forceinline__ void begin(const WarpSmem<__nv_bfloat16, G> &ws, const __nv_bfloat16 *row0,
                                          int n) {
        const int lane = threadIdx.x & 31;
        const int ch = lane & 15, half = lane >> 4;
        const uint32_t base = smem_u32(ws.vt);
#pragma unroll
        for (int i = 0; i < kWT / 2; ++i) {
            const int t = half + 2 * i;
            cp_async16(base + vswz(t, ch), row0 + (size_t)min(t, max(n - 1, 0)) * kD + 8 * ch, t < n);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    __device__ __forceinline__ void rescale(const float (&alpha)[G]) {
        const int lane = threadIdx.x & 31;
        const int h0 = 2 * (lane & 3), h1 = h0 + 1;
        float a0 = 1.f, a1 = 1.f;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            a0 = (h0 == g) ? alpha[g] : a0;
            a1 = (h1 == g) ? alpha[g] : a1;
        }
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            c[mt][0] *= a0;
            c[mt][1] *= a1;
            c[mt][2] *= a0;
            c[mt][3] *= a1;
        }
    }
    __device__ __forceinline__ void accumulate(const WarpSmem<__nv_bfloat16, G> &ws, const __nv_bfloat16 *,
                                               int) {
        const int lane = threadIdx.x & 31;
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncwarp();
        const int head = lane >> 2, tq = 2 * (lane & 3);
        const uint32_t vbase = smem_u32(ws.vt);
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            // B fragments: p of head `head` at tokens 16ks + tq (+1) and +8 (+9)
            uint32_t bh0 = 0u, bh1 = 0u, bl0 = 0u, bl1 = 0u;
            if (head < G) {
                const float2 p01 = *reinterpret_cast<const float2 *>(ws.pT + head * kWT + 16 * ks + tq);
                const float2 p89 = *reinterpret_cast<const float2 *>(ws.pT + head * kWT + 16 * ks + tq + 8);
                const __nv_bfloat162 h01 = __floats2bfloat162_rn(p01.x, p01.y);
                const __nv_bfloat162 h89 = __floats2bfloat162_rn(p89.x, p89.y);
                const __nv_bfloat162 r01 = __floats2bfloat162_rn(p01.x - __low2float(h01), p01.y - __high2float(h01));
                const __nv_bfloat162 r89 = __floats2bfloat162_rn(p89.x - __low2float(h89), p89.y - __high2float(h89));
                bh0 = *reinterpret_cast<const uint32_t *>(&h01);
                bh1 = *reinterpret_cast<const uint32_t *>(&h89);
                bl0 = *reinterpret_cast<const uint32_t *>(&r01);
                bl1 = *reinterpret_cast<const uint32_t *>(&r89);
            }
            const int t = 16 * ks + (lane & 7) + ((lane >> 4) & 1) * 8;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                uint32_t a[4];
                const int ch = 2 * mt + ((lane >> 3) & 1);
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                             : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                             : "r"(vbase + vswz(t, ch)));
                mma_bf16_16816(c[mt], a, bh0, bh1);
                mma_bf16_16816(c[mt], a, bl0, bl1);
            }
        }
        __syncwarp();  // V tile and p buffer free
    }
    __device__ __forceinline__ void store(float *acc_out) const {  // acc_out: [G][kD] of this item
        const int lane = threadIdx.x & 31;
        const int d0 = lane >> 2, h0 = 2 * (lane & 3), h1 = h0 + 1;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            if (h0 < G) {
                acc_out[h0 * kD + 16 * mt + d0] = c[mt][0];
                acc_out[h0 * kD + 16 * mt + d0 + 8] = c[mt][2];
            }
            if (h1 < G) {
                acc_out[h1 * kD + 16 * mt + d0] = c[mt][1];
                acc_out[h1 * kD + 16 * mt + d0 + 8] = c[mt][3];
            }
        }
    }
};

// Write one item's partial state (acc[G][D], m, l) to the workspace.
template <typename E, int G>
__device__ __forceinline__ void write_partial(const DecArgs &a, long bh, int u, const Flash<G> &f,
                                              const PV<E, G> &pv) {
    const int lane = threadIdx.x & 31;
    const size_t row = (size_t)bh * a.units + u;
    pv.store(a.acc + row * G * kD);
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float l = f.l[g];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (lane == 0) {
            a.ml[(row * G + g) * 2 + 0] = f.m[g];
            a.ml[(row * G + g) * 2 + 1] = l;
        }
    }
}

// warps per CTA the kernel is compiled for: 16 (128 registers) for G <= 2,
// 12 (168 registers, no spills) for G >= 4 -- measured faster than 16
// spilling warps on the G = 4 workloads
__host__ __device__ constexpr int dec_max_warps(int G) { return G > 2 ? 12 : kMaxWarps; }

// kF: the recovery F (spark_recovery), or kDegDense: Degenerate F with q.k~
// taken in channel order (every lane visits the same channel at each step, so
// the q' / c table reads are broadcasts) instead of walking each token's kept
// bits.  The channel-order loop also serves caches whose masks hold fewer bits
// than their T value slots (SparK-p: the kept values fill the first slots of
// each token, zeros after; selector kRecoveryDegVar on the host side).
constexpr int kDegDense = kRecoveryDegDense;
__host__ __device__ constexpr bool is_degenerate(int f) { return f == SPARK_F_DEGENERATE || f == kDegDense; }

template <typename E, int G, int kF, bool kPV>
__global__ void __launch_bounds__(dec_max_warps(G) * 32, 1) decode_kernel(DecArgs a) {
    static_assert(!kPV || (sizeof(E) == 2 && is_degenerate(kF)), "packed values: bf16, Degenerate F");
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp >= a.nwarp) return;
    const int es = (int)sizeof(E);

    WarpSmem<E, G> ws;
    {
        unsigned char *base = smem_raw + (size_t)warp * a.warp_bytes;
        ws.vt = base;  // 8 KB for bf16 values, empty for fp32
        ws.pT = reinterpret_cast<float *>(base + dec_vtile_bytes(es));
        ws.tabq = ws.pT + G * kWT;
        ws.tabc = ws.tabq + kD * G;
        ws.pdup = ws.tabc + kD;
        ws.qc = ws.pdup + dec_pdup_bytes(G, es) / sizeof(float);
        ws.bars = reinterpret_cast<uint64_t *>(ws.qc + 16);
        ws.stages = base + dec_table_bytes(G, es);
        ws.vstage_off = (uint32_t)dec_stage_bytes(a.T, es);
        ws.stage_bytes = ws.vstage_off + (kPV ? (uint32_t)dec_stage_bytes(a.Tv, es) : 0u);
    }
    if (lane == 0) {
        for (int st = 0; st < a.nstage; ++st) mbar_init(smem_u32(ws.bars + st), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();

    // Items 0 .. BH*n_pre-1 are prompt chunks (row-major over (head, chunk)),
    // then one dense-tail item per head, so the small tail items fill the idle
    // warps of the last round.  Warps are numbered CTA-fastest so that
    // consecutive items land on different SMs.  Item indices fit in 32 bits
    // (BH * units < 2^31 is checked on the host).
    const int nwt = gridDim.x * a.nwarp;
    const int gw = warp * gridDim.x + blockIdx.x;
    const int n_items = (int)(a.BH * a.units);
    const int n_prompt = (int)(a.BH * a.n_pre);
    auto item_head = [&](int item) -> int { return item < n_prompt ? item / a.n_pre : item - n_prompt; };
    auto item_unit = [&](int item) -> int { return item < n_prompt ? item % a.n_pre : a.n_pre; };

    // prompt tokens of head bh (S is the row stride when rows have lengths)
    auto head_len = [&](int bh) -> int { return row_len(a.lens, bh, a.Hkv, a.S, nullptr); };

    // ---- tile stream of this warp: prompt tiles of its items, in order
    auto item_tiles = [&](int bh, int u) -> int {
        if (u >= a.n_pre) return 0;  // dense-tail items are not streamed
        const long t0 = (long)u * a.chunk;
        const long t1 = min((long)head_len(bh), t0 + a.chunk);
        return t1 > t0 ? (int)((t1 - t0 + kWT - 1) / kWT) : 0;
    };
    // issue cursor: the next prompt tile to copy, with its item decoded once
    struct Cursor {
        int item, tile, ntiles, bh, u;
    };
    auto enter = [&](Cursor &c) {
        c.tile = 0;
        if (c.item < n_items) {
            c.bh = item_head(c.item);
            c.u = item_unit(c.item);
            c.ntiles = item_tiles(c.bh, c.u);
        } else {
            c.ntiles = 0;
        }
    };
    auto settle = [&](Cursor &c) {  // move to the next tile that exists
        while (c.item < n_items && c.tile >= c.ntiles) {
            c.item += nwt;
            enter(c);
        }
    };
    const E *gvals = static_cast<const E *>(a.vals);
    const E *gv = static_cast<const E *>(a.v);
    auto issue = [&](int st, const Cursor &c) {
        const long bh = c.bh;
        const int u = c.u;
        const long t0 = (long)u * a.chunk + (long)c.tile * kWT;
        const long t1 = min((long)head_len((int)bh), (long)u * a.chunk + a.chunk);
        const int n = (int)min((long)kWT, t1 - t0);
        const uint32_t mb = (uint32_t)n * 16u;
        // one whole 32-token group of kept values: T slots, or for a SparK-p
        // cache the group's own slot count, found through goff
        uint32_t vb = (uint32_t)kWT * (uint32_t)a.T * (uint32_t)es;
        const E *vsrc = gvals + (size_t)bh * a.S32 * a.T + (size_t)t0 * a.T;
        if (a.goff) {
            const long gi = bh * (a.S32 / kWT) + t0 / kWT;
            const uint32_t r0 = a.goff[gi], r1 = a.goff[gi + 1];
            vb = (r1 - r0) * (uint32_t)kWT * (uint32_t)es;
            vsrc = gvals + (size_t)r0 * kWT;
        }
        const uint32_t bar = smem_u32(ws.bars + st);
        unsigned char *dst = ws.stages + (size_t)st * ws.stage_bytes;
        const uint32_t vvb = kPV ? (uint32_t)kWT * (uint32_t)a.Tv * (uint32_t)es : 0u;
        mbar_expect_tx(bar, mb + vb + (kPV ? mb + vvb : 0u));
        bulk_g2s(smem_u32(dst), a.mask + ((size_t)bh * a.S + t0) * kMaskWords, mb, bar);
        if (vb) bulk_g2s(smem_u32(dst + kWT * 16), vsrc, vb, bar);
        if constexpr (kPV) {
            bulk_g2s(smem_u32(dst + ws.vstage_off), a.vmask + ((size_t)bh * a.S + t0) * kMaskWords, mb, bar);
            if (vvb)
                bulk_g2s(smem_u32(dst + ws.vstage_off + kWT * 16),
                         static_cast<const E *>(a.vvals) + (size_t)bh * a.S32 * a.Tv + (size_t)t0 * a.Tv, vvb, bar);
        }
    };

    Cursor ic{gw, 0, 0, 0, 0};
    enter(ic);
    settle(ic);
    int issued = 0, consumed = 0;
    if (lane == 0) {
        Cursor c = ic;
        for (int st = 0; st < a.nstage && c.item < n_items; ++st) {
            issue(st, c);
            ++c.tile;
            settle(c);
        }
    }
    for (int st = 0; st < a.nstage && ic.item < n_items; ++st) {  // all lanes track the cursor
        ++issued;
        ++ic.tile;
        settle(ic);
    }

    Flash<G> f;
    PV<E, G> pv;
    int tab_bh = -1;
    bool failed = false;
    float f_mu = 0.f, f_sigma = 0.f;  // sampling recoveries: pruned-score mean, sd

    for (int item = gw; item < n_items && !failed; item += nwt) {
        const int bh = item_head(item);
        const int u = item_unit(item);
        const bool tail = (u == a.n_pre);
        if (tail && a.n_tail == 0) {
            f.reset();
            pv.reset();
            write_partial<E, G>(a, bh, u, f, pv);
            continue;
        }
        // ---- tables of this head: q' (scaled query), c_j = mu / qn_j, Qc
        if (bh != tab_bh) {
            const E *q = static_cast<const E *>(a.q) + (size_t)bh * G * kD;
            const double mu = a.stats[bh * 4 + 3];
            if constexpr (!is_degenerate(kF)) {
                const double n = a.stats[bh * 4 + 0];
                const double var = n > 0.0 ? a.stats[bh * 4 + 2] / n - mu * mu : 0.0;
                f_mu = (float)mu;
                f_sigma = (float)sqrt(var > 0.0 ? var : 0.0);
            }
            float part[G];
#pragma unroll
            for (int g = 0; g < G; ++g) part[g] = 0.f;
#pragma unroll
            for (int i = 0; i < kD / 32; ++i) {
                const int j = lane + 32 * i;
                const float qnj = a.qn[bh * kD + j];
                // Degenerate: c_j = mu / qn_j (folded into Qc); sampling: 1 / qn_j
                const float c = qnj > 0.f ? (is_degenerate(kF) ? (float)(mu / (double)qnj)
                                                                       : (float)(1.0 / (double)qnj))
                                          : 0.f;
                ws.tabc[j] = c;
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float qq = Elem<E>::to_f(q[(size_t)g * kD + j]) * kQScale;
                    ws.tabq[j * G + g] = qq;
                    if constexpr (is_degenerate(kF)) part[g] = fmaf(qq, c, part[g]);
                }
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) part[g] += __shfl_xor_sync(0xffffffffu, part[g], o);
                if (lane == 0) ws.qc[g] = part[g];
            }
            tab_bh = bh;
            __syncwarp();
        }
        f.reset();
        pv.reset();

        if (tail) {
            // ---- dense tail: keys and values read from global memory
            const E *kt = static_cast<const E *>(a.k_tail) + (size_t)bh * a.tail_cap * kD;
            const E *vt = static_cast<const E *>(a.v_tail) + (size_t)bh * a.tail_cap * kD;
            for (int t0 = 0; t0 < a.n_tail; t0 += kWT) {
                const int n = min(kWT, a.n_tail - t0);
                pv.begin(ws, vt + (size_t)t0 * kD, n);
                float s[G];
#pragma unroll
                for (int g = 0; g < G; ++g) s[g] = 0.f;
                if (lane < n) {
                    const E *krow = kt + (size_t)(t0 + lane) * kD;
#pragma unroll 4
                    for (int j4 = 0; j4 < kD; j4 += 4) {
                        float x[4];
                        Row4<E>::load(krow + j4, x);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            QVec<G> qv;
                            qv.load(ws.tabq + (j4 + c) * G);
#pragma unroll
                            for (int g = 0; g < G; ++g) s[g] = fmaf(qv.v[g], x[c], s[g]);
                        }
                    }
                }
#pragma unroll
                for (int g = 0; g < G; ++g) s[g] = (lane < n) ? s[g] : -INFINITY;
                float alpha[G];
                if (tile_softmax<E, G>(ws, f, s, alpha)) pv.rescale(alpha);
                pv.accumulate(ws, vt + (size_t)t0 * kD, n);
            }
            write_partial<E, G>(a, bh, u, f, pv);
            continue;
        }

        // ---- prompt tokens of this item, one 32-token tile at a time
        const int ntiles = item_tiles(bh, u);
        const long t_item = (long)u * a.chunk;
        const long t_end = min((long)head_len(bh), t_item + a.chunk);
        const E *vbase = gv + (size_t)bh * a.S * kD;
        for (int tile = 0; tile < ntiles; ++tile) {
            const long t0 = t_item + (long)tile * kWT;
            const int n = (int)min((long)kWT, t_end - t0);
            // this tile's V rows start moving (registers or shared memory) under
            // the q.k~ below; a pruned value cache arrives with the stage
            if constexpr (!kPV) pv.begin(ws, vbase + (size_t)t0 * kD, n);

            const int st = (int)(consumed % a.nstage);
            const uint32_t par = (uint32_t)((consumed / a.nstage) & 1);
            // every lane waits; the warp agrees on the outcome so that no lane
            // leaves the shuffles and REDUX below on its own
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(ws.bars + st), par))) {
                failed = true;
                break;
            }
            const bool valid = lane < n;

            // q . k~ over the T kept channels of this lane's token
            float s[G];
#pragma unroll
            for (int g = 0; g < G; ++g) s[g] = 0.f;
            if constexpr (!is_degenerate(kF)) {
                // every channel: kept -> stored value, pruned -> sampled score / qn_j
                const uint4 mw = *reinterpret_cast<const uint4 *>(ws.smask(st) + lane * kMaskWords);
                const uint32_t wds[4] = {mw.x, mw.y, mw.z, mw.w};
                const E *vp = ws.svals(st) + lane;
                const long t_tok = t0 + lane;
                int pos = 0;
#pragma unroll 1
                for (int j = 0; j < kD; ++j) {
                    float x;
                    if ((wds[j >> 5] >> (j & 31)) & 1u) {
                        x = Elem<E>::to_f(vp[min(pos, a.T - 1) * kWT]);
                        ++pos;
                    } else {
                        x = sample_score<kF>(a.seed, bh, t_tok, j, f_mu, f_sigma) * ws.tabc[j];
                    }
                    QVec<G> qv;
                    qv.load(ws.tabq + j * G);
#pragma unroll
                    for (int g = 0; g < G; ++g) s[g] = fmaf(qv.v[g], x, s[g]);
                }
            } else if constexpr (kF == kDegDense) {
                // All 128 channels from the top down, the same for every lane:
                // a kept channel takes this token's next packed value from the
                // end (the table reads of the lanes that keep it are one
                // broadcast), a pruned one is skipped by predication.  The kept
                // channels meet the FMAs in the same order as in the walk
                // below, so the scores are bit-identical to the walk's.  A mask
                // with more bits than value slots (a cache never written by
                // spark_prune, or a lane past n) reads nothing.
                const uint4 mw = *reinterpret_cast<const uint4 *>(ws.smask(st) + lane * kMaskWords);
                const int cnt = __popc(mw.x) + __popc(mw.y) + __popc(mw.z) + __popc(mw.w);
                const bool ok = cnt <= a.T;
                const uint32_t wds[4] = {ok ? mw.x : 0u, ok ? mw.y : 0u, ok ? mw.z : 0u, ok ? mw.w : 0u};
                const E *vp = ws.svals(st) + lane + (ok && cnt > 0 ? cnt - 1 : 0) * kWT;
                float2 s2[G / 2 > 0 ? G / 2 : 1];
#pragma unroll
                for (int g = 0; g < (G / 2 > 0 ? G / 2 : 1); ++g) s2[g] = make_float2(0.f, 0.f);
#pragma unroll
                for (int wi = 3; wi >= 0; --wi) {
                    const uint32_t w = wds[wi];
#pragma unroll
                    for (int b4 = 7; b4 >= 0; --b4) {
                        // c_j of four channels in one broadcast read
                        const float4 c4 = *reinterpret_cast<const float4 *>(ws.tabc + 32 * wi + 4 * b4);
                        const float cc[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
                        for (int u = 3; u >= 0; --u) {
                            const int b = 4 * b4 + u;
                            const int j = 32 * wi + b;
                            if ((w >> b) & 1u) {  // predicated, no branch
                                const float x = Elem<E>::to_f(*vp) - cc[u];
                                vp -= kWT;
                                QVec<G> qv;
                                qv.load(ws.tabq + j * G);
                                if constexpr (G % 2 == 0) {
                                    const float2 x2 = make_float2(x, x);
#pragma unroll
                                    for (int g = 0; g < G; g += 2)
                                        s2[g / 2] = __ffma2_rn(make_float2(qv.v[g], qv.v[g + 1]), x2, s2[g / 2]);
                                } else {
#pragma unroll
                                    for (int g = 0; g < G; ++g) s[g] = fmaf(qv.v[g], x, s[g]);
                                }
                            }
                        }
                    }
                }
                if constexpr (G % 2 == 0) {
#pragma unroll
                    for (int g = 0; g < G; g += 2) {
                        s[g] = s2[g / 2].x;
                        s[g + 1] = s2[g / 2].y;
                    }
                }
            } else if (a.T > 0) {
                // Walk the T set bits of the 128-bit mask from the top channel
                // down, pairing the i-th bit from the top with the i-th packed
                // value from the end.  The non-empty mask words are queued in
                // descending order first (cur, n1, n2, n3, with their channel
                // bases as the bytes of bq), so every step is branch-free:
                // find the top bit, clear it, and move to the next queued word
                // once the current one is used up.  All lanes run exactly T
                // steps.  A mask with fewer than T bits (a cache never written
                // by spark_prune, or a lane past n) keeps every index in range.
                const uint4 mw = *reinterpret_cast<const uint4 *>(ws.smask(st) + lane * kMaskWords);
                uint32_t cur = mw.w, n1 = mw.z, n2 = mw.y, n3 = mw.x;
                uint32_t bq = 0x00204060u;  // bases 96, 64, 32, 0 from the low byte up
                queue_nonempty(cur, n1, n2, n3, bq);
                const E *vp = ws.svals(st) + lane + (a.T - 1) * kWT;
                float2 s2[G / 2 > 0 ? G / 2 : 1];  // head pairs: packed fp32x2 FMAs
#pragma unroll
                for (int g = 0; g < (G / 2 > 0 ? G / 2 : 1); ++g) s2[g] = make_float2(0.f, 0.f);
#pragma unroll 8  // 8 measured 1-2 % faster than 4 on the long decode, 2 slower
                for (int i = 0; i < a.T; ++i) {
                    const uint32_t pos = bit_top(cur);        // 0xffffffff when cur == 0
                    const int j = (int)((bq | pos) & (uint32_t)(kD - 1));
                    cur &= bit_mask_below(pos);  // clear the top bit
                    const bool e = cur == 0u;
                    cur = e ? n1 : cur;
                    n1 = e ? n2 : n1;
                    n2 = e ? n3 : n2;
                    bq = e ? (bq >> 8) : bq;
                    const float x = Elem<E>::to_f(vp[-i * kWT]) - ws.tabc[j];
                    QVec<G> qv;
                    qv.load(ws.tabq + j * G);
                    if constexpr (G % 2 == 0) {
                        const float2 x2 = make_float2(x, x);
#pragma unroll
                        for (int g = 0; g < G; g += 2)
                            s2[g / 2] = __ffma2_rn(make_float2(qv.v[g], qv.v[g + 1]), x2, s2[g / 2]);
                    } else {
#pragma unroll
                        for (int g = 0; g < G; ++g) s[g] = fmaf(qv.v[g], x, s[g]);
                    }
                }
                if constexpr (G % 2 == 0) {
#pragma unroll
                    for (int g = 0; g < G; g += 2) {
                        s[g] = s2[g / 2].x;
                        s[g + 1] = s2[g / 2].y;
                    }
                }
            }
            if constexpr (kPV) {
                // expand the pruned values into the swizzled V tile: each lane
                // builds its token's row 8 channels (16 bytes) at a time, top
                // channel first, a kept channel taking the token's next packed
                // value from the end and a pruned one 0, and stores every
                // chunk (the swizzle keeps the warp's 16-byte stores free of
                // bank conflicts); a lane past n, or a mask with more bits
                // than Tv, writes a zero row
                const uint4 mw = *reinterpret_cast<const uint4 *>(ws.svmask(st) + lane * kMaskWords);
                const int cnt = __popc(mw.x) + __popc(mw.y) + __popc(mw.z) + __popc(mw.w);
                const bool ok = valid && cnt <= a.Tv;
                const uint32_t wds[4] = {ok ? mw.x : 0u, ok ? mw.y : 0u, ok ? mw.z : 0u, ok ? mw.w : 0u};
                const uint16_t *vp = reinterpret_cast<const uint16_t *>(ws.svvals(st)) + lane +
                                     (ok && cnt > 0 ? cnt - 1 : 0) * kWT;
                const uint32_t vrow = smem_u32(ws.vt);
#pragma unroll
                for (int wi = 3; wi >= 0; --wi) {
                    const uint32_t w = wds[wi];
#pragma unroll
                    for (int c8 = 3; c8 >= 0; --c8) {
                        uint32_t h[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                        for (int u = 7; u >= 0; --u) {
                            if ((w >> (8 * c8 + u)) & 1u) {  // predicated, no branch
                                h[u >> 1] |= (uint32_t)*vp << (16 * (u & 1));
                                vp -= kWT;
                            }
                        }
                        const uint32_t adr = vrow + vswz(lane, 4 * wi + c8);
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(adr), "r"(h[0]), "r"(h[1]),
                                     "r"(h[2]), "r"(h[3])
                                     : "memory");
                    }
                }
            }
            // the stage is read: hand it to the tile nstage ahead
            __syncwarp();
            ++consumed;
            if (ic.item < n_items) {
                if (lane == 0) {
                    fence_proxy_async_smem();
                    issue(st, ic);
                }
                ++issued;
                ++ic.tile;
                settle(ic);
            }
#pragma unroll
            for (int g = 0; g < G; ++g) s[g] = valid ? s[g] + ws.qc[g] : -INFINITY;
            float alpha[G];
            if (tile_softmax<E, G>(ws, f, s, alpha)) pv.rescale(alpha);
            pv.accumulate(ws, vbase + (size_t)t0 * kD, n);
        }
        if (!failed) write_partial<E, G>(a, bh, u, f, pv);
    }

    if (failed) {
        if (lane == 0) {
            atomicOr(a.status, kDevTimeout);
            // let copies already in flight land before the warp exits
            for (int i = consumed; i < issued; ++i)
                (void)mbar_wait_bounded(smem_u32(ws.bars + (int)(i % a.nstage)),
                                        (uint32_t)((i / a.nstage) & 1));
        }
        __syncwarp();
    }
}

// One CTA of kCombineThreads per (row, query head) merges the head's work
// items: the running maxima first (all threads, then a fixed-order tree),
// then warp w sums the items w, w + W, ... (W warps) with weights
// 2^(m_u - M) (lane = 4 channels, 16-byte loads, four items in flight), and
// the warp sums are added in warp order.  Items with l = 0 (empty) weigh 0.
template <int G, int kCombineThreads>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const float *__restrict__ acc,
                                                                  const float *__restrict__ ml, int units,
                                                                  float *__restrict__ out) {
    constexpr int kW = kCombineThreads / 32;
    __shared__ float wmax[kW];
    __shared__ float wl[kW];
    __shared__ float4 wo[kW][32];
    const long row = blockIdx.x;  // (bh, g)
    const long bh = row / G;
    const int g = (int)(row % G);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t base = (size_t)bh * units * G + g;  // item u of this head: base + u * G
    float M = -INFINITY;
    for (int u = tid; u < units; u += kCombineThreads) M = fmaxf(M, ml[(base + (size_t)u * G) * 2]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (lane == 0) wmax[warp] = M;
    __syncthreads();
    M = wmax[0];
#pragma unroll
    for (int w = 1; w < kW; ++w) M = fmaxf(M, wmax[w]);
    float L = 0.f;
    float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
#pragma unroll 4
        for (int u = warp; u < units; u += kW) {
            const size_t r = base + (size_t)u * G;
            const float2 m_l = *reinterpret_cast<const float2 *>(ml + r * 2);
            const float w = m_l.y > 0.f ? exp2f(m_l.x - M) : 0.f;
            const float4 a4 = *reinterpret_cast<const float4 *>(acc + r * kD + 4 * lane);
            L = fmaf(m_l.y, w, L);
            o4.x = fmaf(a4.x, w, o4.x);
            o4.y = fmaf(a4.y, w, o4.y);
            o4.z = fmaf(a4.z, w, o4.z);
            o4.w = fmaf(a4.w, w, o4.w);
        }
    }
    wo[warp][lane] = o4;
    if (lane == 0) wl[warp] = L;
    __syncthreads();
    if (warp == 0) {
        float Ls = 0.f;
        float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kW; ++w) {
            Ls += wl[w];
            s4.x += wo[w][lane].x;
            s4.y += wo[w][lane].y;
            s4.z += wo[w][lane].z;
            s4.w += wo[w][lane].w;
        }
        const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
        *reinterpret_cast<float4 *>(out + row * kD + 4 * lane) =
            make_float4(s4.x * inv, s4.y * inv, s4.z * inv, s4.w * inv);
    }
}

DecodeGeom decode_geometry(long BH, int S, int T, int Tv, int es, int G, int num_sms) {
    DecodeGeom g{};
    const size_t stage = dec_stage_bytes(T, es) + (Tv >= 0 ? dec_stage_bytes(Tv, es) : 0);
    const size_t table = dec_table_bytes(G, es);
    const size_t budget = 227 * 1024;
    const int max_w = dec_max_warps(G);
    auto warps_for = [&](int ns) {
        const size_t wb = (table + ns * stage + 127) / 128 * 128;
        return (int)std::min<size_t>(max_w, budget / wb);
    };
    // a 4-deep ring if all warps still fit, else 3 deep with >= 3/4 of them
    // unless 2 deep fits more warps (at T = 64: 11 warps of 2 stages ran
    // 4-7 % faster than 9 of 3), else 2 deep with as many warps as fit
    if (warps_for(4) >= max_w) g.nstage = 4;
    else if (warps_for(3) >= max_w * 3 / 4 && warps_for(3) >= warps_for(2)) g.nstage = 3;
    else g.nstage = 2;
    g.nwarp = std::max(1, warps_for(g.nstage));
    g.warp_bytes = (table + g.nstage * stage + 127) / 128 * 128;
    g.smem = g.warp_bytes * g.nwarp;
    g.ctas = num_sms;

    const long nwt = (long)g.ctas * g.nwarp;
    if (S <= 0 || BH <= 0) {
        g.chunk = kWT;
        g.n_pre = 0;
    } else {
        const long overhead = 128;  // per-item cost in token equivalents
        double best = 1e300;
        for (int w = 1; w <= 512; ++w) {
            long n_pre = std::max(1L, (w * nwt) / BH);
            long chunk = ((S + n_pre - 1) / n_pre + kWT - 1) / kWT * kWT;
            n_pre = (S + chunk - 1) / chunk;
            const long waves = (BH * n_pre + nwt - 1) / nwt;
            const double cost = (double)waves * (double)(chunk + overhead);
            if (cost < best) {
                best = cost;
                g.chunk = (int)chunk;
                g.n_pre = (int)n_pre;
            }
            if (chunk == kWT) break;
        }
    }
    g.units = g.n_pre + 1;
    return g;
}

template <typename E, int G, int kF, bool kPV>
static cudaError_t launch_decode_t(const DecArgs &a0, const DecodeGeom &geo, float *out, cudaStream_t st) {
    DecArgs a = a0;
    a.chunk = geo.chunk;
    a.n_pre = geo.n_pre;
    a.units = geo.units;
    a.nstage = geo.nstage;
    a.nwarp = geo.nwarp;
    a.warp_bytes = geo.warp_bytes;
    auto kern = decode_kernel<E, G, kF, kPV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)geo.smem);
    if (e != cudaSuccess) return e;
    kern<<<geo.ctas, geo.nwarp * 32, geo.smem, st>>>(a);
    // few rows with many items (small batches): more warps per row, so that
    // each warp merges a handful of items
    const long rows = a.BH * G;
    if (rows < 2L * geo.ctas && geo.units > 64)
        combine_kernel<G, 1024><<<(unsigned)rows, 1024, 0, st>>>(a.acc, a.ml, geo.units, out);
    else
        combine_kernel<G, 256><<<(unsigned)rows, 256, 0, st>>>(a.acc, a.ml, geo.units, out);
    return cudaGetLastError();
}

template <typename E, int kF, bool kPV = false>
static cudaError_t dispatch_g(const DecArgs &a, const DecodeGeom &geo, int G, float *out, cudaStream_t st) {
    switch (G) {
    case 1: return launch_decode_t<E, 1, kF, kPV>(a, geo, out, st);
    case 2: return launch_decode_t<E, 2, kF, kPV>(a, geo, out, st);
    case 4: return launch_decode_t<E, 4, kF, kPV>(a, geo, out, st);
    case 8: return launch_decode_t<E, 8, kF, kPV>(a, geo, out, st);
    default: return cudaErrorInvalidValue;
    }
}

// From this many kept channels per token on, the channel-order loop (128
// predicated steps of about 8 instructions, broadcast table reads) beats the
// per-token walk (T steps of about 20, table reads that conflict in
// shared-memory banks): measured 25 % slower at T = 26, 12 % faster at T = 64
// and 27 % at T = 90.
constexpr int kDenseMinT = 48;

template <typename E>
static cudaError_t dispatch_f(const DecArgs &a, const DecodeGeom &geo, int G, int recovery, float *out,
                              cudaStream_t st) {
    switch (recovery) {
    case SPARK_F_DEGENERATE:
        return a.T >= kDenseMinT ? dispatch_g<E, kDegDense>(a, geo, G, out, st)
                                 : dispatch_g<E, SPARK_F_DEGENERATE>(a, geo, G, out, st);
    case SPARK_F_GAUSSIAN: return dispatch_g<E, SPARK_F_GAUSSIAN>(a, geo, G, out, st);
    case SPARK_F_EXPONENTIAL: return dispatch_g<E, SPARK_F_EXPONENTIAL>(a, geo, G, out, st);
    case kRecoveryDegVar: return dispatch_g<E, kDegDense>(a, geo, G, out, st);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode(const void *q, const spark_kcache &kc, const void *v, const spark_kcache *vc,
                          const void *k_tail, const void *v_tail, int tail_cap, int n_tail, int G, int recovery,
                          unsigned long long seed, float *out, void *ws, const DecodeGeom &geo, cudaStream_t st,
                          bool topp) {
    const long BH = (long)kc.B * kc.Hkv;
    if (BH == 0) return cudaSuccess;
    DecArgs a{};
    a.q = q;
    a.mask = kc.mask;
    a.vals = kc.vals;
    a.goff = topp ? kc.goff : nullptr;
    a.lens = kc.lens;
    a.Hkv = kc.Hkv;
    a.qn = kc.qn;
    a.stats = kc.stats;
    a.v = v;
    a.k_tail = k_tail;
    a.v_tail = v_tail;
    a.status = static_cast<uint32_t *>(ws);
    a.acc = reinterpret_cast<float *>(static_cast<char *>(ws) + kWsHeader);
    a.ml = a.acc + (size_t)BH * geo.units * G * kD;
    a.BH = BH;
    a.S = kc.S;
    a.S32 = ((long)kc.S + 31) / 32 * 32;
    a.T = kc.T;
    a.tail_cap = tail_cap;
    a.n_tail = n_tail;
    a.seed = seed;
    if (vc) {  // pruned value cache: bf16, Degenerate F (checked by the caller)
        a.vmask = vc->mask;
        a.vvals = vc->vals;
        a.Tv = vc->T;
        return a.T >= kDenseMinT ? dispatch_g<__nv_bfloat16, kDegDense, true>(a, geo, G, out, st)
                                 : dispatch_g<__nv_bfloat16, SPARK_F_DEGENERATE, true>(a, geo, G, out, st);
    }
    if (kc.dtype == SPARK_BF16) return dispatch_f<__nv_bfloat16>(a, geo, G, recovery, out, st);
    return dispatch_f<float>(a, geo, G, recovery, out, st);
}

}  // namespace spark
