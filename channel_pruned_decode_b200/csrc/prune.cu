// Prefill channel pruning for SparK on sm_100a.
//
// Method: "KV Cache 还能再砍一刀：SparK ..." (paper walkthrough) section 3.1
// (relaxed objective max sum_j w^j z^j with sum_j z^j = T, proxy saliency
// w = ||q^j||_2 * ||k^j||_2, greedy top-T), 3.2 (observation-window queries,
// per-token unstructured mask) and 3.3 step 1 (the cache stores the pruned
// key, the channel mask and the saliency statistics).
//
// spark_prune makes three launches on the caller's stream:
//   qnorm_kernel   one CTA per (row, kv head), one thread per channel: the
//                  fp64 sum of squares over the G*W window rows of the group,
//                  rounded once to fp32.
//   prune_kernel   one CTA per chunk of 256 to 1024 tokens (8 to 32 groups of
//                  32, more for large launches) of one (row, kv head).  Four
//                  lanes own one token (32 channels each): exact fp32 keys
//                  w = qn_j * |k_j| in registers, plus 16-bit search keys
//                  fp16(w * 2^-floor(log2 max qn)), two channels per word.
//                  The fp16 threshold is found by binary lifting over a window
//                  around a running estimate; each probe compares the keys
//                  with packed fp16 compares and counts the results on the
//                  tensor cores (mma.sync against an all-ones operand).  A
//                  probe that leaves exactly T keys fixes the mask; otherwise
//                  the exact fp32 keys are bisected inside the fp16 tie band
//                  and remaining exact ties go to the lower channel by a scan
//                  across the quad.  Kept values are staged per warp in the
//                  32-token interleaved layout and written back with 16-byte
//                  stores; fp32 partial sums of the pruned saliencies go to
//                  fp64 per-lane accumulators and one fp64 partial per CTA.
//   stats_kernel   fixed-order fp64 sum of the CTA partials per head, then
//                  N = S*(D-T) and mu_pruned = sum w / N.
// All reductions have a fixed order, so reruns are bit-identical.  SparK-g
// uses prune_kernel with per-group selections: with four groups of 32
// channels the quad's lanes exchange their 16-bit keys through shared memory
// so that lane s searches group s, all four groups at once, with per-lane
// tensor-core counts; other group counts search the groups one after the
// other over the whole quad.  SparK-p (per-token top-p selection) has its own
// kernel, prune_topp_kernel, described with it below.
#include "spark_internal.cuh"

#include <cuda_fp16.h>

namespace spark {

// Four-group key exchange rows (u16 units): group q's 32 keys at kXGroup * q,
// one row per token, rows kXRow apart.  Rows 100 words apart put the 8 tokens
// of a warp in distinct bank quadruples, and groups 24 words apart keep each
// 8-lane phase of the 16-byte reads back free of bank conflicts.
constexpr int kXGroup = 48, kXRow = 200;

// Four-group SparK-g: where each channel's key goes in the exchange row, per
// (row, kv head), from the head's window-query norms; the groups are those of the other modes (rank by
// qn desc, channel asc; group q holds the ranks [32q, 32q + 32)), and a
// channel's slot is kXGroup * group + j with j < 32.  Step c of the scatter
// writes channels c, 32 + c, 64 + c and 96 + c of the warp's 8 tokens; with
// the row stride above it is free of bank conflicts exactly when those four
// channels' words j / 2 differ mod 4 (call j / 2 mod 4 the slot's colour:
// each group has 8 slots of each colour).  Colour = quarter c / 32 makes
// every step conflict-free but may give a group more than 8 channels of a
// colour; swaps of two channels' colours within one step (still distinct)
// then even the groups out, each time the swap that lowers the total excess
// most (first by step, then by pair).  Channels take their colour's slots in
// channel order, and whatever excess is left takes the free slots.  Only the
// bank pattern of the exchange depends on this order, not the result.
// Called by all kD threads of a CTA, thread c holding channel c's norm in
// q[c] (shared); writes the head's kD slots to `out`.
__device__ __forceinline__ void build_group_slots(const float *q, uint8_t *__restrict__ out) {
    __shared__ uint8_t gid[kD], col[kD], slot[kD];
    __shared__ int cnt[4][4];
    const int c = threadIdx.x;
    if (c < 16) cnt[c >> 2][c & 3] = 0;
    __syncthreads();
    {
        const float qc = q[c];
        int rank = 0;
        for (int i = 0; i < kD; ++i) rank += (q[i] > qc || (q[i] == qc && i < c)) ? 1 : 0;
        gid[c] = (uint8_t)(rank >> 5);
        col[c] = (uint8_t)(c >> 5);
        atomicAdd(&cnt[rank >> 5][c >> 5], 1);
    }
    __syncthreads();
    if (c < 32) {  // warp 0 orders the slots (warp-uniform branch); lane = step
        const int lane = c;
        for (int it = 0; it < 64; ++it) {
            int best = 0, bx = 0, by = 0;
            for (int a = 0; a < 4; ++a)
                for (int b = a + 1; b < 4; ++b) {
                    const int x = 32 * a + lane, y = 32 * b + lane;
                    const int gx = gid[x], gy = gid[y], cx = col[x], cy = col[y];
                    if (gx == gy) continue;  // same group: the counts do not change
                    const int before = abs(cnt[gx][cx] - 8) + abs(cnt[gx][cy] - 8) + abs(cnt[gy][cy] - 8) +
                                       abs(cnt[gy][cx] - 8);
                    const int after = abs(cnt[gx][cx] - 9) + abs(cnt[gx][cy] - 7) + abs(cnt[gy][cy] - 9) +
                                      abs(cnt[gy][cx] - 7);
                    if (before - after > best) {
                        best = before - after;
                        bx = x;
                        by = y;
                    }
                }
            const int key = __reduce_max_sync(0xffffffffu, (best << 8) | (255 - lane));
            if ((key >> 8) <= 0) break;  // warp-uniform
            if (lane == 255 - (key & 255)) {
                const int gx = gid[bx], gy = gid[by], cx = col[bx], cy = col[by];
                --cnt[gx][cx];
                ++cnt[gx][cy];
                --cnt[gy][cy];
                ++cnt[gy][cx];
                col[bx] = (uint8_t)cy;
                col[by] = (uint8_t)cx;
            }
            __syncwarp();
        }
        if (lane < 4) {
            const int g = lane;
            uint32_t used = 0u;
            int next[4] = {0, 0, 0, 0};
            for (int ch = 0; ch < kD; ++ch) {
                if (gid[ch] != g) continue;
                const int k = col[ch];
                if (next[k] < 8) {
                    const int i = next[k]++;
                    const int j = 2 * k + (i & 1) + 8 * (i >> 1);  // the slots of colour k
                    used |= 1u << j;
                    slot[ch] = (uint8_t)(kXGroup * g + j);
                } else {
                    slot[ch] = 0xffu;
                }
            }
            for (int ch = 0; ch < kD; ++ch) {
                if (gid[ch] != g || slot[ch] != 0xffu) continue;
                // a group has 32 channels, so a slot is free; NaN norms can
                // break the ranks, and such a group's extra channels share
                // slot 31 (the masks are then unspecified, but every slot
                // stays in its row)
                const int j = used == 0xffffffffu ? 31 : __ffs(~used) - 1;
                used |= 1u << j;
                slot[ch] = (uint8_t)(kXGroup * g + j);
            }
        }
    }
    __syncthreads();
    out[c] = slot[c];
}

// With slots (four-group SparK-g) it also writes the head's exchange slots.
template <typename E>
__global__ void __launch_bounds__(kD) qnorm_kernel(const E *__restrict__ q_obs, int G, int W,
                                                   float *__restrict__ qn, uint8_t *__restrict__ slots) {
    __shared__ float qsh[kD];
    const long bh = blockIdx.x;
    const int j = threadIdx.x;
    const E *base = q_obs + (size_t)bh * G * W * kD + j;
    double acc = 0.0;
    for (int g = 0; g < G; ++g)
        for (int t = 0; t < W; ++t) {
            const double x = (double)Elem<E>::to_f(base[((size_t)g * W + t) * kD]);
            acc = __dadd_rn(acc, __dmul_rn(x, x));  // square of an fp32 value is exact in fp64
        }
    const float q = __double2float_rn(sqrt(acc));
    qn[bh * kD + j] = q;
    if (slots) {  // uniform across the CTA
        qsh[j] = q;
        build_group_slots(qsh, slots + bh * kD);
    }
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
    // (|k_2i|, |k_2i+1|) as fp32
    __device__ __forceinline__ float2 abs_pair(int i) const {
        const uint32_t a = w[i] & 0x7fff7fffu;
        return make_float2(__uint_as_float(a << 16), __uint_as_float(a & 0xffff0000u));
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
    __device__ __forceinline__ float2 abs_pair(int i) const {
        return make_float2(__uint_as_float(w[2 * i] & 0x7fffffffu), __uint_as_float(w[2 * i + 1] & 0x7fffffffu));
    }
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

// fp16x2 a >= b per half: 1.0 / 0.0.  Subnormal halves compare exactly (no
// flush to zero).
__device__ __forceinline__ uint32_t hge2_one(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("set.ge.f16x2.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// fp16x2 a >= b per half: 0xffff / 0x0000.
__device__ __forceinline__ uint32_t hge2_mask(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("set.ge.u32.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// fp16x2 a == b per half: 0xffff / 0x0000.
__device__ __forceinline__ uint32_t heq2_mask(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("set.eq.u32.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// D += A * B for one m16n8k16 fp16 tile with fp16 accumulators.
__device__ __forceinline__ void mma_f16(uint32_t &d0, uint32_t &d1, uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f16.f16.f16.f16 {%0,%1}, {%2,%3,%4,%5}, {%6,%7}, {%0,%1};"
        : "+r"(d0), "+r"(d1)
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Number of the quad's 128 16-bit keys >= the probe p2 (the probe in both
// halves), as an exact fp16 integer.  The 0/1 compare results are the A
// operand of tensor-core tiles whose B operand is all ones: row r of A takes
// its 16 entries from the quad r mod 8 of the warp, so each row sum counts
// keys of one token, and rows r and r + 8 (the two accumulator registers)
// together cover all 128 channels.  Which channel sits in which column is
// irrelevant to a sum.  Every lane of the quad receives the count.
//
// With bsel in place of the all-ones operand (see own_count_operand) each
// lane instead receives the count of its own 32 keys.
constexpr uint32_t kOne2 = 0x3c003c00u;  // fp16 (1, 1)

__device__ __forceinline__ __half count_ge16(const uint32_t (&kp)[16], uint32_t p2, uint32_t bsel = kOne2) {
    uint32_t d0 = 0u, d1 = 0u;
#pragma unroll
    for (int m = 0; m < 4; ++m)
        mma_f16(d0, d1, hge2_one(kp[4 * m + 0], p2), hge2_one(kp[4 * m + 1], p2), hge2_one(kp[4 * m + 2], p2),
                hge2_one(kp[4 * m + 3], p2), bsel, bsel);
    const __half2 c = __hadd2(*reinterpret_cast<const __half2 *>(&d0), *reinterpret_cast<const __half2 *>(&d1));
    return __low2half(c);
}

// B operand that makes count_ge16 a per-lane count.  Columns k = 2s, 2s+1,
// 2s+8, 2s+9 of an A row come from position s of the row's quad; B column
// 2s is one on exactly those rows and every odd column is zero, so output
// column 2s, which lands in the low half of the quad's position-s lane,
// counts that lane's keys alone.  B rows 2s', 2s'+1, 2s'+8, 2s'+9 of column n
// sit in the lane at quad n, position s'.
__device__ __forceinline__ uint32_t own_count_operand(int lane) {
    return (lane >> 2) == 2 * (lane & 3) ? kOne2 : 0u;
}

// Number of the quad's keys >= mid among the channels of `gm` (bit i =
// channel i of this lane's quarter takes part).
__device__ __forceinline__ int quad_count32(const uint32_t (&key)[32], uint32_t mid, uint32_t gm) {
    int c = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) c += (key[i] >= mid && ((gm >> i) & 1u)) ? 1 : 0;
    return quad_sum(c);
}

__device__ __forceinline__ float half_bits_to_float(uint32_t p) {
    return __half2float(__ushort_as_half((unsigned short)p));
}

constexpr uint32_t kTop16 = 0x7c01u;  // above +inf: no key reaches it, never probed
constexpr uint32_t kGallop16 = 256u;  // first gallop step of the fallback search, fp16 units
constexpr int kLift = 11;             // search window 2^11 fp16 units (2 octaves) around the estimate
constexpr int kLiftCold = 12;         // first token of a quad: 2^12 units (4 octaves) below its top key
// one lane per group of 32 channels: the threshold of a few of 32 keys moves
// more from token to token, so the window spans 2 octaves on each side
constexpr int kLiftLane = 12;

// Phase 1 of the selection: the fp16 threshold lo of the T largest 16-bit
// keys.  kp[i] holds the keys of two channels (which two does not matter to
// the counts); the keys are the fp32 keys scaled by a power of two and
// rounded to fp16, which is monotone in the key.  With kOwn false the keys of
// the quad's four lanes are counted together (one token, 128 channels); with
// kOwn true each lane counts its own 32 keys.
//
// Binary lifting over the window [base, base + 2^K): assuming count(>= base)
// >= T, after the probe for bit b, lo is the largest point base + j * 2^b
// with count(>= lo) >= T.  A probe that counts exactly T keys fixes the
// selection (keys >= lo: `exact`), and later probes keep that true, so the
// loop ends as soon as every searcher of the warp has seen one.  Otherwise
// the band of fp16 keys equal to lo holds the boundary and count(>= lo + 1)
// < T; if the window may not have bracketed it (lo never moved, or reached
// the window's top) a gallop + bisection over the whole key range redoes the
// search.  Every loop has a warp-uniform trip count (finished searchers
// idle), so the shuffles and the warp-wide tensor-core counts see the full
// warp.  Keys that must not count are set negative, below every probe.
template <bool kOwn>
__device__ __forceinline__ void search_fp16(const uint32_t (&kp)[16], int T, uint32_t base, int K, bool skip,
                                            uint32_t bsel, uint32_t &lo_out, bool &exact_out) {
    const __half hT = __int2half_rn(T);
    uint32_t lo = base;
    bool exact = skip;  // searchers past the end of the keys take no part
    for (int b = K - 1; b >= 0; --b) {
        const uint32_t p = lo + (1u << b);
        const __half c = count_ge16(kp, p * 0x10001u, kOwn ? bsel : kOne2);
        lo = __hge(c, hT) ? p : lo;
        exact = exact || __heq(c, hT);
        if (__all_sync(0xffffffffu, exact)) break;
    }
    const bool suspect = !exact && (lo == base || lo == base + (1u << K) - 1u);
    if (__any_sync(0xffffffffu, suspect)) {
        // count(>= glo) >= T > count(>= ghi); gallop from lo away from the
        // open side of the bracket (step doubling), then bisect
        uint32_t glo = 0u, ghi = kTop16;
        bool done = !suspect;
        uint32_t step = kGallop16;
        uint32_t mid = min(max(lo, 1u), kTop16 - 1u);
        while (__any_sync(0xffffffffu, !done)) {
            const __half c = count_ge16(kp, mid * 0x10001u, kOwn ? bsel : kOne2);
            const bool ge = __hge(c, hT);
            const bool act = !done;
            glo = (act && ge) ? mid : glo;
            ghi = (act && !ge) ? mid : ghi;
            const bool eq = __heq(c, hT);
            exact = exact || (act && eq);
            done = done || eq || (ghi - glo <= 1u);
            const bool up = ghi == kTop16, down = glo == 0u;
            const uint32_t gal_up = min(glo + step, kTop16 - 1u);
            const uint32_t gal_dn = (uint32_t)max((int)ghi - (int)step, 1);
            const uint32_t bis = glo + ((ghi - glo) >> 1);
            mid = up ? gal_up : (down ? gal_dn : bis);
            step <<= 1;
        }
        // not exact: the bisection ended with ghi = glo + 1
        lo = suspect ? glo : lo;
    }
    lo_out = lo;
    exact_out = exact;
}

constexpr int kBandPicks = 4;  // most one-at-a-time picks from an fp16 band before bisecting instead

// Phase 2: the mask word (32 channels of this lane's quarter) of the T
// largest exact fp32 keys among the quad's channels of gm (bit i = channel i
// of this lane's quarter takes part), ties to the lower channel index, given
// the phase-1 result: m16 = the channels of gm whose fp16 key is >= lo, which
// is the answer when `exact`; otherwise count(fp16 >= lo) >= T > count(fp16
// >= lo + 1).  kp holds the 16-bit keys (channels i and i + 16 in kp[i]).
// Warp-uniform: every lane of the warp calls it.
//
// The fp16 rounding is monotone, so the A keys with an fp16 key above lo are
// all kept and the boundary lies in the band of nb keys whose fp16 key is
// lo: of these the r = T - A largest (equal keys: lower channel first) are
// kept.  Usually the band holds two or three keys, so the kernel picks the r
// largest one at a time when r <= nb - r, or drops the nb - r smallest (equal
// keys: higher channel first) otherwise, each pick a quad max or min and a
// lowest-channel search.  A wider band, more than kBandPicks picks in any
// quad of the warp, takes a bisection over the fp32 bit patterns instead.
__device__ __forceinline__ uint32_t refine_fp32(const uint32_t (&key)[32], const uint32_t (&kp)[16], int T,
                                                int s, float inv_scale, uint32_t lo, bool exact, uint32_t gm,
                                                uint32_t m16) {
    if (!__any_sync(0xffffffffu, !exact)) return m16;
    {
        uint32_t band = 0u;
        const uint32_t lo2 = lo * 0x10001u;
#pragma unroll
        for (int i = 0; i < 16; ++i) band |= heq2_mask(kp[i], lo2) & (0x00010001u << i);
        band = exact ? 0u : band & gm;
        const int above = quad_sum(__popc(m16 & ~band));
        const int nb = quad_sum(__popc(band));
        const int r = T - above;  // 0 < r < nb unless exact
        const bool pmax = 2 * r <= nb;
        const int take = exact ? 0 : (pmax ? r : nb - r);
        const int most = __reduce_max_sync(0xffffffffu, take);
        if (most <= kBandPicks) {
            uint32_t cand = band, picked = 0u;
            for (int it = 0; it < most; ++it) {
                uint32_t mx = 0u, mn = 0xffffffffu;  // keys are non-negative: u32 order is fp32 order
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    if ((cand >> i) & 1u) {
                        mx = max(mx, key[i]);
                        mn = min(mn, key[i]);
                    }
                }
#pragma unroll
                for (int o = 1; o <= 2; o <<= 1) {
                    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                }
                const uint32_t ext = pmax ? mx : mn;
                uint32_t eqm = 0u;
#pragma unroll
                for (int i = 0; i < 32; ++i) eqm |= (key[i] == ext ? 1u : 0u) << i;
                eqm = it < take ? eqm & cand : 0u;
                // the pick: lowest channel of the quad for a max, highest for a min
                const int order = pmax ? s : 3 - s;
                int first = eqm ? order : 4;
                first = min(first, __shfl_xor_sync(0xffffffffu, first, 1));
                first = min(first, __shfl_xor_sync(0xffffffffu, first, 2));
                if (eqm && order == first) {
                    const uint32_t bit = pmax ? (eqm & (0u - eqm)) : (0x80000000u >> __clz(eqm));
                    picked |= bit;
                    cand &= ~bit;
                }
            }
            if (exact) return m16;
            return pmax ? ((m16 & ~band) | picked) : (m16 & ~picked);
        }
    }
    const uint32_t hi = lo + 1u;

    // With v = the fp16 value of lo - 1 and u that of hi = lo + 1, every key
    // whose fp16 key is >= lo is > v / scale, and every key >= u / scale has
    // an fp16 key >= hi, so [v / scale, u / scale) in fp32 bit patterns
    // brackets the T-th largest key.
    uint32_t lo32 = lo == 0u ? 0u : __float_as_uint(half_bits_to_float(lo - 1u) * inv_scale);
    uint32_t hi32 = hi >= kTop16 ? 0x7f800001u : __float_as_uint(half_bits_to_float(hi) * inv_scale);
    {
        // Narrow the bracket to the keys inside it: with no key in [lo32,
        // kmin) or (kmax, hi32), count(>= kmin) = count(>= lo32) >= T and
        // count(>= kmax + 1) = count(>= hi32) < T.  A band of equal keys
        // (bf16 values under unit norms are exact in fp16) leaves a bracket
        // one wide, and the tie scan below settles it.
        uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const bool in = ((gm >> i) & 1u) && (key[i] - lo32 < hi32 - lo32);
            kmin = in ? min(kmin, key[i]) : kmin;
            kmax = in ? max(kmax, key[i]) : kmax;
        }
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
            kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
            kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
        }
        if (!exact && kmax >= kmin) {
            lo32 = kmin;
            hi32 = kmax + 1u;
        }
    }
    bool exact32 = exact;
    bool done2 = exact || (hi32 - lo32 <= 1u);
    while (__any_sync(0xffffffffu, !done2)) {
        const uint32_t mid32 = lo32 + ((hi32 - lo32) >> 1);
        const int c = quad_count32(key, mid32, gm);
        if (!done2) {
            if (c >= T) {
                lo32 = mid32;
                if (c == T) { exact32 = true; done2 = true; }
            } else {
                hi32 = mid32;
            }
            if (hi32 - lo32 <= 1u) done2 = true;
        }
    }
    // exact32: exactly T keys are >= lo32.  Otherwise lo32 is the T-th
    // largest key: the keys above it are kept, and of the keys equal to it the
    // first T - (number above) in channel order over the quad.
    const uint32_t thr = exact32 ? lo32 : lo32 + 1u;
    uint32_t m32 = 0u;
#pragma unroll
    for (int i = 0; i < 32; ++i) m32 |= (key[i] >= thr ? 1u : 0u) << i;
    m32 &= gm;
    if (__any_sync(0xffffffffu, !exact32)) {  // warp-uniform: the scans below shuffle
        const int above = quad_sum(__popc(m32));
        int e = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) e += (key[i] == lo32 && ((gm >> i) & 1u)) ? 1 : 0;
        int r = quad_excl_scan(e, s);
        if (!exact32) {
            const int need = T - above;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if (key[i] == lo32 && ((gm >> i) & 1u)) {
                    if (r < need) m32 |= 1u << i;
                    ++r;
                }
            }
        }
    }
    return exact ? m16 : m32;
}

// fp16 decision of one quarter: bit i of the word = channel i, set where the
// channel's 16-bit key is >= its threshold.  p2[i] holds the thresholds of
// channels (i, i + 16), the layout of kp.
__device__ __forceinline__ uint32_t decide_fp16(const uint32_t (&kp)[16], const uint32_t (&p2)[16]) {
    uint32_t m = 0u;
#pragma unroll
    for (int i = 0; i < 16; ++i) m |= hge2_mask(kp[i], p2[i]) & (0x00010001u << i);
    return m;
}

// Mask word (32 channels) of this lane's quarter of the token: the T largest
// exact fp32 keys over the quad's channels of gm, ties to the lower channel
// index.  0 < T < 128.  kp[i] holds the 16-bit keys of channels i (low half)
// and i + 16 (high half); the caller sets the keys of channels outside gm
// negative.
__device__ __forceinline__ uint32_t select_top_t(const uint32_t (&key)[32], const uint32_t (&kp)[16], int T,
                                                 int s, float inv_scale, uint32_t base, int K, bool skip,
                                                 uint32_t gm, uint32_t &tau) {
    uint32_t lo;
    bool exact;
    search_fp16<false>(kp, T, base, K, skip, kOne2, lo, exact);
    tau = lo;
    uint32_t p2[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) p2[i] = lo * 0x10001u;
    return refine_fp32(key, kp, T, s, inv_scale, lo, exact, gm, decide_fp16(kp, p2));
}

// SparK-g groups: number of groups and each group's kept-channel budget.
struct GroupArgs {
    int n;
    int T[kMaxGroups];
};

// prune_kernel modes: one top-T selection per token; SparK-g with any number
// of groups, searched one after the other over the whole quad; SparK-g with
// four groups of 32 channels, one group per lane of the quad.
constexpr int kModePlain = 0, kModeGroups = 1, kModeLaneGroups = 2;

template <typename E, int kMode>
__global__ void __launch_bounds__(kPruneThreads, 4)
    prune_kernel(const E *__restrict__ k, const float *__restrict__ qn, uint32_t *__restrict__ mask,
                 E *__restrict__ vals, double *__restrict__ partial, int S, int T, int n_chunks, int gpc,
                 GroupArgs ga, const int32_t *__restrict__ lens, int Hkv, uint32_t *__restrict__ status,
                 const uint8_t *__restrict__ slots) {
    using Raw = typename RawT<E>::type;
    constexpr bool kGrouped = kMode != kModePlain, kLane = kMode == kModeLaneGroups;
    // per-warp staging of the kept values: [kept index][8 tokens of the warp]
    __shared__ __align__(16) Raw vtile[kPruneThreads / 32][kD * 8];
    __shared__ double red[2][kPruneThreads / 32];
    __shared__ uint32_t qmax[kPruneThreads / 32];
    // window-query norms of this head, one padded row per quarter (stride 36
    // floats): the 4 quarters' 16-byte reads fall in distinct banks
    __shared__ __align__(16) float qs[4 * 36];

    const long bh = blockIdx.x / n_chunks;
    const int chunk = blockIdx.x % n_chunks;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int s = lane & 3;                 // quarter: channels [32s, 32s+32)
    const int tq = lane >> 2;               // token within the warp's 8
    const int tl = warp * 8 + tq;           // token within the 32-token group
    const long S32 = ((long)S + 31) / 32 * 32;
    const int Sb = row_len(lens, bh, Hkv, S, tid == 0 ? status : nullptr);  // tokens of this row (S: its stride)

    // the 16-bit keys are fp16(key * scale), scale = 2^-floor(log2 max_j qn_j),
    // so the largest window-query norm maps into [1, 2) and the keys of
    // ordinary keys sit in fp16's normal range
    {
        const float q = __ldg(qn + bh * kD + tid);  // kPruneThreads == kD
        qs[(tid >> 5) * 36 + (tid & 31)] = q;
        const uint32_t mx = __reduce_max_sync(0xffffffffu, __float_as_uint(q) & 0x7fffffffu);
        if (lane == 0) qmax[warp] = mx;
    }
    __syncthreads();
    float scale = 1.f, inv_scale = 1.f;
    {
        uint32_t mx = qmax[0];
#pragma unroll
        for (int w = 1; w < kPruneThreads / 32; ++w) mx = max(mx, qmax[w]);
        const int e = (int)(mx >> 23);
        if (e > 0 && e < 255) {
            const int x = min(max(127 - e, -64), 64);
            scale = __uint_as_float((uint32_t)(127 + x) << 23);
            inv_scale = __uint_as_float((uint32_t)(127 - x) << 23);
        }
    }
    const float2 scale2 = make_float2(scale, scale);

    // SparK-g: channel groups by window-query norm rank (equal norms: lower
    // channel first; group q holds ranks [q*D/n, (q+1)*D/n)).  Per group and
    // quarter: the channel bit mask and the 16 select words that keep the
    // group's halves of the packed 16-bit keys.
    __shared__ uint8_t sgid[kGrouped ? kD : 1];
    __shared__ uint32_t gmask[kGrouped ? kMaxGroups : 1][4];
    __shared__ __align__(16) uint32_t gsel[kMode == kModeGroups ? kMaxGroups : 1][4][16];
    __shared__ int gT[kGrouped ? kMaxGroups : 1];
    __shared__ uint32_t staus[kMode == kModeGroups ? kMaxGroups : 1][kPruneThreads];  // per-lane estimates
    // Four groups: each quarter scatters its 16-bit keys into a per-warp
    // exchange row per token in group order (the slots of build_group_slots),
    // and lane s reads group s back with four 16-byte loads.
    __shared__ __align__(16) uint16_t xkeys[kLane ? kPruneThreads / 32 : 1][kLane ? 8 * kXRow : 1];
    // per lane: the shared address of each of its quarter's 32 channels in
    // its token's exchange row, [channel / 4][thread] (conflict-free reads)
    __shared__ __align__(16) uint4 xaddr[kLane ? 8 : 1][kLane ? kPruneThreads : 1];
    // per quarter: byte selectors that build the threshold pair of kp[i]
    // (groups of channels i and i + 16) from the four group thresholds
    __shared__ __align__(16) uint32_t psel[kLane ? 4 : 1][16];
    __shared__ uint8_t sslot[kLane ? kD : 1];
    if constexpr (kGrouped) {
        if constexpr (kLane) {
            const uint8_t sl = __ldg(slots + bh * kD + tid);
            sslot[tid] = sl;
            sgid[tid] = (uint8_t)(sl / kXGroup);
        } else {
            const float qj = qs[(tid >> 5) * 36 + (tid & 31)];
            int rank = 0;
            for (int i = 0; i < kD; ++i) {
                const float qi = qs[(i >> 5) * 36 + (i & 31)];
                rank += (qi > qj || (qi == qj && i < tid)) ? 1 : 0;
            }
            int gq = 0;
            for (int q = 1; q < ga.n; ++q) gq += rank >= q * kD / ga.n ? 1 : 0;
            sgid[tid] = (uint8_t)gq;
        }
        if (tid < kMaxGroups) gT[tid] = tid < ga.n ? ga.T[tid] : 0;
        __syncthreads();
        if constexpr (!kLane) {
            for (int e = tid; e < ga.n * 64; e += kPruneThreads) {
                const int q = e >> 6, qs4 = (e >> 4) & 3, i = e & 15;
                gsel[q][qs4][i] = (sgid[32 * qs4 + i] == q ? 0x0000ffffu : 0u) |
                                  (sgid[32 * qs4 + i + 16] == q ? 0xffff0000u : 0u);
            }
        }
        if (tid < ga.n * 4) {
            const int q = tid >> 2, qs4 = tid & 3;
            uint32_t b = 0u;
            for (int c = 0; c < 32; ++c) b |= (sgid[32 * qs4 + c] == q ? 1u : 0u) << c;
            gmask[q][qs4] = b;
        }
        __syncthreads();
        if constexpr (kLane) {
            const uint32_t row = (uint32_t)__cvta_generic_to_shared(&xkeys[warp][(lane >> 2) * kXRow]);
            const int s4 = lane & 3;
#pragma unroll
            for (int ii = 0; ii < 8; ++ii) {
                uint32_t a[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) a[e] = row + 2u * sslot[32 * s4 + 4 * ii + e];
                xaddr[ii][tid] = make_uint4(a[0], a[1], a[2], a[3]);
            }
            if (tid < 64) {
                const int qs4 = tid >> 4, i = tid & 15;
                const uint32_t ql = sgid[32 * qs4 + i], qh = sgid[32 * qs4 + i + 16];
                psel[qs4][i] = (2u * ql) | (2u * ql + 1u) << 4 | (2u * qh) << 8 | (2u * qh + 1u) << 12;
            }
            __syncthreads();
        }
    }

    Raw *vt = vtile[warp];
    uint32_t tau = 1u;
    const uint32_t bsel = own_count_operand(lane);  // four-group mode: per-lane counts
    double acc_w = 0.0, acc_w2 = 0.0;
    const long g_first = (long)chunk * gpc;
    const E *krow = k + ((size_t)bh * S + g_first * 32 + tl) * kD + 32 * s;  // this lane's slice, group 0
    E *gvals = vals + (size_t)bh * S32 * T + (size_t)g_first * 32 * T;      // group 0's values

    // one 32-token group: select, write the mask, stage and store the kept
    // values, accumulate the pruned-saliency sums.  `cur` holds this group's
    // slice; the next group's slice is loaded into `nxt` first.
    auto group = [&](int gi, KSlice<E> &cur, KSlice<E> &nxt) {
        const long t = (g_first + gi) * 32 + tl;
        const bool valid = t < Sb;
        if (gi + 1 < gpc && t + 32 < Sb) nxt.load(krow + (size_t)(gi + 1) * 32 * kD);
        else nxt.zero();

        // exact fp32 saliency keys w_j = qn_j * |k_j| (packed fp32 multiplies,
        // each rounded like a scalar one), and their scaled copies
        uint32_t key[32];
        float2 wsc[16];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float4 q4 = *reinterpret_cast<const float4 *>(qs + s * 36 + 4 * c);
            const float2 w01 = __fmul2_rn(make_float2(q4.x, q4.y), cur.abs_pair(2 * c));
            const float2 w23 = __fmul2_rn(make_float2(q4.z, q4.w), cur.abs_pair(2 * c + 1));
            key[4 * c + 0] = __float_as_uint(w01.x);
            key[4 * c + 1] = __float_as_uint(w01.y);
            key[4 * c + 2] = __float_as_uint(w23.x);
            key[4 * c + 3] = __float_as_uint(w23.y);
            wsc[2 * c] = __fmul2_rn(w01, scale2);
            wsc[2 * c + 1] = __fmul2_rn(w23, scale2);
        }
        uint32_t m;
        if (T <= 0) {
            m = 0u;
        } else if (T >= kD) {
            m = 0xffffffffu;
        } else {
            // 16-bit keys of channels (i, i + 16)
            uint32_t kp[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float a = (i & 1) ? wsc[i >> 1].y : wsc[i >> 1].x;
                const float b = (i & 1) ? wsc[8 + (i >> 1)].y : wsc[8 + (i >> 1)].x;
                const __half2 h = __floats2half2_rn(a, b);
                kp[i] = *reinterpret_cast<const uint32_t *>(&h);
            }
            // one top-Tq selection over the channels of gm, with its own
            // running threshold estimate tq
            auto select_with = [&](const uint32_t(&kq)[16], int Tq, uint32_t gm, uint32_t &tq) -> uint32_t {
                uint32_t base;
                int K;
                if (gi == 0) {
                    // first token of this quad: the window ends at its largest
                    // key (negative keys of channels outside gm count as 0)
                    __half2 mx = *reinterpret_cast<const __half2 *>(&kq[0]);
#pragma unroll
                    for (int i = 1; i < 16; ++i) mx = __hmax2(mx, *reinterpret_cast<const __half2 *>(&kq[i]));
                    const uint32_t mb = *reinterpret_cast<const uint32_t *>(&mx);
                    const uint32_t l16 = mb & 0xffffu, h16 = mb >> 16;
                    uint32_t m16 = max((l16 & 0x8000u) ? 0u : l16, (h16 & 0x8000u) ? 0u : h16);
                    m16 = max(m16, __shfl_xor_sync(0xffffffffu, m16, 1));
                    m16 = max(m16, __shfl_xor_sync(0xffffffffu, m16, 2));
                    K = kLiftCold;
                    base = m16 > (1u << K) - 1u ? m16 - ((1u << K) - 1u) : 0u;
                } else {
                    // later tokens: centred on the running threshold estimate
                    K = kLift;
                    base = tq > (1u << (K - 1)) ? tq - (1u << (K - 1)) : 0u;
                }
                base = min(base, kTop16 - (1u << K));
                uint32_t lo;
                uint32_t mm = select_top_t(key, kq, Tq, s, inv_scale, base, K, !valid, gm, lo);
                mm = valid ? mm : 0u;
                // next estimate: running mean of this quad's thresholds
                tq = gi == 0 ? lo : (uint32_t)((int)tq + (((int)lo - (int)tq) >> 1));
                tq = valid ? tq : 1u;
                return mm;
            };
            if constexpr (!kGrouped) {
                m = select_with(kp, T, 0xffffffffu, tau);
            } else if constexpr (kLane) {
                // scatter this quarter's 16-bit keys into the token's exchange
                // row, then read back group s (32 keys, two per word)
                __syncwarp();
#pragma unroll
                for (int ii = 0; ii < 8; ++ii) {
                    const uint4 a = xaddr[ii][tid];
                    const uint32_t av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c = 4 * ii + e;
                        const uint32_t h = c < 16 ? kp[c] : (kp[c - 16] >> 16);
                        asm volatile("st.shared.u16 [%0], %1;" ::"r"(av[e]), "h"((unsigned short)h) : "memory");
                    }
                }
                __syncwarp();
                uint32_t kg[16];
                {
                    const uint32_t src =
                        (uint32_t)__cvta_generic_to_shared(&xkeys[warp][tq * kXRow + kXGroup * s]);
#pragma unroll
                    for (int i4 = 0; i4 < 4; ++i4)
                        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                                     : "=r"(kg[4 * i4]), "=r"(kg[4 * i4 + 1]), "=r"(kg[4 * i4 + 2]),
                                       "=r"(kg[4 * i4 + 3])
                                     : "r"(src + 16u * i4)
                                     : "memory");
                }
                // this lane's group: top Tq of its 32 keys
                const int Tq = gT[s];
                const bool triv = Tq <= 0 || Tq >= 32;
                uint32_t base;
                int K;
                if (gi == 0) {
                    __half2 mx = *reinterpret_cast<const __half2 *>(&kg[0]);
#pragma unroll
                    for (int i = 1; i < 16; ++i) mx = __hmax2(mx, *reinterpret_cast<const __half2 *>(&kg[i]));
                    const uint32_t mb = *reinterpret_cast<const uint32_t *>(&mx);
                    const uint32_t m16 = max(mb & 0xffffu, mb >> 16);
                    K = kLiftCold;
                    base = m16 > (1u << K) - 1u ? m16 - ((1u << K) - 1u) : 0u;
                } else {
                    K = kLiftLane;
                    base = tau > (1u << (K - 1)) ? tau - (1u << (K - 1)) : 0u;
                }
                base = min(base, kTop16 - (1u << K));
                uint32_t lo;
                bool ex;
                search_fp16<true>(kg, Tq, base, K, !valid || triv, bsel, lo, ex);
                if (!triv) tau = gi == 0 ? lo : (uint32_t)((int)tau + (((int)lo - (int)tau) >> 1));
                tau = valid ? tau : 1u;
                if (triv) {
                    lo = Tq <= 0 ? kTop16 : 0u;  // kTop16 is a NaN pattern: no key compares >= it
                    ex = true;
                }
                // the four groups' thresholds (bit 15: boundary inside the fp16
                // band) to every lane of the quad, then the fp16 decision with
                // each channel's own group threshold
                const uint32_t v = lo | (ex ? 0u : 0x8000u);
                const uint32_t w1 = __shfl_xor_sync(0xffffffffu, v, 1);
                const uint32_t pr = (s & 1) ? (w1 | (v << 16)) : (v | (w1 << 16));
                const uint32_t ot = __shfl_xor_sync(0xffffffffu, pr, 2);
                const uint32_t P01 = (s & 2) ? ot : pr, P23 = (s & 2) ? pr : ot;
                const uint32_t T01 = P01 & 0x7fff7fffu, T23 = P23 & 0x7fff7fffu;
                uint32_t p2[16];
                {
                    const uint4 *ps = reinterpret_cast<const uint4 *>(psel[s]);
#pragma unroll
                    for (int i4 = 0; i4 < 4; ++i4) {
                        const uint4 sv = ps[i4];
                        p2[4 * i4 + 0] = __byte_perm(T01, T23, sv.x);
                        p2[4 * i4 + 1] = __byte_perm(T01, T23, sv.y);
                        p2[4 * i4 + 2] = __byte_perm(T01, T23, sv.z);
                        p2[4 * i4 + 3] = __byte_perm(T01, T23, sv.w);
                    }
                }
                m = decide_fp16(kp, p2);
                // exact fp32 phase for the groups whose fp16 band holds the
                // boundary, on the quad's channels of that group
                const uint32_t nex =
                    ((P01 >> 15) & 1u) | ((P01 >> 30) & 2u) | ((P23 >> 13) & 4u) | ((P23 >> 28) & 8u);
                const uint32_t any_nex = __reduce_or_sync(0xffffffffu, nex);
#pragma unroll 1
                for (int q = 0; q < 4; ++q) {
                    if (!((any_nex >> q) & 1u)) continue;  // warp-uniform
                    const uint32_t gm = gmask[q][s];
                    const uint32_t lq = ((q < 2 ? T01 : T23) >> (16 * (q & 1))) & 0xffffu;
                    const uint32_t mq = refine_fp32(key, kp, gT[q], s, inv_scale, lq, !((nex >> q) & 1u), gm, m & gm);
                    m = (m & ~gm) | mq;
                }
                m = valid ? m : 0u;
            } else {
                m = 0u;
#pragma unroll 1
                for (int q = 0; q < ga.n; ++q) {
                    const int Tq = gT[q];
                    const int sz = (q + 1) * kD / ga.n - q * kD / ga.n;
                    const uint32_t gm = gmask[q][s];
                    if (Tq <= 0) continue;  // uniform: kernel arguments
                    if (Tq >= sz) {
                        m |= gm;
                        continue;
                    }
                    uint32_t kq[16];
                    const uint4 *sel4 = reinterpret_cast<const uint4 *>(&gsel[q][s][0]);
#pragma unroll
                    for (int i4 = 0; i4 < 4; ++i4) {
                        const uint4 v = sel4[i4];
                        const uint32_t sv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e)  // members keep their key, others -1.0
                            kq[4 * i4 + e] = (kp[4 * i4 + e] & sv[e]) | (0xbc00bc00u & ~sv[e]);
                    }
                    uint32_t tq = staus[q][tid];
                    m |= select_with(kq, Tq, gm, tq);
                    staus[q][tid] = tq;
                }
            }
        }
        if (valid) mask[((size_t)bh * S + t) * kMaskWords + s] = m;

        // pruned-saliency sums (fp32 over this lane's 32 channels, fp64 across
        // tokens) and the kept values, in ascending channel order, into the
        // warp's staging tile
        Raw *dst = vt + quad_excl_scan(__popc(m), s) * 8 + tq;
        float sw = 0.f, sw2 = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if ((m >> i) & 1u) {
                *dst = (Raw)cur.raw(i);
                dst += 8;
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
        __syncwarp();
        // kept index i of the warp's 8 tokens: 8 * sizeof(E) contiguous bytes
        // of the interleaved layout, in 16-byte pieces
        constexpr int kParts = (int)sizeof(E) / 2;  // 16-byte pieces per row
        unsigned char *g = reinterpret_cast<unsigned char *>(gvals + (size_t)gi * 32 * T + warp * 8);
        const unsigned char *src = reinterpret_cast<const unsigned char *>(vt);
        for (int c = lane; c < T * kParts; c += 32) {
            const int row = c / kParts, part = c % kParts;
            __stcs(reinterpret_cast<uint4 *>(g + (size_t)row * 32 * sizeof(E) + part * 16),
                   *reinterpret_cast<const uint4 *>(src + row * 8 * sizeof(E) + part * 16));
        }
        __syncwarp();
    };

    KSlice<E> ka, kb;
    if (g_first * 32 + tl < Sb) ka.load(krow);
    else ka.zero();
    if constexpr (kLane) {
        // one call site: the four-group body is large enough that a second
        // inlined copy no longer fits the instruction cache
#pragma unroll 1
        for (int gi = 0; gi < gpc; ++gi) {
            if ((g_first + gi) * 32 >= Sb) break;  // uniform across the CTA
            group(gi, ka, kb);
            ka = kb;
        }
    } else {
        for (int gi = 0; gi < gpc; gi += 2) {
            if ((g_first + gi) * 32 >= Sb) break;  // uniform across the CTA
            group(gi, ka, kb);
            if ((g_first + gi + 1) * 32 >= Sb) break;
            group(gi + 1, kb, ka);
        }
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
                             double *__restrict__ stats, const int32_t *__restrict__ lens, int Hkv) {
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
        const double n = (double)row_len(lens, bh, Hkv, S, nullptr) * (double)(kD - T);
        stats[bh * 4 + 0] = n;
        stats[bh * 4 + 1] = a;
        stats[bh * 4 + 2] = b;
        stats[bh * 4 + 3] = n > 0.0 ? a / n : 0.0;
    }
}

template <typename E>
static cudaError_t launch_prune_t(const void *k, const void *q_obs, int G, int W,
                                  const spark_kcache &kc, void *ws, cudaStream_t st, const GroupArgs *ga) {
    const long BH = (long)kc.B * kc.Hkv;
    if (BH == 0) return cudaSuccess;
    double *partial = reinterpret_cast<double *>(static_cast<char *>(ws) + kWsHeader);
    const bool lane_groups = ga && ga->n == 4 && kD == 128;
    uint8_t *slots = lane_groups ? static_cast<uint8_t *>(ws) + prune_slots_offset(BH, kc.S) : nullptr;
    qnorm_kernel<E><<<(unsigned)BH, kD, 0, st>>>(static_cast<const E *>(q_obs), G, W, kc.qn, slots);
    const int gpc = prune_groups_per_cta(BH, kc.S);
    const int nch = prune_chunks(kc.S, gpc);
    if (nch > 0) {
        if (lane_groups) {
            prune_kernel<E, kModeLaneGroups><<<(unsigned)(BH * nch), kPruneThreads, 0, st>>>(
                static_cast<const E *>(k), kc.qn, kc.mask, static_cast<E *>(kc.vals), partial, kc.S, kc.T,
                nch, gpc, *ga, kc.lens, kc.Hkv, static_cast<uint32_t *>(ws), slots);
        } else if (ga)
            prune_kernel<E, kModeGroups><<<(unsigned)(BH * nch), kPruneThreads, 0, st>>>(
                static_cast<const E *>(k), kc.qn, kc.mask, static_cast<E *>(kc.vals), partial, kc.S, kc.T,
                nch, gpc, *ga, kc.lens, kc.Hkv, static_cast<uint32_t *>(ws), nullptr);
        else
            prune_kernel<E, kModePlain><<<(unsigned)(BH * nch), kPruneThreads, 0, st>>>(
                static_cast<const E *>(k), kc.qn, kc.mask, static_cast<E *>(kc.vals), partial, kc.S, kc.T,
                nch, gpc, GroupArgs{}, kc.lens, kc.Hkv, static_cast<uint32_t *>(ws), nullptr);
    }
    stats_kernel<<<(unsigned)((BH + 3) / 4), 128, 0, st>>>(partial, nch, BH, kc.S, kc.T, kc.stats, kc.lens,
                                                           kc.Hkv);
    return cudaGetLastError();
}

cudaError_t launch_qnorm(const void *q_obs, int G, int W, long BH, int dtype, float *qn, cudaStream_t st) {
    if (BH == 0) return cudaSuccess;
    if (dtype == SPARK_BF16)
        qnorm_kernel<__nv_bfloat16><<<(unsigned)BH, kD, 0, st>>>(static_cast<const __nv_bfloat16 *>(q_obs), G, W, qn, nullptr);
    else
        qnorm_kernel<float><<<(unsigned)BH, kD, 0, st>>>(static_cast<const float *>(q_obs), G, W, qn, nullptr);
    return cudaGetLastError();
}

cudaError_t launch_prune(const void *k, const void *q_obs, int G, int W, const spark_kcache &kc,
                         void *ws, cudaStream_t st) {
    if (kc.dtype == SPARK_BF16) return launch_prune_t<__nv_bfloat16>(k, q_obs, G, W, kc, ws, st, nullptr);
    return launch_prune_t<float>(k, q_obs, G, W, kc, ws, st, nullptr);
}

__global__ void fill_ones_kernel(float *__restrict__ qn) { qn[(size_t)blockIdx.x * kD + threadIdx.x] = 1.f; }

// Value-channel pruning: the key kernel with every channel norm 1, so the
// saliency is |v| exactly (a multiply by 1 is exact).
cudaError_t launch_prune_values(const void *v, const spark_kcache &vc, void *ws, cudaStream_t st) {
    const long BH = (long)vc.B * vc.Hkv;
    if (BH == 0) return cudaSuccess;
    fill_ones_kernel<<<(unsigned)BH, kD, 0, st>>>(vc.qn);
    double *partial = reinterpret_cast<double *>(static_cast<char *>(ws) + kWsHeader);
    const int gpc = prune_groups_per_cta(BH, vc.S);
    const int nch = prune_chunks(vc.S, gpc);
    if (nch > 0) {
        if (vc.dtype == SPARK_BF16)
            prune_kernel<__nv_bfloat16, kModePlain><<<(unsigned)(BH * nch), kPruneThreads, 0, st>>>(
                static_cast<const __nv_bfloat16 *>(v), vc.qn, vc.mask, static_cast<__nv_bfloat16 *>(vc.vals),
                partial, vc.S, vc.T, nch, gpc, GroupArgs{}, vc.lens, vc.Hkv, static_cast<uint32_t *>(ws), nullptr);
        else
            prune_kernel<float, kModePlain><<<(unsigned)(BH * nch), kPruneThreads, 0, st>>>(
                static_cast<const float *>(v), vc.qn, vc.mask, static_cast<float *>(vc.vals), partial, vc.S, vc.T,
                nch, gpc, GroupArgs{}, vc.lens, vc.Hkv, static_cast<uint32_t *>(ws), nullptr);
    }
    stats_kernel<<<(unsigned)((BH + 3) / 4), 128, 0, st>>>(partial, nch, BH, vc.S, vc.T, vc.stats, vc.lens,
                                                           vc.Hkv);
    return cudaGetLastError();
}

cudaError_t launch_prune_grouped(const void *k, const void *q_obs, int G, int W, int n_groups,
                                 const int *group_T, const spark_kcache &kc, void *ws, cudaStream_t st) {
    GroupArgs ga{};
    ga.n = n_groups;
    for (int q = 0; q < n_groups; ++q) ga.T[q] = group_T[q];
    if (kc.dtype == SPARK_BF16) return launch_prune_t<__nv_bfloat16>(k, q_obs, G, W, kc, ws, st, &ga);
    return launch_prune_t<float>(k, q_obs, G, W, kc, ws, st, &ga);
}

// ---------------------------------------------------------------------------
// SparK-p ("KV Cache 还能再砍一刀：SparK ..." section 5.2): every token keeps
// the fewest channels, taken in the greedy order of section 3.1 (saliency
// desc, lower channel first), whose cumulative saliency reaches p of its
// total, at most Tcap of them.  The decision is taken on fp64 sums of the
// fp32 saliencies (the pages leave the arithmetic open).  The search below
// first finds the boundary with fp32 masses: each lane adds its 32 channels
// in ascending order in fp32 from +0, then the quad adds
// (lane 0 + lane 1) + (lane 2 + lane 3) (fp32 addition is commutative, so
// every lane of the quad holds the same bits), target = fp32(p * total).  An
// fp64 check then moves the boundary where fp32 rounding put it on the wrong
// side.
//
// A set {16-bit key >= P} is a threshold set of the exact keys (the 16-bit
// key is monotone in them), hence a greedy prefix, and its mass M(P) does
// not increase with P.  The search uses the masses of the 16-bit keys
// themselves (count_mass_ge16, on the tensor cores) against p times their
// total; they are within fp16 rounding of the exact masses, so the search
// may stop a channel off the exact boundary, and the fp64 step after it moves
// the boundary from any greedy prefix.  The search finds the
// largest level lo with M(lo) >= target by binary lifting, tracking the
// lowest failing level hi: over [0, 2^15) for the first token of a quad
// (M(0) is the total, nothing reaches 2^15), otherwise over a 2^11-level
// window around a running estimate, redone over [0, 2^15) when the window
// did not bracket lo.  It leaves early once {key >= lo} and {key >= hi}
// differ by one channel for every quad of the warp: that channel ends the
// prefix.  Otherwise the band between them is added one channel at a time
// in greedy order (exact keys desc, lower channel first) until the exact
// fp32 mass reaches the exact fp32 target.  A prefix longer than Tcap is replaced by the top-Tcap
// set (select_top_t).

// this lane's channels whose 16-bit key is >= P (bit i = channel i)
__device__ __forceinline__ uint32_t ge16_bits(const uint32_t (&kp)[16], uint32_t P) {
    const uint32_t p2 = P * 0x10001u;
    uint32_t m = 0u;
#pragma unroll
    for (int i = 0; i < 16; ++i) m |= hge2_mask(kp[i], p2) & (0x00010001u << i);
    return m;
}

// fp32 mass of the quad's channels in m, in the order described above
__device__ __forceinline__ float quad_mass(const uint32_t (&key)[32], uint32_t m) {
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) acc = ((m >> i) & 1u) ? __fadd_rn(acc, __uint_as_float(key[i])) : acc;
    const float a = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, 1));
    return __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, 2));
}

// D += A * B for one m16n8k16 tile, fp16 operands, fp32 accumulators.
__device__ __forceinline__ void mma_f16_f32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Count and mass of the quad's 16-bit keys >= the probe p2, on the tensor
// cores (the layout of count_ge16): the 0/1 compare results count the keys
// in fp16, and the keys times those results (the keys of the set, exact) are
// summed with fp32 accumulators.  The mass is that of the fp16 keys, within
// fp16 rounding of the exact scaled mass; every lane of the quad receives
// both.
__device__ __forceinline__ void count_mass_ge16(const uint32_t (&kp)[16], uint32_t p2, int &cnt, float &mass) {
    uint32_t c0 = 0u, c1 = 0u;
    float f[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        uint32_t a[4], w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            a[e] = hge2_one(kp[4 * m + e], p2);
            const __half2 x = __hmul2(*reinterpret_cast<const __half2 *>(&a[e]),
                                      *reinterpret_cast<const __half2 *>(&kp[4 * m + e]));
            w[e] = *reinterpret_cast<const uint32_t *>(&x);
        }
        mma_f16(c0, c1, a[0], a[1], a[2], a[3], kOne2, kOne2);
        mma_f16_f32(f, w[0], w[1], w[2], w[3], kOne2, kOne2);
    }
    const __half2 c = __hadd2(*reinterpret_cast<const __half2 *>(&c0), *reinterpret_cast<const __half2 *>(&c1));
    cnt = __half2int_rn(__low2half(c));
    mass = __fadd_rn(f[0], f[2]);  // rows r and r + 8: the token's two halves
}

// search state of one quad: M(lo) >= target > M(hi) once both are known
struct TopPBracket {
    uint32_t lo, hi;
    int clo, chi;    // channel counts of {key >= lo}, {key >= hi}
    bool klo, khi;   // lo / hi established by a probe (or known bounds)
};

// Binary lifting of lo over [lo, lo + 2^K) for the active quads on the
// fp16-key masses (target: p times the fp16-key total); every loop trip is
// warp-uniform (the tensor-core counts see all lanes).
__device__ __forceinline__ void topp_lift(const uint32_t (&kp)[16], float target, int K, bool active,
                                          TopPBracket &b) {
    bool done = !active || (b.klo && b.khi && b.clo - b.chi <= 1);
    for (int bit = K - 1; bit >= 0; --bit) {
        if (__all_sync(0xffffffffu, done)) break;
        const uint32_t P = b.lo + (1u << bit);
        int c;
        float M;
        count_mass_ge16(kp, P * 0x10001u, c, M);
        if (!done) {
            if (M >= target) {
                b.lo = P;
                b.clo = c;
                b.klo = true;
            } else {
                b.hi = P;
                b.chi = c;
                b.khi = true;
            }
            done = b.klo && b.khi && b.clo - b.chi <= 1;
        }
    }
}

// the whole 16-bit key range: M(0) = total >= target, no key reaches 2^15
__device__ __forceinline__ void topp_full_range(TopPBracket &b) {
    b.lo = 0u;
    b.hi = 0x8000u;
    b.clo = kD;
    b.chi = 0;
    b.klo = b.khi = true;
}

template <typename E>
__global__ void __launch_bounds__(kPruneThreads, 3)
    prune_topp_kernel(const E *__restrict__ k, const float *__restrict__ qn, uint32_t *__restrict__ mask,
                      uint32_t *__restrict__ tg, double *__restrict__ partial, int S, int Tcap, int n_chunks,
                      int gpc, float p) {
    __shared__ double red[3][kPruneThreads / 32];
    __shared__ uint32_t qmax[kPruneThreads / 32];
    __shared__ __align__(16) float qs[4 * 36];

    const long bh = blockIdx.x / n_chunks;
    const int chunk = blockIdx.x % n_chunks;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int s = lane & 3;
    const int tq = lane >> 2;
    const int tl = warp * 8 + tq;
    const long S32 = ((long)S + 31) / 32 * 32;

    {
        const float q = __ldg(qn + bh * kD + tid);
        qs[(tid >> 5) * 36 + (tid & 31)] = q;
        const uint32_t mx = __reduce_max_sync(0xffffffffu, __float_as_uint(q) & 0x7fffffffu);
        if (lane == 0) qmax[warp] = mx;
    }
    __syncthreads();
    float scale = 1.f, inv_scale = 1.f;
    {
        uint32_t mx = qmax[0];
#pragma unroll
        for (int w = 1; w < kPruneThreads / 32; ++w) mx = max(mx, qmax[w]);
        const int e = (int)(mx >> 23);
        if (e > 0 && e < 255) {
            const int x = min(max(127 - e, -64), 64);
            scale = __uint_as_float((uint32_t)(127 + x) << 23);
            inv_scale = __uint_as_float((uint32_t)(127 - x) << 23);
        }
    }
    const float2 scale2 = make_float2(scale, scale);

    uint32_t tau = 0u;  // running estimate of the quad's mass level
    double acc_w = 0.0, acc_w2 = 0.0, acc_n = 0.0;
    const long g_first = (long)chunk * gpc;
    const long ng = S32 / 32;
    const E *krow = k + ((size_t)bh * S + g_first * 32 + tl) * kD + 32 * s;

    auto group = [&](int gi, KSlice<E> &cur, KSlice<E> &nxt) {
        const long t = (g_first + gi) * 32 + tl;
        const bool valid = t < S;
        if (gi + 1 < gpc && t + 32 < S) nxt.load(krow + (size_t)(gi + 1) * 32 * kD);
        else nxt.zero();

        uint32_t key[32];
        float2 wsc[16];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float4 q4 = *reinterpret_cast<const float4 *>(qs + s * 36 + 4 * c);
            const float2 w01 = __fmul2_rn(make_float2(q4.x, q4.y), cur.abs_pair(2 * c));
            const float2 w23 = __fmul2_rn(make_float2(q4.z, q4.w), cur.abs_pair(2 * c + 1));
            key[4 * c + 0] = __float_as_uint(w01.x);
            key[4 * c + 1] = __float_as_uint(w01.y);
            key[4 * c + 2] = __float_as_uint(w23.x);
            key[4 * c + 3] = __float_as_uint(w23.y);
            wsc[2 * c] = __fmul2_rn(w01, scale2);
            wsc[2 * c + 1] = __fmul2_rn(w23, scale2);
        }
        uint32_t kp[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float a = (i & 1) ? wsc[i >> 1].y : wsc[i >> 1].x;
            const float b = (i & 1) ? wsc[8 + (i >> 1)].y : wsc[8 + (i >> 1)].x;
            const __half2 h = __floats2half2_rn(a, b);
            kp[i] = *reinterpret_cast<const uint32_t *>(&h);
        }

        // target = p * total; a token with target 0 (p = 0 or no saliency)
        // keeps nothing.  The search runs on the fp16 keys' masses (target16
        // from their total); the band walk and the fp64 decision below use
        // the exact keys, and the fp64 step moves the boundary to its exact
        // place from wherever the search put it.
        const float total = quad_mass(key, 0xffffffffu);
        const float target = __fmul_rn(p, total);
        const bool active = valid && target > 0.f && Tcap > 0;
        float target16;
        {
            int c_all;
            float m_all;
            count_mass_ge16(kp, 0u, c_all, m_all);
            target16 = __fmul_rn(p, m_all);
        }

        TopPBracket b;
        if (gi == 0) {
            topp_full_range(b);
        } else {
            b.lo = min(tau > 1024u ? tau - 1024u : 0u, kTop16 - 2048u);
            b.hi = b.lo + 2048u;
            b.clo = kD;
            b.chi = 0;
            b.klo = b.khi = false;
        }
        topp_lift(kp, target16, gi == 0 ? 15 : 11, active, b);
        const bool suspect = active && !(b.klo && b.khi);
        if (__any_sync(0xffffffffu, suspect)) {
            if (suspect) topp_full_range(b);
            topp_lift(kp, target16, 15, suspect, b);
        }

        uint32_t m = active ? ge16_bits(kp, b.lo) : 0u;
        const bool band = active && b.clo - b.chi >= 2;
        if (__any_sync(0xffffffffu, band)) {
            // the prefix {key >= hi} falls short; add the band's channels in
            // greedy order until the mass reaches the target
            uint32_t mA = ge16_bits(kp, min(b.hi, kTop16));
            uint32_t mB = band ? (m & ~mA) : 0u;
            bool open = band;
            for (int it = 0; it < kD && __any_sync(0xffffffffu, open); ++it) {
                uint32_t bk = 0u;
                int bi = -1;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const bool take = ((mB >> i) & 1u) && (bi < 0 || key[i] > bk);
                    bk = take ? key[i] : bk;
                    bi = take ? i : bi;
                }
                // quad arg-max of (exact key desc, channel asc)
                uint32_t wk = bk;
                int wc = bi < 0 ? 4 * kD : 32 * s + bi;
#pragma unroll
                for (int o = 1; o <= 2; o <<= 1) {
                    const uint32_t ok = __shfl_xor_sync(0xffffffffu, wk, o);
                    const int oc = __shfl_xor_sync(0xffffffffu, wc, o);
                    const bool better = oc < 4 * kD && (wc >= 4 * kD || ok > wk || (ok == wk && oc < wc));
                    wk = better ? ok : wk;
                    wc = better ? oc : wc;
                }
                if (open && wc < 4 * kD && (wc >> 5) == s) {
                    mA |= 1u << (wc & 31);
                    mB &= ~(1u << (wc & 31));
                }
                const float M = quad_mass(key, mA);
                if (open && (M >= target || wc >= 4 * kD)) open = false;
            }
            m = band ? mA : m;
        }
        // The fp32 search above finds a greedy prefix whose fp32 mass reaches
        // the fp32 target.  The boundary itself is decided on the cumulative
        // saliency in fp64 (each fp32 key is exact in fp64, sums of 128 keys
        // round at 2^-46 relative): the prefix must reach target64 and, less
        // its last channel in greedy order, fall short of it.  Tokens that
        // fail (near-ties of the fp32 arithmetic) move the boundary one
        // channel at a time in greedy order.
        {
            double tot64 = 0.0, m64 = 0.0;
            float wl = __int_as_float(0x7f800000);  // smallest kept saliency
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float x = __uint_as_float(key[i]);
                const bool in = (m >> i) & 1u;
                tot64 = __dadd_rn(tot64, (double)x);
                m64 = in ? __dadd_rn(m64, (double)x) : m64;
                wl = in ? fminf(wl, x) : wl;
            }
#pragma unroll
            for (int o = 1; o <= 2; o <<= 1) {
                tot64 = __dadd_rn(tot64, __shfl_xor_sync(0xffffffffu, tot64, o));
                m64 = __dadd_rn(m64, __shfl_xor_sync(0xffffffffu, m64, o));
                wl = fminf(wl, __shfl_xor_sync(0xffffffffu, wl, o));
            }
            const double target64 = __dmul_rn((double)p, tot64);
            const bool act64 = valid && target64 > 0.0 && Tcap > 0;
            const bool some = quad_sum(__popc(m)) > 0;
            if (!act64) m = 0u;  // p = 0 or no saliency: nothing to keep
            bool open = act64 && (m64 < target64 || (some && __dsub_rn(m64, (double)wl) >= target64));
            for (int it = 0; it < 2 * kD && __any_sync(0xffffffffu, open); ++it) {
                // greedy-next channel outside the set: (key desc, channel asc);
                // greedy-last inside it: (key asc, channel desc)
                uint32_t nk = 0u, lk = 0xffffffffu;
                int ni = -1, li = -1;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const bool in = (m >> i) & 1u;
                    const bool tn = !in && (ni < 0 || key[i] > nk);
                    nk = tn ? key[i] : nk;
                    ni = tn ? i : ni;
                    const bool tl2 = in && (li < 0 || key[i] <= lk);
                    lk = tl2 ? key[i] : lk;
                    li = tl2 ? i : li;
                }
                int nc = ni < 0 ? -1 : 32 * s + ni, lc = li < 0 ? -1 : 32 * s + li;
#pragma unroll
                for (int o = 1; o <= 2; o <<= 1) {
                    const uint32_t onk = __shfl_xor_sync(0xffffffffu, nk, o);
                    const int onc = __shfl_xor_sync(0xffffffffu, nc, o);
                    const bool bn = onc >= 0 && (nc < 0 || onk > nk || (onk == nk && onc < nc));
                    nk = bn ? onk : nk;
                    nc = bn ? onc : nc;
                    const uint32_t olk = __shfl_xor_sync(0xffffffffu, lk, o);
                    const int olc = __shfl_xor_sync(0xffffffffu, lc, o);
                    const bool bl = olc >= 0 && (lc < 0 || olk < lk || (olk == lk && olc > lc));
                    lk = bl ? olk : lk;
                    lc = bl ? olc : lc;
                }
                if (open) {
                    if (m64 < target64 && nc >= 0) {
                        if ((nc >> 5) == s) m |= 1u << (nc & 31);
                        m64 = __dadd_rn(m64, (double)__uint_as_float(nk));
                    } else if (lc >= 0 && __dsub_rn(m64, (double)__uint_as_float(lk)) >= target64) {
                        if ((lc >> 5) == s) m &= ~(1u << (lc & 31));
                        m64 = __dsub_rn(m64, (double)__uint_as_float(lk));
                    } else {
                        open = false;
                    }
                }
            }
        }
        const int n_keep = quad_sum(__popc(m));
        if (active) tau = gi == 0 ? b.lo : (uint32_t)((int)tau + (((int)b.lo - (int)tau) >> 1));

        // capacity: a longer prefix becomes the top-Tcap set
        const bool cap = active && n_keep > Tcap;
        if (__any_sync(0xffffffffu, cap)) {
            const uint32_t base = min(b.lo, kTop16 - (1u << kLiftCold));
            uint32_t lo_cap;
            const uint32_t mc = select_top_t(key, kp, Tcap, s, inv_scale, base, kLiftCold, !cap, 0xffffffffu, lo_cap);
            m = cap ? mc : m;
        }
        if (valid) mask[((size_t)bh * S + t) * kMaskWords + s] = m;

        // the group's slot count: the largest kept count of its tokens (the
        // four warps of the CTA each bring their 8 tokens)
        const int kept = quad_sum(__popc(m));  // every lane shuffles; m = 0 on padding tokens
        const int wmax = __reduce_max_sync(0xffffffffu, kept);
        if (lane == 0 && wmax > 0) atomicMax(tg + (size_t)bh * ng + g_first + gi, (unsigned)wmax);

        // pruned-saliency sums: fp32 over this lane's 32 channels
        float sw = 0.f, sw2 = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (!((m >> i) & 1u)) {
                const float w = __uint_as_float(key[i]);
                sw = __fadd_rn(sw, w);
                sw2 = __fmaf_rn(w, w, sw2);
            }
        }
        if (valid) {
            acc_w = __dadd_rn(acc_w, (double)sw);
            acc_w2 = __dadd_rn(acc_w2, (double)sw2);
            acc_n = __dadd_rn(acc_n, (double)(32 - __popc(m)));
        }
    };

    // one call site: a second inlined copy of the group body does not fit
    // the instruction cache
    KSlice<E> ka, kb;
    if (g_first * 32 + tl < S) ka.load(krow);
    else ka.zero();
#pragma unroll 1
    for (int gi = 0; gi < gpc; ++gi) {
        if ((g_first + gi) * 32 >= S) break;  // uniform across the CTA
        group(gi, ka, kb);
        ka = kb;
    }

#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        acc_w = __dadd_rn(acc_w, __shfl_xor_sync(0xffffffffu, acc_w, o));
        acc_w2 = __dadd_rn(acc_w2, __shfl_xor_sync(0xffffffffu, acc_w2, o));
        acc_n = __dadd_rn(acc_n, __shfl_xor_sync(0xffffffffu, acc_n, o));
    }
    if (lane == 0) {
        red[0][warp] = acc_w;
        red[1][warp] = acc_w2;
        red[2][warp] = acc_n;
    }
    __syncthreads();
    if (tid == 0) {
        double a = 0.0, b2 = 0.0, n = 0.0;
        for (int i = 0; i < kPruneThreads / 32; ++i) {
            a = __dadd_rn(a, red[0][i]);
            b2 = __dadd_rn(b2, red[1][i]);
            n = __dadd_rn(n, red[2][i]);
        }
        partial[((size_t)bh * n_chunks + chunk) * 3 + 0] = a;
        partial[((size_t)bh * n_chunks + chunk) * 3 + 1] = b2;
        partial[((size_t)bh * n_chunks + chunk) * 3 + 2] = n;
    }
}

// SparK-p statistics: the pruned count is data-dependent, summed like the
// saliency sums (exact: integers below 2^53).
__global__ void stats_topp_kernel(const double *__restrict__ partial, int n_chunks, long BH,
                                  double *__restrict__ stats) {
    const long bh = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (bh >= BH) return;
    double a = 0.0, b = 0.0, n = 0.0;
    for (int c = lane; c < n_chunks; c += 32) {
        a = __dadd_rn(a, partial[((size_t)bh * n_chunks + c) * 3 + 0]);
        b = __dadd_rn(b, partial[((size_t)bh * n_chunks + c) * 3 + 1]);
        n = __dadd_rn(n, partial[((size_t)bh * n_chunks + c) * 3 + 2]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a = __dadd_rn(a, __shfl_xor_sync(0xffffffffu, a, o));
        b = __dadd_rn(b, __shfl_xor_sync(0xffffffffu, b, o));
        n = __dadd_rn(n, __shfl_xor_sync(0xffffffffu, n, o));
    }
    if (lane == 0) {
        stats[bh * 4 + 0] = n;
        stats[bh * 4 + 1] = a;
        stats[bh * 4 + 2] = b;
        stats[bh * 4 + 3] = n > 0.0 ? a / n : 0.0;
    }
}

// ---- SparK-p value layout.  The selection kernel leaves tg[i] = the largest
// kept count of group i (zeroed before it runs).  Three small launches turn
// the counts into group offsets in rows of 32 elements -- per-head totals, a
// scan of the head totals, per-head scans plus the head bases -- integer
// sums, so the offsets are the same on every run.  topp_gather_kernel then
// reads the key rows a second time and writes each group's kept values.
constexpr int kScanThreads = 1024;

// exclusive prefix of v over the CTA (kScanThreads threads); *tot = the sum
__device__ __forceinline__ uint32_t cta_excl_scan(uint32_t v, uint32_t *sh, uint32_t &tot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = sh[lane];  // kScanThreads / 32 == 32 warp totals
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        sh[32 + lane] = w;
    }
    __syncthreads();
    tot = sh[63];
    const uint32_t r = (warp > 0 ? sh[32 + warp - 1] : 0u) + x - v;
    __syncthreads();  // sh is reused by the caller's next round
    return r;
}

// rows of each head: the sum of its groups' slot counts
__global__ void __launch_bounds__(kScanThreads) topp_head_rows_kernel(const uint32_t *__restrict__ tg, long ng,
                                                                      uint32_t *__restrict__ hrows) {
    __shared__ uint32_t sh[64];
    const long bh = blockIdx.x;
    uint32_t acc = 0u;
    for (long g = threadIdx.x; g < ng; g += kScanThreads) acc += tg[bh * ng + g];
    uint32_t tot;
    (void)cta_excl_scan(acc, sh, tot);
    if (threadIdx.x == 0) hrows[bh] = tot;
}

// first row of each head (exclusive scan of the head totals, one CTA), and
// the total rows into the last entry of goff
__global__ void __launch_bounds__(kScanThreads) topp_head_base_kernel(const uint32_t *__restrict__ hrows, long BH,
                                                                      uint32_t *__restrict__ hbase,
                                                                      uint32_t *__restrict__ goff_end) {
    __shared__ uint32_t sh[64];
    uint32_t carry = 0u;
    for (long b0 = 0; b0 < BH; b0 += kScanThreads) {
        const long bh = b0 + threadIdx.x;
        const uint32_t v = bh < BH ? hrows[bh] : 0u;
        uint32_t tot;
        const uint32_t ex = cta_excl_scan(v, sh, tot);
        if (bh < BH) hbase[bh] = carry + ex;
        carry += tot;
    }
    if (threadIdx.x == 0) *goff_end = carry;
}

// goff of each group: its head's base plus the exclusive scan of the head's
// slot counts
__global__ void __launch_bounds__(kScanThreads) topp_goff_kernel(const uint32_t *__restrict__ tg, long ng,
                                                                 const uint32_t *__restrict__ hbase,
                                                                 uint32_t *__restrict__ goff) {
    __shared__ uint32_t sh[64];
    const long bh = blockIdx.x;
    uint32_t carry = hbase[bh];
    for (long g0 = 0; g0 < ng; g0 += kScanThreads) {
        const long g = g0 + threadIdx.x;
        const uint32_t v = g < ng ? tg[bh * ng + g] : 0u;
        uint32_t tot;
        const uint32_t ex = cta_excl_scan(v, sh, tot);
        if (g < ng) goff[bh * ng + g] = carry + ex;
        carry += tot;
    }
}

// Kept values of the SparK-p cache: one warp per 32-token group.  The
// group's key rows arrive by one bulk copy; then lane = token, and every
// lane runs the group's T_g slots from the top (the same slot j for the
// whole warp, so each slot of the 32 tokens is one coalesced store): slot j
// takes the token's j-th kept channel in ascending order -- found by walking
// the mask bits from the top channel down -- or 0 past the token's count.
constexpr int kGatherWarps = 4;

// shared memory of one gather warp: 32 key rows at a stride of one row + 16
// bytes (each lane's bulk copy lands 4 banks further on, so lanes reading
// the same channel meet at most 4 to a bank instead of all 32), then the
// group's value slots in their output layout, [slot][32 tokens]
template <typename E> __host__ __device__ constexpr int gather_row_stride() { return kD * (int)sizeof(E) + 16; }
template <typename E> __host__ __device__ constexpr int gather_warp_smem() {
    return 32 * gather_row_stride<E>() + kD * 32 * (int)sizeof(typename RawT<E>::type);
}

// One warp per 32-token group.  Each lane brings its token's key row into
// shared memory with one bulk copy, then every lane steps through the 128
// channels from the top together: a kept channel's key goes to the token's
// next slot from the end (slot n-1 for the highest kept channel, slot 0 for
// the lowest), so the slots come out in ascending channel order; slots from
// the token's count up to T_g are zero.  The slots are staged in the output
// layout, and the group's T_g * 32 values, one contiguous block, are written
// with 16-byte stores.
template <typename E>
__global__ void __launch_bounds__(kGatherWarps * 32)
    topp_gather_kernel(const E *__restrict__ k, const uint32_t *__restrict__ mask, const uint32_t *__restrict__ goff,
                       E *__restrict__ vals, uint32_t *__restrict__ status, int S, long ng, long n_groups) {
    using Raw = typename RawT<E>::type;
    constexpr int kRowB = kD * (int)sizeof(E), kRowP = gather_row_stride<E>();
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ uint64_t bars[kGatherWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long idx = (long)blockIdx.x * kGatherWarps + warp;
    if (idx >= n_groups) return;
    const long bh = idx / ng, g = idx % ng;
    const long t0 = g * 32;
    const int rows = (int)min(32L, (long)S - t0);
    unsigned char *tile = smem_raw + (size_t)warp * gather_warp_smem<E>();
    Raw *stage = reinterpret_cast<Raw *>(tile + 32 * kRowP);
    const uint32_t bar = smem_u32(&bars[warp]);
    if (lane == 0) {
        mbar_init(bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        mbar_expect_tx(bar, (uint32_t)rows * (uint32_t)kRowB);
    }
    __syncwarp();
    const bool valid = lane < rows;
    if (valid) bulk_g2s(smem_u32(tile + lane * kRowP), k + ((size_t)bh * S + t0 + lane) * kD, (uint32_t)kRowB, bar);
    uint4 mw = make_uint4(0u, 0u, 0u, 0u);
    if (valid) mw = *reinterpret_cast<const uint4 *>(mask + ((size_t)bh * S + t0 + lane) * kMaskWords);
    const int n = __popc(mw.x) + __popc(mw.y) + __popc(mw.z) + __popc(mw.w);
    const uint32_t r0 = goff[idx];
    const int Tg = (int)min(goff[idx + 1] - r0, (uint32_t)kD);
    // slots past this token's count read zero (n <= T_g for a cache that
    // spark_prune_topp wrote; a larger n only fills slots that are not copied)
    for (int j = n; j < Tg; ++j) stage[j * 32 + lane] = (Raw)0;
    const bool ok = mbar_wait_bounded(bar, 0u);
    if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) {
            atomicOr(status, kDevTimeout);
            (void)mbar_wait_bounded(bar, 0u);  // let the copies in flight land before the warp exits
        }
        __syncwarp();
        return;
    }
    {
        const Raw *row = reinterpret_cast<const Raw *>(tile + lane * kRowP);
        const uint32_t wds[4] = {mw.x, mw.y, mw.z, mw.w};
        int j = n;
#pragma unroll
        for (int wi = 3; wi >= 0; --wi) {
#pragma unroll
            for (int b = 31; b >= 0; --b) {
                if ((wds[wi] >> b) & 1u) {
                    --j;
                    stage[j * 32 + lane] = row[32 * wi + b];
                }
            }
        }
    }
    __syncwarp();
    // the group's slots: T_g rows of 32 values, contiguous in the stream
    constexpr int kChunks = 32 * (int)sizeof(Raw) / 16;  // 16-byte pieces per slot row
    const uint4 *src = reinterpret_cast<const uint4 *>(stage);
    uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<Raw *>(vals) + (size_t)r0 * 32);
    for (int c = lane; c < Tg * kChunks; c += 32) __stcs(dst + c, src[c]);
}

template <typename E>
static cudaError_t launch_prune_topp_t(const void *k, const void *q_obs, int G, int W, float p,
                                       const spark_kcache &kc, void *ws, cudaStream_t st) {
    const long BH = (long)kc.B * kc.Hkv;
    if (BH == 0) return cudaSuccess;
    const long ng = ((long)kc.S + 31) / 32;
    const ToppWs tw = topp_ws_layout(ws, BH, kc.S);
    qnorm_kernel<E><<<(unsigned)BH, kD, 0, st>>>(static_cast<const E *>(q_obs), G, W, kc.qn, nullptr);
    const int gpc = prune_groups_per_cta(BH, kc.S);
    const int nch = prune_chunks(kc.S, gpc);
    if (ng > 0) {
        cudaError_t e = cudaMemsetAsync(tw.tg, 0, (size_t)BH * ng * sizeof(uint32_t), st);
        if (e != cudaSuccess) return e;
        prune_topp_kernel<E><<<(unsigned)(BH * nch), kPruneThreads, 0, st>>>(
            static_cast<const E *>(k), kc.qn, kc.mask, tw.tg, tw.partial, kc.S, kc.T, nch, gpc, p);
    }
    stats_topp_kernel<<<(unsigned)((BH + 3) / 4), 128, 0, st>>>(tw.partial, nch, BH, kc.stats);
    // group offsets (the last entry, the total, also when there are no groups)
    if (ng > 0) topp_head_rows_kernel<<<(unsigned)BH, kScanThreads, 0, st>>>(tw.tg, ng, tw.hrows);
    else {
        cudaError_t e = cudaMemsetAsync(tw.hrows, 0, (size_t)BH * sizeof(uint32_t), st);
        if (e != cudaSuccess) return e;
    }
    topp_head_base_kernel<<<1, kScanThreads, 0, st>>>(tw.hrows, BH, tw.hbase, kc.goff + BH * ng);
    if (ng > 0) {
        topp_goff_kernel<<<(unsigned)BH, kScanThreads, 0, st>>>(tw.tg, ng, tw.hbase, kc.goff);
        const int smem = kGatherWarps * gather_warp_smem<E>();
        cudaError_t e = cudaFuncSetAttribute(topp_gather_kernel<E>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        const long n_groups = BH * ng;
        topp_gather_kernel<E><<<(unsigned)((n_groups + kGatherWarps - 1) / kGatherWarps), kGatherWarps * 32, smem, st>>>(
            static_cast<const E *>(k), kc.mask, kc.goff, static_cast<E *>(kc.vals), static_cast<uint32_t *>(ws),
            kc.S, ng, n_groups);
    }
    return cudaGetLastError();
}

cudaError_t launch_prune_topp(const void *k, const void *q_obs, int G, int W, float p, const spark_kcache &kc,
                              void *ws, cudaStream_t st) {
    if (kc.dtype == SPARK_BF16) return launch_prune_topp_t<__nv_bfloat16>(k, q_obs, G, W, p, kc, ws, st);
    return launch_prune_topp_t<float>(k, q_obs, G, W, p, kc, ws, st);
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

// Device address of the scratch array in the current context.  Host code
// cannot use the symbol itself: there it names a host-side stand-in.  The
// address is looked up on every call rather than cached: after a device
// reset, or under another context of the same device, the module is loaded
// again and the array can sit elsewhere.  The first lookup in a context loads
// the module (set-up); later ones read the runtime's table.
static void *prune_scratch() {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_prune_scratch) != cudaSuccess) return nullptr;
    return p;
}

}  // namespace spark

extern "C" SPARK_API int spark_prune_noalloc(const void *k, const void *q_obs, int G, int W,
                                             const spark_kcache *out, void *stream) {
    using namespace spark;
    const int rc = check_prune_args(k, q_obs, G, W, out);
    if (rc != SPARK_OK) return rc;
    const long BH = (long)out->B * out->Hkv;
    if (BH == 0) return SPARK_OK;
    if (prune_workspace(BH, out->S) > kNoAllocScratchBytes) return SPARK_ERR_WORKSPACE;
    void *ws = prune_scratch();
    if (!ws) return SPARK_ERR_CUDA;
    cudaError_t e = launch_prune(k, q_obs, G, W, *out, ws, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SPARK_OK : SPARK_ERR_CUDA;
}
