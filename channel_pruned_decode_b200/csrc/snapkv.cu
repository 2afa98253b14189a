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
//   snap_tc_kernel<0/1>  the keys of each (row, kv head) split over several
//       CTAs; the G*W x S logits are a dense contraction, computed by
//       tcgen05.mma (bf16 -> fp32 in tensor memory) from 128-byte-swizzled
//       shared-memory tiles, the key tiles fetched by TMA.  Pass 0 writes
//       each split's running max and
//       exp-sum of every window row (online softmax); pass 1 merges them in a
//       fixed order, recomputes the logits and sums the normalised
//       probabilities of each key over the rows (one MUFU exp2 per score,
//       the row's 1 / l folded into the exponent).
//   snap_select_kernel  one CTA per head: max-pool, exact radix select of the
//       (keep-W)-th largest pooled score on its fp32 bit pattern (scores are
//       >= 0; 8-bit digits, each digit found by a warp scan of the
//       histogram), and an order-preserving compaction (ties to the lower
//       index; contiguous token ranges per thread, two block scans).
//   snap_gather_kernel  copies the kept K and V rows (16-byte vectors).
#include "spark_internal.cuh"

#include <cuda.h>  // CUtensorMap and its enums (the encoder is fetched at run time)

#include <algorithm>

namespace spark {

constexpr int kSnapMaxSplit = 16;  // CTAs per (row, kv head)
constexpr int kSnapMaxRows = 128;  // window rows G * W
constexpr int kSelThreads = 1024;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    const int n = valid ? 16 : 0;  // zero-fill when the source row does not exist
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// log2(e) / sqrt(128)
constexpr float kSnapScale = 0.12751743074602467f;

// 2^x on the MUFU unit in one instruction (results below 2^-126 flush to 0:
// a probability that small does not move a sum that holds the row's maximum)
__device__ __forceinline__ float ex2_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
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
                       int pool, int *__restrict__ idx, const int32_t *__restrict__ keep_rows, int Hkv,
                       int keep_cap, uint32_t *__restrict__ status) {
    __shared__ int hist[256];
    __shared__ int wsum[32];
    __shared__ uint32_t sel[3];  // prefix, remaining rank, digit
    const long bh = blockIdx.x;
    const int tid = threadIdx.x;
    const long P = (long)S - W;
    if (keep_rows) {  // a budget per row (uniform over the CTA)
        keep = keep_rows[bh / Hkv];
        if (keep < W || keep > S || keep > keep_cap) {
            if (tid == 0) atomicOr(status, kDevBadArg);
            return;
        }
    }
    const int kp = keep - W;
    const float *sc = scores + (size_t)bh * P;
    uint32_t *pk = pooled + (size_t)bh * P;
    int *out = idx + (size_t)bh * keep_cap;
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
        if (tid < 32) {
            // the largest digit d whose count from the top, inclusive, reaches
            // rem: lane l sums digits 255 - 8l ... 248 - 8l, a warp scan gives
            // the count above each lane's block, and the lane whose block
            // crosses rem walks its 8 digits (digit 0 if no block crosses)
            const int lane = tid;
            int c[8], loc = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                c[j] = hist[255 - 8 * lane - j];
                loc += c[j];
            }
            int incl = loc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const int before = incl - loc;
            const bool cross = before < rem && incl >= rem;
            const unsigned who = __ballot_sync(0xffffffffu, cross);
            if (who == 0u) {
                if (lane == 31) {  // no block reaches rem: digit 0 with everything above it
                    sel[0] = prefix;
                    sel[1] = (uint32_t)(rem - (incl - c[7]));
                }
            } else if (cross) {
                int above = before, d = 255 - 8 * lane;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (above + c[j] >= rem) {
                        d = 255 - 8 * lane - j;
                        break;
                    }
                    above += c[j];
                }
                sel[0] = prefix | ((uint32_t)d << shift);
                sel[1] = (uint32_t)(rem - above);
            }
        }
        __syncthreads();
        prefix = sel[0];
        rem = (int)sel[1];
        pmask |= 255u << shift;
        __syncthreads();
    }
    // keep: key > prefix, plus the first `rem` keys == prefix in index order.
    // Thread i owns the contiguous tokens [i*E, (i+1)*E), so two block scans
    // (equal keys before it, kept tokens before it) place every kept index.
    const long E = (P + kSelThreads - 1) / kSelThreads;
    const long tb = min(P, (long)tid * E), te = min(P, tb + E);
    int n_eq = 0;
    for (long t = tb; t < te; ++t) n_eq += (kp > 0 && pk[t] == prefix) ? 1 : 0;
    int tot;
    const int eq_before = block_excl_scan(n_eq, wsum, tot);
    int n_keep = 0;
    for (long t = tb, r = eq_before; t < te && kp > 0; ++t) {
        const uint32_t key = pk[t];
        const bool eq = key == prefix;
        n_keep += (key > prefix || (eq && r < rem)) ? 1 : 0;
        r += eq ? 1 : 0;
    }
    int pos = block_excl_scan(n_keep, wsum, tot);
    for (long t = tb, r = eq_before; t < te && kp > 0; ++t) {
        const uint32_t key = pk[t];
        const bool eq = key == prefix;
        if (key > prefix || (eq && r < rem)) out[pos++] = (int)t;
        r += eq ? 1 : 0;
    }
    for (int w = tid; w < W; w += kSelThreads) out[kp + w] = (int)(P + w);
}

__global__ void snap_gather_kernel(const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                                   const int *__restrict__ idx, int S, int W, int keep, int row_vec,
                                   uint4 *__restrict__ k_out, uint4 *__restrict__ v_out,
                                   const int32_t *__restrict__ keep_rows, int Hkv, int keep_cap) {
    const long bh = blockIdx.y;
    const long i = (long)blockIdx.x * (blockDim.x / row_vec) + threadIdx.x / row_vec;
    const int c = threadIdx.x % row_vec;
    if (keep_rows) {
        keep = keep_rows[bh / Hkv];
        if (keep < W || keep > S || keep > keep_cap) return;  // recorded by the select kernel
    }
    if (i >= keep) return;
    const long t = idx[bh * keep_cap + i];
    k_out[((size_t)bh * keep_cap + i) * row_vec + c] = k[((size_t)bh * S + t) * row_vec + c];
    v_out[((size_t)bh * keep_cap + i) * row_vec + c] = v[((size_t)bh * S + t) * row_vec + c];
}

// ---------------------------------------------------------------------------
// tcgen05 version of the two score passes.  Per CTA: 256 threads (8 warps);
// a 128 x 128 query tile (window rows, zero-padded) and a ring of two 128-key
// tiles in shared memory, K-major with the 128-byte swizzle that the UMMA
// descriptors describe; two 128-column fp32 accumulators in tensor memory.
// Thread 0 fetches the key tiles by TMA (completion on a per-buffer
// mbarrier), issues the tcgen05.mma instructions once a tile has landed and
// commits them to a per-accumulator mbarrier; every thread then reads half of
// one accumulator row (tcgen05.ld:
// warp w reads TMEM lanes 32*(w%4).. and columns 64*(w/4)..).  Pass 0
// computes S = Q K^T (a row is a window row: its running max and exp-sum are
// kept per half and merged at the end); pass 1 computes S^T = K Q^T (a row is
// a key: its probability sum over the window rows is summed per half, then
// the halves are added).
constexpr int kTcKeys = 128;                  // keys per tile (MMA M or N)
constexpr int kTcThreads = 256;  // two warps per TMEM lane quarter, one per column half
constexpr uint32_t kTcTileBytes = 128 * 256;  // 128 rows x 128 bf16
constexpr uint32_t kTcCols = 256;             // two accumulators

// byte offset of 16-byte chunk cc (0..15) of row r in a K-major 128B-swizzled
// tile: two K-blocks of 64 elements, 128 bytes per row, chunks XOR-ed with the
// row's low 3 bits inside each 8-row, 1024-byte atom
__device__ __forceinline__ uint32_t tc_off(int r, int cc) {
    return (uint32_t)((cc >> 3) * (128 * 128) + r * 128 + (((cc & 7) ^ (r & 7)) << 4));
}

// UMMA shared-memory descriptor of the K-major SW128 tile at `addr` (1024-byte
// aligned atoms; the 8-row groups 1024 bytes apart), for the 16-element K step
// `ks`: start address, stride byte offset 1024, version 1, layout SWIZZLE_128B
__device__ __forceinline__ uint64_t tc_desc(uint32_t tile_addr, int ks) {
    const uint32_t a = tile_addr + (uint32_t)(ks >> 2) * (128 * 128) + (uint32_t)(ks & 3) * 32;
    return (uint64_t)((a >> 4) & 0x3fff) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// instruction descriptor: fp32 accumulate, bf16 A and B, both K-major, N = 128, M = 128
constexpr uint32_t kTcIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t da, uint64_t db, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        :
        : "r"(d_tmem), "l"(da), "l"(db), "r"(kTcIdesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 32 consecutive fp32 accumulator columns of this thread's TMEM lane (the
// caller waits for the load with tc_wait_ld)
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// Wait for this thread's TMEM loads.  The registers pass through the asm
// ("+r"), so no use of them can be scheduled before the wait.
__device__ __forceinline__ void tc_wait_ld(uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.wait::ld.sync.aligned;"
        : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
          "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
          "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]),
          "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
          "+r"(r[30]), "+r"(r[31])
        :
        : "memory");
}

// TMA: one box of the 3-D key tensor [head][token][channel] (64 channels x
// 128 tokens, 128-byte swizzle) into shared memory, completion counted on
// `bar`.  x = channel offset (0 or 64: 128-byte aligned), y = first token
// (tokens past S read as zero), z = head.  No multicast.
__device__ __forceinline__ void tma_load_keys(uint32_t dst, const CUtensorMap *tm, int x, int y, int z,
                                              uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

template <int kMode>
__global__ void __launch_bounds__(kTcThreads, 2)
    snap_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __nv_bfloat16 *__restrict__ q_obs, int S,
                   int G, int W, int nsplit, float *__restrict__ ml, float *__restrict__ scores,
                   uint32_t *__restrict__ status) {
    extern __shared__ unsigned char sm_raw[];
    __shared__ uint64_t bars[2];  // accumulator b complete (MMA commit)
    __shared__ uint64_t full[2];  // key buffer b landed (TMA)
    __shared__ uint32_t tmem_base_s;
    __shared__ __align__(16) float rowb[kSnapMaxRows];  // pass 1: m + log2(l) of each window row (+inf past R)
    __shared__ float half_a[kSnapMaxRows], half_b[kSnapMaxRows];  // the upper column half's partial results
    __shared__ float half_p[2][kSnapMaxRows];  // pass 1: upper-half sums, one buffer per tile parity
    __shared__ int fail_s;
    // 1024-byte aligned tiles: queries, then two key buffers
    const uint32_t base = (smem_u32(sm_raw) + 1023u) & ~1023u;
    const uint32_t sq = base, sk0 = base + kTcTileBytes;

    const long bh = blockIdx.x / nsplit;
    const int split = blockIdx.x % nsplit;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int R = G * W;
    const long P = (long)S - W;
    const __nv_bfloat16 *qb = q_obs + (size_t)bh * R * kD;
    const int ntile = (S + kTcKeys - 1) / kTcKeys;
    const int per = (ntile + nsplit - 1) / nsplit;
    const int tile_lo = min(ntile, split * per), tile_hi = min(ntile, tile_lo + per);
    float *mlh = ml + (size_t)bh * nsplit * kSnapMaxRows * 2;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_s)),
                     "r"(kTcCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        mbar_init(smem_u32(&bars[0]), 1);
        mbar_init(smem_u32(&bars[1]), 1);
        mbar_init(smem_u32(&full[0]), 1);
        mbar_init(smem_u32(&full[1]), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fail_s = 0;
    }
    // queries (rows past R are zero)
    for (int i = tid; i < 128 * 16; i += kTcThreads) {
        const int r = i >> 4, cc = i & 15;
        cp_async16(sq + tc_off(r, cc), qb + (size_t)min(r, R - 1) * kD + cc * 8, r < R);
    }
    // one thread fetches a key tile: two TMA boxes (channels 0-63, 64-127),
    // which land in the two K-blocks of the swizzled tile
    auto load_tile = [&](int tile) {
        const uint32_t dst = sk0 + (uint32_t)(tile & 1) * kTcTileBytes;
        const uint32_t fb = smem_u32(&full[tile & 1]);
        mbar_expect_tx(fb, kTcTileBytes);
        tma_load_keys(dst, &tmap_k, 0, tile * kTcKeys, (int)bh, fb);
        tma_load_keys(dst + 128 * 128, &tmap_k, 64, tile * kTcKeys, (int)bh, fb);
    };
    // parity of the use of buffer / accumulator `tile & 1` that `tile` makes
    auto use_parity = [&](int tile) -> uint32_t { return (uint32_t)(((tile - tile_lo) >> 1) & 1); };
    if (kMode == 1) {
        // merged row statistics in split order (split 0 holds key 0, which
        // every row sees); rows past R contribute nothing (1 / l = 0)
        if (tid < kSnapMaxRows) {
            float m = -INFINITY, l = 0.f;
            if (tid < R) {
                for (int sp = 0; sp < nsplit; ++sp) {
                    const float ma = mlh[((size_t)sp * kSnapMaxRows + tid) * 2];
                    const float la = mlh[((size_t)sp * kSnapMaxRows + tid) * 2 + 1];
                    const float n = fmaxf(m, ma);
                    l = (m == -INFINITY ? 0.f : l * exp2f(m - n)) + (ma == -INFINITY ? 0.f : la * exp2f(ma - n));
                    m = n;
                }
            }
            // p = 2^(x - m) / l = 2^(x - (m + log2 l)): one exponent per score
            rowb[tid] = (tid < R && l > 0.f) ? m + log2f(l) : INFINITY;
        }
    }
    cp_async_commit();  // the queries
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();  // barrier initialisation and the TMEM address are visible
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tmem_base_s;
    int loaded_hi = tile_lo, waited_hi = tile_lo;  // thread 0: tiles fetched / whose fetch it waited for
    if (tid == 0) {
        if (tile_lo < tile_hi) load_tile(tile_lo);
        if (tile_lo + 1 < tile_hi) load_tile(tile_lo + 1);
        loaded_hi = min(tile_hi, tile_lo + 2);
    }

    // MMA of `tile` into accumulator tile & 1: pass 0 A = queries, B = keys;
    // pass 1 A = keys, B = queries
    auto issue = [&](int tile) {
        if (tid == 0) {
            const uint32_t kt = sk0 + (uint32_t)(tile & 1) * kTcTileBytes;
            const uint32_t a_t = kMode == 0 ? sq : kt, b_t = kMode == 0 ? kt : sq;
            const uint32_t d = tmem + (uint32_t)(tile & 1) * 128u;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) tc_mma(d, tc_desc(a_t, ks), tc_desc(b_t, ks), ks > 0 ? 1u : 0u);
            tc_commit(smem_u32(&bars[tile & 1]));
        }
    };
    // the queries landed: make them visible to the tensor core's proxy; the
    // MMA issuer waits for each key tile's TMA on its own
    cp_async_wait<0>();
    fence_proxy_async_smem();
    __syncthreads();
    bool failed = false;
    if (tile_lo < tile_hi && tid == 0) {
        if (mbar_wait_limit(smem_u32(&full[tile_lo & 1]), 0u, 1000000000ull)) {
            waited_hi = tile_lo + 1;
            issue(tile_lo);
        } else {
            failed = true;
        }
    }

    const int row = 32 * (warp & 3) + (tid & 31);  // this thread's TMEM lane
    const int chalf = warp >> 2;                    // its column half
    float m_run = -INFINITY, l_run = 0.f;          // pass 0: this window row's statistics
    const long lim_row = P + (row % W);
    // One CTA barrier per tile, at its end: the epilogue is done (its
    // accumulator and key buffer may be reused), the copies of the tile after
    // next have landed and are visible to the tensor core, and the threads
    // agree on any timed-out wait.
    for (int tile = tile_lo; tile < tile_hi; ++tile) {
        // the next tile's keys landed: issue its MMA before this tile's
        // epilogue (its accumulator was freed by the previous barrier)
        if (tid == 0 && tile + 1 < tile_hi && !failed) {
            if (mbar_wait_limit(smem_u32(&full[(tile + 1) & 1]), use_parity(tile + 1), 1000000000ull)) {
                waited_hi = tile + 2;
                issue(tile + 1);
            } else {
                failed = true;
            }
        }
        // this tile's accumulator is complete
        const bool ok = mbar_wait_limit(smem_u32(&bars[tile & 1]), use_parity(tile), 1000000000ull);
        if (!__all_sync(0xffffffffu, ok)) failed = true;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        // its key buffer is free (the MMA read it): fetch the tile after next
        if (tid == 0 && tile + 2 < tile_hi && !failed) {
            load_tile(tile + 2);
            loaded_hi = tile + 3;
        }
        const uint32_t taddr =
            tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(tile & 1) * 128u + (uint32_t)(64 * chalf);
        const long t0 = (long)tile * kTcKeys;
        float acc_lo = 0.f;  // pass 1: this key's lower-half sum (added after the barrier)
        if (failed) {
            // skip the epilogue; the barrier below ends the loop
        } else if (kMode == 0) {
            // S[row][key]: this row's logits for the tile's 128 keys
            const bool mask = t0 + kTcKeys - 1 > P;
            // both 32-column chunks in flight before one wait
            uint32_t rr[2][32];
            tc_ld32(taddr, rr[0]);
            tc_ld32(taddr + 32u, rr[1]);
            tc_wait_ld(rr[0]);  // waits for both loads
            tc_wait_ld(rr[1]);  // (already complete: orders the second chunk's uses)
#pragma unroll
            for (int c0 = 0; c0 < kTcKeys / 2; c0 += 32) {
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(rr[c0 >> 5][i]);
                if (mask) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const long t = t0 + 64 * chalf + c0 + i;
                        v[i] = (t <= lim_row && t < S) ? v[i] : -INFINITY;
                    }
                }
                float x = -INFINITY;
#pragma unroll
                for (int i = 0; i < 32; ++i) x = fmaxf(x, v[i]);
                const float n = fmaxf(m_run, x * kSnapScale);
                const float b = n == -INFINITY ? 0.f : n;
                float s = 0.f;
#pragma unroll
                for (int i = 0; i < 32; ++i) s += ex2_fast(fmaf(v[i], kSnapScale, -b));
                l_run = (m_run == -INFINITY ? 0.f : l_run * exp2f(m_run - n)) + s;
                m_run = n;
            }
        } else {
            // S^T[key][row]: this key's probabilities over the window rows
            float acc = 0.f;
            uint32_t rr[2][32];
            tc_ld32(taddr, rr[0]);
            tc_ld32(taddr + 32u, rr[1]);
            tc_wait_ld(rr[0]);  // waits for both loads
            tc_wait_ld(rr[1]);  // (already complete: orders the second chunk's uses)
#pragma unroll
            for (int c0 = 0; c0 < kSnapMaxRows / 2; c0 += 32) {
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(rr[c0 >> 5][i]);
                // the warp reads the same biases: 16-byte broadcasts
                const float4 *rb = reinterpret_cast<const float4 *>(rowb + 64 * chalf + c0);
#pragma unroll
                for (int i4 = 0; i4 < 8; ++i4) {
                    const float4 b = rb[i4];
                    acc += ex2_fast(fmaf(v[4 * i4 + 0], kSnapScale, -b.x));
                    acc += ex2_fast(fmaf(v[4 * i4 + 1], kSnapScale, -b.y));
                    acc += ex2_fast(fmaf(v[4 * i4 + 2], kSnapScale, -b.z));
                    acc += ex2_fast(fmaf(v[4 * i4 + 3], kSnapScale, -b.w));
                }
            }
            // lower half + upper half, in that order (after the barrier)
            if (chalf == 1) half_p[tile & 1][row] = acc;
            acc_lo = acc;
        }
        // accumulator tile & 1 may be reused; the threads agree on timeouts
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        if (__syncthreads_or(failed ? 1 : 0)) {
            failed = true;
            break;
        }
        if (kMode == 1) {
            // half_p[tile & 1] is rewritten two tiles on, after the next barrier
            const long t = t0 + row;
            if (chalf == 0 && t < P) scores[(size_t)bh * (P > 0 ? P : 0) + t] = acc_lo + half_p[tile & 1][row];
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    }
    cp_async_wait<0>();
    if (failed && tid == 0) atomicOr(status, kDevTimeout);
    if (kMode == 0) {
        // merge the two column halves of each row (lower half first)
        if (chalf == 1) {
            half_a[row] = m_run;
            half_b[row] = l_run;
        }
        __syncthreads();
        if (chalf == 0 && !failed && row < R) {
            const float mb = half_a[row], lb = half_b[row];
            const float n = fmaxf(m_run, mb);
            const float l = (m_run == -INFINITY ? 0.f : l_run * exp2f(m_run - n)) +
                            (mb == -INFINITY ? 0.f : lb * exp2f(mb - n));
            mlh[((size_t)split * kSnapMaxRows + row) * 2] = n;
            mlh[((size_t)split * kSnapMaxRows + row) * 2 + 1] = l;
        }
    }
    // release the tensor memory (a timed-out MMA is waited for once more,
    // with a bound, before the columns are freed)
    if (failed && tid == 0) {
        for (int b = 0; b < 2; ++b) (void)mbar_wait_limit(smem_u32(&bars[b]), 0u, 1000000ull);
        // key tiles still in flight land before the CTA leaves
        for (int t = waited_hi; t < loaded_hi; ++t)
            (void)mbar_wait_limit(smem_u32(&full[t & 1]), use_parity(t), 1000000ull);
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcCols));
    }
}

size_t snapkv_tc_smem_bytes() { return 3 * (size_t)kTcTileBytes + 1024; }

// CTAs per head: about six waves of two CTAs per SM over the whole launch,
// at least four 128-key tiles per CTA, at most kSnapMaxSplit
int snapkv_splits(long BH, int S, int num_sms) {
    const int ntile = (S + kTcKeys - 1) / kTcKeys;
    long ns = (12L * num_sms + BH - 1) / (BH > 0 ? BH : 1);
    ns = std::min<long>(ns, kSnapMaxSplit);
    ns = std::min<long>(ns, std::max(1, ntile / 4));
    return (int)std::max<long>(ns, 1);
}

size_t snapkv_partials_bytes(long BH) { return (size_t)BH * kSnapMaxSplit * kSnapMaxRows * 2 * sizeof(float); }

// cuTensorMapEncodeTiled, fetched from the driver through the runtime (no
// link-time dependency on the driver library)
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// Keys as a 3-D tensor [head][token][channel] of bf16; one box is 64
// channels (128 bytes, the swizzle span) x 128 tokens of one head.  Tokens
// past S are out of bounds and read as zero.
static bool make_key_map(CUtensorMap *tm, const void *k, long BH, int S) {
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)S, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)S * kD * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)kTcKeys, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(k), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_snapkv(const void *k, const void *v, const void *q_obs, long BH, int S, int G, int W, int keep,
                          int pool, void *k_out, void *v_out, int *idx_out, void *ws, cudaStream_t st,
                          const int32_t *keep_rows, int Hkv, int keep_cap) {
    const long P = (long)S - W;
    float *scores = reinterpret_cast<float *>(static_cast<char *>(ws) + kWsHeader);
    uint32_t *pooled = reinterpret_cast<uint32_t *>(scores + (size_t)BH * P);
    float *ml = reinterpret_cast<float *>(pooled + (size_t)BH * P);
    const size_t smem = snapkv_tc_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(snap_tc_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(snap_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const int ns = snapkv_splits(BH, S, nsm);
    const __nv_bfloat16 *qb = static_cast<const __nv_bfloat16 *>(q_obs);
    uint32_t *status = static_cast<uint32_t *>(ws);
    CUtensorMap tmap;
    if (!make_key_map(&tmap, k, BH, S)) return cudaErrorInvalidValue;
    snap_tc_kernel<0><<<(unsigned)(BH * ns), kTcThreads, smem, st>>>(tmap, qb, S, G, W, ns, ml, scores, status);
    snap_tc_kernel<1><<<(unsigned)(BH * ns), kTcThreads, smem, st>>>(tmap, qb, S, G, W, ns, ml, scores, status);
    if (!keep_rows) keep_cap = keep;
    snap_select_kernel<<<(unsigned)BH, kSelThreads, 0, st>>>(scores, pooled, S, W, keep, pool, idx_out, keep_rows,
                                                              Hkv, keep_cap, status);
    const int row_vec = kD * 2 / 16;  // bf16 rows
    const int rows_per_cta = 256 / row_vec;
    snap_gather_kernel<<<dim3((unsigned)((keep_cap + rows_per_cta - 1) / rows_per_cta), (unsigned)BH), 256, 0,
                         st>>>(static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), idx_out, S, W, keep,
                               row_vec, static_cast<uint4 *>(k_out), static_cast<uint4 *>(v_out), keep_rows, Hkv,
                               keep_cap);
    return cudaGetLastError();
}

}  // namespace spark
