// Fused lightning-indexer score -> per-query top-k
// (cf-1.com/news/5231315 §3.1: each query keeps the top-k compressed entries
// by index score; §3.4: the indexer's QK runs in FP4; §4.4: the index score is
// BF16, which makes the selector's cost its score bytes).
//
// The result is exactly topk_select applied to the BF16 scores indexer_score
// writes: the same FP4 MMA, the same fp32 head sum (fmaf over heads in order,
// weights pre-multiplied by the global scales), the same RNE rounding to BF16,
// equal keys for +0 and -0, the same tie rule (equal scores -> smaller index)
// and ascending output.  The score matrix never leaves the SM.
//
// A persistent CTA per SM walks groups of kG = 8 consecutive query rows of one
// sequence (longest rows first):
//   phase 1  a producer warp streams the visible FP4 key rows in chunks of 256
//            entries (TMA, two K halves of 256 rows x 16 B each, in the
//            no-swizzle K-major layout; the scale bytes by cp.async), an MMA
//            thread runs two M = 128 block-scaled FP4 MMAs per chunk with the
//            8 rows' HI heads as N, and 16 epilogue warps turn the fp32
//            accumulators into 16-bit order-preserving keys of the BF16 scores
//            in shared memory ([row][entry]) and record each row's largest key;
//   phase 2  two warps per row: each histograms (max - key) over its half of
//            the row's keys for the 512 keys below the row's largest; the
//            combined histogram gives the k-th largest key K exactly and how
//            many keys == K to take (when fewer than k keys lie in the window
//            it moves down to the largest key below it, at most 128 times);
//            each warp then writes its half's selections in index order (one
//            warp scan of per-lane counts per 256 keys).
// The producer and the MMA thread run ahead into the next group (its query
// tile, key chunks and first accumulators) while the epilogue warps select.
//
// Rows whose visible count n is at most k take all of 0 .. n-1 (then -1),
// like topk_select.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace csa::ixk {

constexpr int kG = 8;                    // query rows per group
constexpr int kCW = 16;                  // epilogue / selection warps
constexpr int kProd = 16, kMma = 17;     // warp roles
constexpr int kThreads = 18 * 32;
constexpr int kChunk = 256;              // entries per chunk (two MMA tiles)
constexpr int kBins = 512;               // selection window (keys)
constexpr int kStages = 8;
constexpr int kHalfBytes = kChunk * 16;  // one K half (32 FP4 values) of a chunk's 256 key rows
constexpr int kSfBytes = 512;            // scale bytes of one 128-entry tile
constexpr int kStageBytes = 2 * kHalfBytes + 2 * kSfBytes;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColSf = 384;         // scale-factor columns follow the accumulators
constexpr int kMaxWindowMoves = 65536 / kBins;

template <int HI> struct Shape {
  static constexpr int N = kG * HI;                   // MMA N: the group's (row, head) pairs
  static constexpr int NACC = HI <= 4 ? 6 : 3;        // chunks whose accumulators are in flight
  static constexpr int CPW = 2 * HI;                  // TMEM columns per epilogue warp and tile
  static_assert(NACC * 2 * N <= static_cast<int>(kColSf), "accumulators fit below the scale columns");
};

struct Args {
  const uint8_t* q_fp4;
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  const float* w;
  float g;
  int T, row0, T_chunk, S, k_bstride, m, k;
  const int32_t* q_pos0;
  int32_t* idx;
  int n_qtiles, n_groups, npad;
  int* status;
  unsigned long long wait_ns;
};

struct __align__(1024) Smem {
  uint8_t ring[kStages][kStageBytes];     // key halves [2][256][16 B], then two tiles' scales
  uint32_t hist[kCW][kBins / 2];          // selection histograms, one per warp (16-bit counters)
  uint8_t qB[2][64 * 32];                 // query tiles (B operand, N <= 64 rows), double-buffered
  uint8_t sfb[2][512];
  uint32_t rmax[2][kCW][2];               // [group parity][warp][row of the warp's pair]: largest key
  uint32_t pmax[kG][2];                   // window moves: each half's largest key below the window
  float wbuf[2][kG * 8];                  // [group parity][row * HI + head]: head weights x global scales
  uint64_t full[kStages], empty[kStages], acc_full[8], acc_empty[8], q_full[2], q_empty[2], drain;
  uint32_t tmem;
  int abort_flag;
};

__device__ __forceinline__ uint32_t cm_off(int r, int c16) { return (r >> 3) * 256 + c16 * 128 + (r & 7) * 16; }
__device__ __forceinline__ uint32_t sf_off(int r) { return (r & 31) * 16 + (r >> 5) * 4; }

__device__ __forceinline__ bool try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
      : "memory");
  return ok != 0;
}
// Bounded wait of one thread; false if another role aborted or the limit passed.
__device__ __noinline__ bool wait1(uint64_t* bar, uint32_t parity, const Args& a, volatile int* abort_flag,
                                   int site) {
  if (try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_ns() - t0 > a.wait_ns) break;
  }
  atomicCAS(a.status, 0, CSA_ERR_TIMEOUT | (site << 8));
  *abort_flag = 1;
  return false;
}
__device__ __forceinline__ bool waitw(uint64_t* bar, uint32_t parity, const Args& a, volatile int* abort_flag,
                                      int site) {
  const bool ok = wait1(bar, parity, a, abort_flag, site);
  return __all_sync(0xffffffffu, ok);
}
// Exit-time wait with a fixed short limit.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!try_wait(bar, parity))
    if (global_ns() - t0 > 1000000ull) break;
}

// TMA 4D tiled load (no multicast) -> smem, completing on `bar`.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int x0, int x1, int x2, int x3,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
      "%5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x0), "r"(x1), "r"(x2), "r"(x3), "r"(smem_u32(bar))
      : "memory");
}

#define CSA_TMEM_LD_X8(taddr, r)                                                                       \
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"              \
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), \
                 "=r"(r[7])                                                                            \
               : "r"(taddr))

// Ties registers to this point of the program: reads of r after it cannot be
// scheduled before the tcgen05.wait::ld that precedes it.
template <int NR>
__device__ __forceinline__ void reg_fence(uint32_t (&r)[NR]) {
#pragma unroll
  for (int i = 0; i < NR; ++i) asm volatile("" : "+r"(r[i]));
}

// Two BF16 values (RNE of lo, hi) as order-preserving 16-bit keys in one word:
// key = 0x8000 + magnitude for x >= 0, 0x8000 - magnitude for x < 0 (so -0 and
// +0 share 0x8000 and every finite value maps above 0, the padding key).
__device__ __forceinline__ uint32_t score_keys2(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  const uint32_t u = *reinterpret_cast<const uint32_t*>(&b);
  const uint32_t mag = u & 0x7FFF7FFFu;
  const uint32_t neg = ((u >> 15) & 0x00010001u) * 0xFFFFu;
  return 0x80008000u + (mag & ~neg) - (mag & neg);
}
__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Group gi -> (sequence, row tile), the tiles with the most visible entries first.
struct Group {
  int bi, tq0, ntok, nch, n_min;
  long long pbase;
};
__device__ __forceinline__ int visible(long long pbase, int t, const Args& a) {
  long long v = (pbase + t + 1) / a.m;
  if (v > a.S) v = a.S;
  if (v < 0) v = 0;
  return static_cast<int>(v);
}
__device__ __forceinline__ Group group_of(int gi, const Args& a) {
  Group gr;
  gr.bi = gi / a.n_qtiles;
  const int qt = a.n_qtiles - 1 - (gi - gr.bi * a.n_qtiles);
  gr.tq0 = qt * kG;
  gr.ntok = min(kG, a.T_chunk - gr.tq0);
  gr.pbase = static_cast<long long>(a.q_pos0[gr.bi]) + a.row0 + gr.tq0;
  const int n_last = visible(gr.pbase, gr.ntok - 1, a);
  gr.nch = (n_last + kChunk - 1) / kChunk;
  gr.n_min = visible(gr.pbase, 0, a);
  return gr;
}

// ---------------------------------------------------------------- selection
// Histograms count keys by d = anchor - key in kBins bins, two 16-bit counters
// per word (bin d in word d / 2, half d % 2).  Lane L of a warp owns bins
// [16 L, 16 L + 16) when scanning.
struct BinHit {
  int bin;       // first bin at which the running count of both halves reaches the target, -1 if none
  int before;    // both halves' keys in bins before it
  int beforeA;   // half 0's keys in bins before it
  int atA;       // half 0's keys in it
  int total, totalA;
};
__device__ __forceinline__ int lo16(uint32_t w) { return static_cast<int>(w & 0xFFFFu); }
__device__ __forceinline__ int hi16(uint32_t w) { return static_cast<int>(w >> 16); }

__device__ __forceinline__ BinHit find_bin(const uint32_t* hA, const uint32_t* hB, int target, int lane) {
  int cA = 0, cB = 0;
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    const int wd = 8 * lane + ((b + (lane >> 2)) & 7);   // rotated: no bank conflicts
    const uint32_t a = hA[wd], c = hB[wd];
    cA += lo16(a) + hi16(a);
    cB += lo16(c) + hi16(c);
  }
  const int cnt = cA + cB;
  const int incl = warp_incl_scan(cnt);
  const int inclA = warp_incl_scan(cA);
  const int excl = incl - cnt, exclA = inclA - cA;
  BinHit r{-1, 0, 0, 0, __shfl_sync(0xffffffffu, incl, 31), __shfl_sync(0xffffffffu, inclA, 31)};
  const unsigned bl = __ballot_sync(0xffffffffu, excl < target && target <= incl);
  if (bl == 0) return r;
  const int fl = __ffs(bl) - 1;
  int dd = 0, cb = 0, ga = 0, ea = 0;
  if (lane == fl) {
    int run = excl, runA = exclA;
    for (int b = 0; b < 16; ++b) {
      const uint32_t a = hA[8 * lane + (b >> 1)], c = hB[8 * lane + (b >> 1)];
      const int na = (b & 1) ? hi16(a) : lo16(a);
      const int h = na + ((b & 1) ? hi16(c) : lo16(c));
      if (run + h >= target) {
        dd = 16 * lane + b;
        cb = run;
        ga = runA;
        ea = na;
        break;
      }
      run += h;
      runA += na;
    }
  }
  r.bin = __shfl_sync(0xffffffffu, dd, fl);
  r.before = __shfl_sync(0xffffffffu, cb, fl);
  r.beforeA = __shfl_sync(0xffffffffu, ga, fl);
  r.atA = __shfl_sync(0xffffffffu, ea, fl);
  return r;
}

// Phase 2 for row t (n > k visible keys) by the warp pair hf = 0, 1, each on
// its half of the row's chunks; lane L reads keys 8 L .. 8 L + 7 of a chunk.
// Keys at e >= n are 0 (padding); the window never reaches key 0.
__device__ __forceinline__ void select_row(Smem& sm, const uint16_t* __restrict__ row, int n, int t, int hf,
                                           uint32_t anchor, int32_t* __restrict__ out, const Args& a, int lane) {
  const int k = a.k;
  const int nchr = (n + kChunk - 1) / kChunk;
  const int h0 = (nchr + 1) >> 1;
  const int c0 = hf ? h0 : 0, c1 = hf ? nchr : h0;
  uint32_t* hist = sm.hist[2 * t + hf];
  const uint32_t* hA = sm.hist[2 * t];        // half 0
  const uint32_t* hB = sm.hist[2 * t + 1];    // half 1
  const int bar_id = 2 + t;
  // K = anchor - D; G keys > K in the row, G0 of them and E0 keys == K in half 0
  int krem = k, above0 = 0;
  int D = -1, G = 0, G0 = 0, E0 = 0;
#pragma unroll 1
  for (int it = 0; it < kMaxWindowMoves && D < 0; ++it) {
#pragma unroll
    for (int i = 0; i < kBins / 64; ++i) hist[i * 32 + lane] = 0u;
    __syncwarp();
    // window [anchor - nb + 1, anchor]; nb <= anchor keeps the padding key 0 out
    const uint32_t nb = anchor < static_cast<uint32_t>(kBins) ? anchor : static_cast<uint32_t>(kBins);
#pragma unroll 2
    for (int c = c0; c < c1; ++c) {
      const uint4 u = *reinterpret_cast<const uint4*>(row + c * kChunk + 8 * lane);
      const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t d0 = anchor - (wv[j] & 0xFFFFu), d1 = anchor - (wv[j] >> 16);
        if (d0 < nb) atomicAdd(&hist[d0 >> 1], 1u << ((d0 & 1u) << 4));
        if (d1 < nb) atomicAdd(&hist[d1 >> 1], 1u << ((d1 & 1u) << 4));
      }
    }
    named_bar_sync(bar_id, 64);
    const BinHit hit = find_bin(hA, hB, krem, lane);
    if (hit.bin >= 0) {
      D = hit.bin;
      G = (k - krem) + hit.before;
      G0 = above0 + hit.beforeA;
      E0 = hit.atA;
    } else {
      // fewer than krem keys in the window: move it down to the largest key below
      krem -= hit.total;
      above0 += hit.totalA;
      const uint32_t lo = anchor - nb;
      uint32_t mx = 0;
#pragma unroll 2
      for (int c = c0; c < c1; ++c) {
        const uint4 u = *reinterpret_cast<const uint4*>(row + c * kChunk + 8 * lane);
        const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t k0 = wv[j] & 0xFFFFu, k1 = wv[j] >> 16;
          if (k0 <= lo) mx = max(mx, k0);
          if (k1 <= lo) mx = max(mx, k1);
        }
      }
      mx = __reduce_max_sync(0xffffffffu, mx);
      if (lane == 0) sm.pmax[t][hf] = mx;
      named_bar_sync(bar_id, 64);   // also: both warps are done reading the histograms
      anchor = max(sm.pmax[t][0], sm.pmax[t][1]);
    }
  }
  if (D < 0) {   // unreachable: the window reaches every key within kMaxWindowMoves moves
    if (lane == 0) atomicCAS(a.status, 0, CSA_ERR_UNSUPPORTED);
    return;
  }
  // ---- every key > K, and the first take_eq keys == K in index order
  const uint32_t K = anchor - static_cast<uint32_t>(D);
  const int take_eq = k - G;
  // half 1 starts after half 0's selections: its keys > K and its share of the == K ones
  int pos = hf ? G0 + min(E0, take_eq) : 0;
  int eq_seen = hf ? E0 : 0;
#pragma unroll 2
  for (int c = c0; c < c1; ++c) {
    const uint4 u = *reinterpret_cast<const uint4*>(row + c * kChunk + 8 * lane);
    const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
    uint32_t gtm = 0, eqm = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t key = (j & 1) ? (wv[j >> 1] >> 16) : (wv[j >> 1] & 0xFFFFu);
      gtm |= static_cast<uint32_t>(key > K) << j;
      eqm |= static_cast<uint32_t>(key == K) << j;
    }
    const int cg = __popc(gtm), ce = __popc(eqm);
    const int packed = cg | (ce << 16);
    const int incl = warp_incl_scan(packed);
    const int excl = incl - packed;
    const int tot = __shfl_sync(0xffffffffu, incl, 31);
    const int eq_before = eq_seen + (excl >> 16);
    const int take_mine = max(0, min(ce, take_eq - eq_before));
    int p = pos + (excl & 0xFFFF) + max(0, min(excl >> 16, take_eq - eq_seen));
    uint32_t em = eqm, sel = gtm;
    for (int i = 0; i < take_mine; ++i) {
      const uint32_t lowest = em & (0u - em);
      sel |= lowest;
      em ^= lowest;
    }
    const int e0 = c * kChunk + 8 * lane;
    while (sel) {
      const int j = __ffs(sel) - 1;
      out[p++] = e0 + j;
      sel &= sel - 1;
    }
    pos += (tot & 0xFFFF) + max(0, min(tot >> 16, take_eq - eq_seen));
    eq_seen += tot >> 16;
  }
}

template <int HI>
__global__ void __launch_bounds__(kThreads, 1) indexer_topk_kernel(const __grid_constant__ Args args,
                                                                   const __grid_constant__ CUtensorMap kmap) {
  using Sh = Shape<HI>;
  constexpr int N = Sh::N, NACC = Sh::NACC, CPW = Sh::CPW;
  const Args& a = args;
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  Smem& sm = *reinterpret_cast<Smem*>(dsm);
  uint16_t* keys = reinterpret_cast<uint16_t*>(dsm + sizeof(Smem));
  volatile int* abort_flag = &sm.abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == kMma) {
    tmem_alloc(&sm.tmem, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 33);          // 32 cp.async arrivals + the TMA byte count
      mbar_init(&sm.empty[s], 1);
    }
    for (int s = 0; s < NACC; ++s) {
      mbar_init(&sm.acc_full[s], 1);
      mbar_init(&sm.acc_empty[s], kCW);      // one arrive per epilogue warp
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.q_full[s], 32);
      mbar_init(&sm.q_empty[s], 1);
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  // scale words of query rows N .. 127 stay zero
  for (int i = tid; i < 2 * 128; i += kThreads) {
    const int n = i & 127;
    if (n >= N) *reinterpret_cast<uint32_t*>(sm.sfb[i >> 7] + sf_off(n)) = 0u;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem;

  if (warp == kProd) {
    // ---- producer: query tile per group, key chunks through the ring
    int gc = 0, j = 0, armed = -1;
#pragma unroll 1
    for (int gi = blockIdx.x; gi < a.n_groups; gi += gridDim.x, ++j) {
      const Group gr = group_of(gi, a);
      const int b = j & 1;
      if (j >= 2 && !waitw(&sm.q_empty[b], ((j >> 1) - 1) & 1, a, abort_flag, 1)) break;
      for (int n = lane; n < N; n += 32) {
        const int t = n / HI;
        const bool ok = t < gr.ntok;
        const size_t qrow = ok ? (static_cast<size_t>(gr.bi) * a.T + a.row0 + gr.tq0 + t) * HI + (n - t * HI) : 0;
        cp_async16(smem_u32(sm.qB[b] + cm_off(n, 0)), a.q_fp4 + qrow * 32, ok ? 16u : 0u);
        cp_async16(smem_u32(sm.qB[b] + cm_off(n, 1)), a.q_fp4 + qrow * 32 + 16, ok ? 16u : 0u);
        cp_async4(smem_u32(sm.sfb[b] + sf_off(n)), a.q_sf + qrow * 4, ok ? 4u : 0u);
      }
      cp_async_mbar_arrive(&sm.q_full[b]);
      bool ok = true;
#pragma unroll 1
      for (int c = 0; c < gr.nch; ++c, ++gc) {
        const int st = gc % kStages;
        if (gc >= kStages && !waitw(&sm.empty[st], ((gc / kStages) - 1) & 1, a, abort_flag, 2)) {
          ok = false;
          break;
        }
        uint8_t* base = sm.ring[st];
        if (lane == 0) {
          mbar_arrive_expect_tx(&sm.full[st], 2 * kHalfBytes);
          tma_load_4d(smem_u32(base), &kmap, 0, 0, c * kChunk, gr.bi, &sm.full[st]);
          tma_load_4d(smem_u32(base + kHalfBytes), &kmap, 0, 1, c * kChunk, gr.bi, &sm.full[st]);
        }
        armed = gc;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = 32 * i + lane;
          const int s = c * kChunk + r;
          const bool okr = s < a.S;
          const size_t krow = static_cast<size_t>(gr.bi) * a.k_bstride + (okr ? s : 0);
          cp_async4(smem_u32(base + 2 * kHalfBytes + (r >> 7) * kSfBytes + sf_off(r & 127)), a.k_sf + krow * 4,
                    okr ? 4u : 0u);
        }
        cp_async_mbar_arrive(&sm.full[st]);
      }
      if (!ok) break;
    }
    cp_async_commit();
    cp_async_wait<0>();
    // copies still in flight (after an abort) land before the CTA exits
    if (*abort_flag && armed >= 0 && lane == 0) drain_wait(&sm.full[armed % kStages], (armed / kStages) & 1);
    __syncwarp();
  } else if (warp == kMma) {
    // ---- MMA: per chunk two M = 128 tiles into accumulator buffer gc % NACC
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_nvfp4(128, N);
      int gc = 0, j = 0;
      bool ok = true;
#pragma unroll 1
      for (int gi = blockIdx.x; ok && gi < a.n_groups; gi += gridDim.x, ++j) {
        const Group gr = group_of(gi, a);
        const int b = j & 1;
        if (!wait1(&sm.q_full[b], (j >> 1) & 1, a, abort_flag, 3)) break;
        fence_proxy_async();
        tc_fence_after();
        const uint32_t t_sfb = tmem + kColSf + 8 * NACC + 4 * b;
        tmem_cp_32x128b_x4(t_sfb, make_sdesc(smem_u32(sm.sfb[b]), 128, 128, kLayoutNone));
        const uint64_t bdesc = make_sdesc(smem_u32(sm.qB[b]), 128, 256, kLayoutNone);
#pragma unroll 1
        for (int c = 0; c < gr.nch; ++c, ++gc) {
          const int st = gc % kStages, buf = gc % NACC;
          if (!wait1(&sm.full[st], (gc / kStages) & 1, a, abort_flag, 4) ||
              (gc >= NACC && !wait1(&sm.acc_empty[buf], ((gc / NACC) - 1) & 1, a, abort_flag, 5))) {
            ok = false;
            break;
          }
          fence_proxy_async();
          tc_fence_after();
          const uint32_t rb = smem_u32(sm.ring[st]);
#pragma unroll
          for (int jp = 0; jp < 2; ++jp) {
            const uint32_t t_sfa = tmem + kColSf + 8 * buf + 4 * jp;
            tmem_cp_32x128b_x4(t_sfa, make_sdesc(rb + 2 * kHalfBytes + jp * kSfBytes, 128, 128, kLayoutNone));
            // K halves 4 KB apart (leading byte offset), 8-row groups 128 B apart
            const uint64_t adesc = make_sdesc(rb + jp * 2048, kHalfBytes, 128, kLayoutNone);
            mma_nvfp4(tmem + buf * 2 * N + jp * N, adesc, bdesc, idesc, t_sfa, t_sfb, 0u);
          }
          tc_commit(&sm.empty[st]);
          tc_commit(&sm.acc_full[buf]);
        }
        tc_commit(&sm.q_empty[b]);   // the group's MMAs (the readers of qB[b]) are done
      }
      tc_commit(&sm.drain);
      drain_wait(&sm.drain, 0);
    }
    __syncwarp();
  } else {
    // ---- epilogue / selection warps: warp (q, tp) = lane quarter q, rows 2 tp, 2 tp + 1
    const int q = warp & 3, tp = warp >> 2;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    int gc = 0, j = 0;
    // head weights (times the global scales) of a group's rows, staged in
    // shared memory by warp 0 one group ahead
    auto fetch_w = [&](int gi, int slot) {
      if (warp != 0 || gi >= a.n_groups) return;
      const Group gr = group_of(gi, a);
      for (int i = lane; i < kG * HI; i += 32) {
        const int t = i / HI;
        const bool ok = t < gr.ntok;
        sm.wbuf[slot][i] =
            ok ? a.w[(static_cast<size_t>(gr.bi) * a.T + a.row0 + gr.tq0 + t) * HI + (i - t * HI)] * a.g : 0.f;
      }
    };
    fetch_w(blockIdx.x, 0);
    named_bar_sync(1, 32 * kCW);
    float wr[2][HI];
    bool ok = true;
#pragma unroll 1
    for (int gi = blockIdx.x; gi < a.n_groups; gi += gridDim.x, ++j) {
      const Group gr = group_of(gi, a);
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int h = 0; h < HI; ++h) wr[u][h] = sm.wbuf[j & 1][(2 * tp + u) * HI + h];
      int nv[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) nv[u] = 2 * tp + u < gr.ntok ? visible(gr.pbase, 2 * tp + u, a) : 0;
      uint16_t* krow0 = keys + static_cast<size_t>(2 * tp) * a.npad;
      uint32_t rm[2] = {0u, 0u};
      uint32_t v[2][2][CPW];   // [chunk of the pair][tile][column]
      auto load = [&](int cg, uint32_t (&dst)[2][CPW]) {
        const uint32_t col = tmem + lane_base + (cg % NACC) * 2 * N + tp * CPW;
#pragma unroll
        for (int jp = 0; jp < 2; ++jp) {
          if constexpr (CPW == 8) {
            CSA_TMEM_LD_X8(col + jp * N, dst[jp]);
          } else {
            tmem_ld16(col + jp * N, dst[jp]);
          }
        }
      };
      auto consume = [&](int c, const uint32_t (&src)[2][CPW]) {
        const int e = c * kChunk + 32 * q + lane;           // entries e (tile 0) and e + 128 (tile 1)
        const bool full_chunk = c * kChunk + kChunk <= gr.n_min;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          float a0 = 0.f, a1 = 0.f;
#pragma unroll
          for (int h = 0; h < HI; ++h) {
            a0 = fmaf(wr[u][h], fmaxf(__uint_as_float(src[0][u * HI + h]), 0.f), a0);
            a1 = fmaf(wr[u][h], fmaxf(__uint_as_float(src[1][u * HI + h]), 0.f), a1);
          }
          uint32_t k2 = score_keys2(a0, a1);
          if (!full_chunk) {
            if (e >= nv[u]) k2 &= 0xFFFF0000u;
            if (e + 128 >= nv[u]) k2 &= 0x0000FFFFu;
          }
          rm[u] = vmax_u16x2(rm[u], k2);
          uint16_t* kr = krow0 + static_cast<size_t>(u) * a.npad + e;
          kr[0] = static_cast<uint16_t>(k2 & 0xFFFFu);
          kr[128] = static_cast<uint16_t>(k2 >> 16);
        }
      };
      // two chunks per synchronisation: the later chunk's commit covers both
      // (the MMA thread commits in order), one TMEM load wait for four tiles
      const int nch = gr.nch;
#pragma unroll 1
      for (int c = 0; ok && c < nch; c += 2) {
        const int g0 = gc + c;
        const bool two = c + 1 < nch;
        const int gl = two ? g0 + 1 : g0;
        if (!waitw(&sm.acc_full[gl % NACC], (gl / NACC) & 1, a, abort_flag, 6)) {
          ok = false;
          break;
        }
        tc_fence_after();
        load(g0, v[0]);
        if (two) load(g0 + 1, v[1]);
        tmem_ld_wait();
        reg_fence(v[0][0]);
        reg_fence(v[0][1]);
        reg_fence(v[1][0]);
        reg_fence(v[1][1]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sm.acc_empty[g0 % NACC]);
          if (two) mbar_arrive(&sm.acc_empty[(g0 + 1) % NACC]);
        }
        consume(c, v[0]);
        if (two) consume(c + 1, v[1]);
      }
      gc += nch;
      // each row's largest key: this warp's 32 lanes x 2 tiles
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint32_t m2 = max(rm[u] & 0xFFFFu, rm[u] >> 16);
        const uint32_t mx = __reduce_max_sync(0xffffffffu, m2);
        if (lane == 0) sm.rmax[j & 1][warp][u] = mx;
      }
      named_bar_sync(1, 32 * kCW);
      if (!ok || *abort_flag) break;
      fetch_w(gi + gridDim.x, (j + 1) & 1);
      // ---- phase 2: warps 2 t and 2 t + 1 select row t
      const int t = warp >> 1, hf = warp & 1;
      if (t < gr.ntok) {
        const int n = visible(gr.pbase, t, a);
        int32_t* out = a.idx + (static_cast<size_t>(gr.bi) * a.T_chunk + gr.tq0 + t) * a.k;
        if (n <= a.k) {
          for (int i = lane + 32 * hf; i < a.k; i += 64) out[i] = i < n ? i : -1;
        } else {
          // the row's keys came from the four quarter warps of pair t / 2, slot t & 1
          uint32_t anchor = 0;
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) anchor = max(anchor, sm.rmax[j & 1][4 * (t >> 1) + qq][t & 1]);
          select_row(sm, keys + static_cast<size_t>(t) * a.npad, n, t, hf, anchor, out, a, lane);
        }
      }
      named_bar_sync(1, 32 * kCW);   // keys are rewritten by the next group
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 ixk_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// FP4 key rows [B][k_bstride][32 B] seen as (16 bytes, K half, row, sequence);
// a box is one K half of 256 rows: 256 x 16 B, the no-swizzle K-major layout.
bool key_map(CUtensorMap* m, const void* k_fp4, int B, int k_bstride) {
  auto enc = ixk_encoder();
  if (enc == nullptr) return false;
  const uint64_t rows = static_cast<uint64_t>(k_bstride > 0 ? k_bstride : 1);
  cuuint64_t dims[4] = {16, 2, rows, static_cast<cuuint64_t>(B > 0 ? B : 1)};
  cuuint64_t strides[3] = {16, 32, rows * 32};
  cuuint32_t box[4] = {16, 1, static_cast<cuuint32_t>(kChunk), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(k_fp4), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace csa::ixk

using namespace csa;

extern "C" int indexer_topk_max_entries(int HI, int DI) {
  if (DI != 64 || (HI != 4 && HI != 8)) return 0;
  int dev = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return 0;
  const long long room = static_cast<long long>(optin) - static_cast<long long>(sizeof(ixk::Smem)) - 1024;
  if (room <= 0) return 0;
  return static_cast<int>(room / (2 * ixk::kG) / ixk::kChunk * ixk::kChunk);
}

extern "C" int indexer_topk(const uint8_t* q_fp4, const uint8_t* q_sf, float q_gscale, const uint8_t* k_fp4,
                            const uint8_t* k_sf, float k_gscale, const float* w, int B, int T, int row0,
                            int T_chunk, int S, int k_bstride, int HI, int DI, int m, const int32_t* q_pos0,
                            int32_t* idx, int k, int32_t* status_out, csa_stream_t stream) {
  CSA_REQUIRE(q_fp4 && q_sf && k_fp4 && k_sf && w && q_pos0 && idx, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(B >= 0 && T >= 0 && row0 >= 0 && T_chunk >= 0 && row0 + T_chunk <= T, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(S >= 0 && k_bstride >= S && m >= 1 && k >= 1, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(q_gscale > 0.f && k_gscale > 0.f, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(DI == 64 && (HI == 4 || HI == 8), CSA_ERR_UNSUPPORTED);
  CSA_REQUIRE(aligned16(q_fp4) && aligned16(k_fp4) && (reinterpret_cast<uintptr_t>(k_sf) & 3) == 0 &&
                  (reinterpret_cast<uintptr_t>(q_sf) & 3) == 0,
              CSA_ERR_ALIGNMENT);
  if (B == 0 || T_chunk == 0) return CSA_OK;
  CSA_REQUIRE(S <= indexer_topk_max_entries(HI, DI), CSA_ERR_UNSUPPORTED);
  int dev = 0, optin = 0, n_sm = 0;
  CSA_REQUIRE(cudaGetDevice(&dev) == cudaSuccess, CSA_ERR_CUDA);
  CSA_REQUIRE(cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess,
              CSA_ERR_CUDA);
  CSA_REQUIRE(cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess, CSA_ERR_CUDA);
  ixk::Args a{};
  a.q_fp4 = q_fp4;
  a.q_sf = q_sf;
  a.k_sf = k_sf;
  a.w = w;
  a.g = q_gscale * k_gscale;
  a.T = T;
  a.row0 = row0;
  a.T_chunk = T_chunk;
  a.S = S;
  a.k_bstride = k_bstride;
  a.m = m;
  a.k = k;
  a.q_pos0 = q_pos0;
  a.idx = idx;
  a.n_qtiles = (T_chunk + ixk::kG - 1) / ixk::kG;
  CSA_REQUIRE(static_cast<long long>(B) * a.n_qtiles < (1ll << 31), CSA_ERR_UNSUPPORTED);
  a.n_groups = B * a.n_qtiles;
  a.npad = (S + ixk::kChunk - 1) / ixk::kChunk * ixk::kChunk;
  if (a.npad == 0) a.npad = ixk::kChunk;
  const size_t smem = sizeof(ixk::Smem) + 1024 + static_cast<size_t>(ixk::kG) * a.npad * 2;
  CSA_REQUIRE(smem <= static_cast<size_t>(optin), CSA_ERR_UNSUPPORTED);
  a.status = status_word(status_out);
  CSA_REQUIRE(a.status != nullptr, CSA_ERR_CUDA);
  a.wait_ns = wait_limit_ns();
  CUtensorMap kmap;
  CSA_REQUIRE(ixk::key_map(&kmap, k_fp4, B, k_bstride), CSA_ERR_CUDA);
  const int grid = a.n_groups < n_sm ? a.n_groups : n_sm;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the shared-memory floor (above half an SM) keeps one CTA per SM, so the
  // 512-column TMEM allocation never waits on another CTA
  const size_t smem_launch = smem < 120 * 1024 ? 120 * 1024 : smem;
  if (HI == 4) {
    cudaFuncSetAttribute(ixk::indexer_topk_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem_launch));
    ixk::indexer_topk_kernel<4><<<grid, ixk::kThreads, smem_launch, st>>>(a, kmap);
  } else {
    cudaFuncSetAttribute(ixk::indexer_topk_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem_launch));
    ixk::indexer_topk_kernel<8><<<grid, ixk::kThreads, smem_launch, st>>>(a, kmap);
  }
  return check_launch();
}
