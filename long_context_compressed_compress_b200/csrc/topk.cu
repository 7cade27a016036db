// Per-query top-k selection over the lightning-indexer scores
// (cf-1.com/news/5231315 §3.1: each query picks its top-k compressed entries;
// §4.4: the scores are stored in BF16, which halves the selector's traffic).
//
// Radix select on order-preserving integer keys: a float's bit pattern is
// mapped so that unsigned integer order equals float order (+0 and -0 map to
// the same key); BF16 rows use 16-bit keys, FP32 rows 32-bit keys.  8-bit
// digits are resolved from the top: a 256-bin histogram of the candidates that
// still match the chosen prefix (per-warp shared-memory histograms), one block
// scan over the bins, and the bin holding the k-th largest key fixes the next
// digit.  After the last digit the threshold key K is exact: every key > K is
// selected, plus the (k - #greater) keys == K with the smallest indices.
//
// The output is an in-order compaction: each warp owns a contiguous segment of
// the row and walks it 32 keys at a time with ballots, so indices come out
// ascending, shared-memory reads are conflict-free, and only the warps'
// totals cross a barrier.  Bit-exact and independent of scheduling.
//
// One CTA (128 threads) per query row; the visible prefix of the row is staged
// in shared memory when it fits, otherwise every pass re-reads it from L2.
#include <mutex>

#include "common.cuh"

namespace csa {

constexpr int kTopkThreads = 128;
constexpr int kTopkDpt = 256 / kTopkThreads;   // histogram digits per thread in the scan
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr size_t kTopkSmemMax = 160 * 1024;

template <typename T> struct KeyOf;
template <> struct KeyOf<float> {
  using K = uint32_t;
  static constexpr int bits = 32;
  static __device__ __forceinline__ K get(float x) {
    uint32_t u = __float_as_uint(x);
    if (u == 0x80000000u) u = 0u;                       // -0 == +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  }
};
template <> struct KeyOf<__nv_bfloat16> {
  using K = uint16_t;
  static constexpr int bits = 16;
  static __device__ __forceinline__ K get(__nv_bfloat16 x) {
    uint32_t u = __bfloat16_as_ushort(x);
    if (u == 0x8000u) u = 0u;
    return static_cast<K>((u & 0x8000u) ? (~u & 0xFFFFu) : (u | 0x8000u));
  }
};

// Inclusive scan of one int per thread across the CTA (thread order).
__device__ __forceinline__ int block_incl_scan(int v, int* wsum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int inc = warp_incl_scan(v);
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  int before = 0;
#pragma unroll
  for (int w = 0; w < kTopkWarps; ++w) before += (w < warp) ? wsum[w] : 0;
  __syncthreads();
  return before + inc;
}

template <typename T, bool kSmem>
__global__ void __launch_bounds__(kTopkThreads) topk_row_kernel(const T* __restrict__ score, int T_chunk, int S,
                                                               int ld, int k, int m, int row0,
                                                               const int32_t* __restrict__ q_pos0,
                                                               int32_t* __restrict__ idx) {
  using KO = KeyOf<T>;
  using K = typename KO::K;
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ int hist[kTopkWarps][256];
  __shared__ int wsum[kTopkWarps];
  __shared__ int wcnt[kTopkWarps][2];
  __shared__ int sel_digit, sel_above;

  const int row = blockIdx.x;
  const int bi = row / T_chunk;
  const int r = row - bi * T_chunk;
  const long long p = static_cast<long long>(q_pos0[bi]) + row0 + r;
  long long nv = (p + 1) / m;
  if (nv > S) nv = S;
  if (nv < 0) nv = 0;
  const int n = static_cast<int>(nv);
  int32_t* out = idx + static_cast<size_t>(row) * k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (n <= k) {
    for (int i = tid; i < k; i += kTopkThreads) out[i] = i < n ? i : -1;
    return;
  }
  const T* srow = score + static_cast<size_t>(row) * ld;
  K* keys = reinterpret_cast<K*>(dsm);
  if (kSmem) {
    // 16-byte loads (several in flight per thread), keys stored 16 bytes at a time
    constexpr int V = 16 / sizeof(T);
    int done = 0;
    if ((reinterpret_cast<uintptr_t>(srow) & 15) == 0) {
      const int nvec = n / V;
#pragma unroll 4
      for (int j = tid; j < nvec; j += kTopkThreads) {
        const uint4 u = reinterpret_cast<const uint4*>(srow)[j];
        const T* e = reinterpret_cast<const T*>(&u);
        K kk[V];
#pragma unroll
        for (int q = 0; q < V; ++q) kk[q] = KO::get(e[q]);
        if constexpr (sizeof(K) * V == 16) {
          *reinterpret_cast<uint4*>(keys + static_cast<size_t>(j) * V) = *reinterpret_cast<const uint4*>(kk);
        } else {
#pragma unroll
          for (int q = 0; q < V; ++q) keys[static_cast<size_t>(j) * V + q] = kk[q];
        }
      }
      done = nvec * V;
    }
    for (int i = done + tid; i < n; i += kTopkThreads) keys[i] = KO::get(srow[i]);
    __syncthreads();
  }
  auto key_at = [&](int i) -> K { return kSmem ? keys[i] : KO::get(srow[i]); };

  uint32_t prefix = 0, pmask = 0;
  int krem = k;
#pragma unroll 1
  for (int shift = KO::bits - 8; shift >= 0; shift -= 8) {
#pragma unroll
    for (int w = 0; w < kTopkWarps; ++w)
#pragma unroll
      for (int q = 0; q < kTopkDpt; ++q) hist[w][tid + q * kTopkThreads] = 0;
    __syncthreads();
    for (int base = 0; base < n; base += kTopkThreads) {
      const int i = base + tid;
      const uint32_t key = i < n ? static_cast<uint32_t>(key_at(i)) : 0u;
      const bool cand = i < n && (key & pmask) == prefix;
      const uint32_t dig = (key >> shift) & 0xFFu;
      if (cand) atomicAdd(&hist[warp][dig], 1);
    }
    __syncthreads();
    // thread t owns digits 255 - kTopkDpt t - q (descending): the inclusive scan
    // in thread order counts the candidates with a larger-or-equal digit
    int cq[kTopkDpt], csum = 0;
#pragma unroll
    for (int q = 0; q < kTopkDpt; ++q) {
      const int d = 255 - kTopkDpt * tid - q;
      int c = 0;
#pragma unroll
      for (int w = 0; w < kTopkWarps; ++w) c += hist[w][d];
      cq[q] = c;
      csum += c;
    }
    int above = block_incl_scan(csum, wsum) - csum;
#pragma unroll
    for (int q = 0; q < kTopkDpt; ++q) {
      if (above < krem && krem <= above + cq[q]) {
        sel_digit = 255 - kTopkDpt * tid - q;
        sel_above = above;
      }
      above += cq[q];
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(sel_digit) << shift;
    pmask |= 0xFFu << shift;
    krem -= sel_above;
  }
  // threshold key = prefix; take every key > prefix and the first `krem` keys == prefix.
  const int seg = (n + kTopkWarps * 32 - 1) / (kTopkWarps * 32) * 32;
  const int s0 = warp * seg, s1 = min(n, s0 + seg);
  int n_gt = 0, n_eq = 0;
  for (int b0 = s0; b0 < s1; b0 += 32) {
    const int i = b0 + lane;
    const uint32_t key = i < s1 ? static_cast<uint32_t>(key_at(i)) : 0u;
    n_gt += __popc(__ballot_sync(0xffffffffu, i < s1 && key > prefix));
    n_eq += __popc(__ballot_sync(0xffffffffu, i < s1 && key == prefix));
  }
  if (lane == 0) {
    wcnt[warp][0] = n_gt;
    wcnt[warp][1] = n_eq;
  }
  __syncthreads();
  int out_pos = 0, eq_before = 0;
  for (int w = 0; w < warp; ++w) {
    const int take_eq = max(0, min(wcnt[w][1], krem - eq_before));
    out_pos += wcnt[w][0] + take_eq;
    eq_before += wcnt[w][1];
  }
  const unsigned below = (1u << lane) - 1u;
  for (int b0 = s0; b0 < s1; b0 += 32) {
    const int i = b0 + lane;
    const uint32_t key = i < s1 ? static_cast<uint32_t>(key_at(i)) : 0u;
    const bool gt = i < s1 && key > prefix;
    const bool eq = i < s1 && key == prefix;
    const unsigned eqm = __ballot_sync(0xffffffffu, eq);
    const bool take = gt || (eq && eq_before + __popc(eqm & below) < krem);
    const unsigned tm = __ballot_sync(0xffffffffu, take);
    if (take) out[out_pos + __popc(tm & below)] = i;
    out_pos += __popc(tm);
    eq_before += __popc(eqm);
  }
}

// ---------------------------------------------------------------------------
// Shared-memory select, one CTA per row, each thread owning a contiguous run.
// The row's keys are staged so that thread t holds keys [t L, (t+1) L) at
// shared offset t Lp, with Lp / V odd (V keys per 16-byte vector): the 16-byte
// reads of a quarter-warp then fall in distinct bank groups.  The first digit's
// histogram is taken while the row is loaded; each later digit re-reads the
// runs.  Histogram atomics go to RunCopies<NT>::n copies picked by lane, so
// lanes whose keys share a bin (scores crowd into a few exponents) rarely collide.
// Compaction: per-thread counts of keys > K and == K, two block scans for the
// output offsets, then every thread writes its own selections in index order.
// ---------------------------------------------------------------------------
// Histogram copies per block size.  128-thread rows (up to 16K keys) trade
// atomic collisions for occupancy: fewer copies leave shared memory for more
// CTAs per SM (2 copies: 0.34 ms against 0.39 ms with 8 on the 32K-token
// prefill rows).  512-thread rows run one CTA per SM and keep 8.
template <int NT> struct RunCopies { static constexpr int n = NT <= 128 ? 2 : 8; };

template <int NT>
__device__ __forceinline__ int block_excl_scan_nt(int v, int* wsum, int* total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int inc = warp_incl_scan(v);
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  int before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const int x = wsum[w];
    before += (w < warp) ? x : 0;
    tot += x;
  }
  __syncthreads();
  *total = tot;
  return before + inc - v;
}

// Run length L (a multiple of V) and padded stride Lp for n keys on NT threads.
template <int NT, int V>
__host__ __device__ __forceinline__ void run_shape(int n, int* L, int* Lp) {
  const int l = ((n + NT - 1) / NT + V - 1) / V * V;
  *L = l;
  *Lp = ((l / V) & 1) ? l : l + V;
}

// Radix select over 16-bit keys held in registers (kk[0, cntp) per thread):
// the key value K of the r-th largest (1 <= r <= total) and krem = r - #(> K).
template <int NT, int MAXP>
__device__ __forceinline__ void block_select16(const uint32_t (&kk)[MAXP], int cntp, int r, int* hflat, int* wsum,
                                               int* sel_digit, int* sel_above, uint32_t* K_out, int* krem_out) {
  constexpr int DPT = (256 + NT - 1) / NT;
  const int tid = threadIdx.x;
  const int cp = tid & (RunCopies<NT>::n - 1);
  uint32_t prefix = 0, pmask = 0;
  int krem = r;
#pragma unroll 1
  for (int shift = 8; shift >= 0; shift -= 8) {
    for (int i = tid; i < RunCopies<NT>::n * 256; i += NT) hflat[i] = 0;
    __syncthreads();
#pragma unroll
    for (int q = 0; q < MAXP; ++q)
      if (q < cntp && (kk[q] & pmask) == prefix) atomicAdd(&hflat[cp * 256 + ((kk[q] >> shift) & 0xFFu)], 1);
    __syncthreads();
    int cq[DPT], csum = 0;
#pragma unroll
    for (int q = 0; q < DPT; ++q) {
      const int d = 255 - DPT * tid - q;
      int c = 0;
      if (d >= 0) {
#pragma unroll
        for (int c2 = 0; c2 < RunCopies<NT>::n; ++c2) c += hflat[c2 * 256 + d];
      }
      cq[q] = c;
      csum += c;
    }
    int tot;
    int above = block_excl_scan_nt<NT>(csum, wsum, &tot);
#pragma unroll
    for (int q = 0; q < DPT; ++q) {
      if (above < krem && krem <= above + cq[q]) {
        *sel_digit = 255 - DPT * tid - q;
        *sel_above = above;
      }
      above += cq[q];
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(*sel_digit) << shift;
    pmask |= 0xFFu << shift;
    krem -= *sel_above;
  }
  *K_out = prefix;
  *krem_out = krem;
}

constexpr int kCandCap = 2048;   // candidates a sampled threshold may admit

template <typename T, int NT>
__global__ void __launch_bounds__(NT) topk_run_kernel(const T* __restrict__ score, int T_chunk, int S, int ld,
                                                      int k, int m, int row0, const int32_t* __restrict__ q_pos0,
                                                      int32_t* __restrict__ idx, int cand_off) {
  using KO = KeyOf<T>;
  using K = typename KO::K;
  static_assert(sizeof(K) == sizeof(T), "key and score widths match");
  constexpr int V = 16 / sizeof(K);
  constexpr int DPT = (256 + NT - 1) / NT;
  constexpr int top = KO::bits - 8;
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ int hist[RunCopies<NT>::n][256];
  __shared__ int wsum[NT / 32];
  __shared__ int sel_digit, sel_above;

  const int row = blockIdx.x;
  const int bi = row / T_chunk;
  const int r = row - bi * T_chunk;
  long long nv = (static_cast<long long>(q_pos0[bi]) + row0 + r + 1) / m;
  if (nv > S) nv = S;
  if (nv < 0) nv = 0;
  const int n = static_cast<int>(nv);
  int32_t* out = idx + static_cast<size_t>(row) * k;
  const int tid = threadIdx.x, lane = tid & 31;
  if (n <= k) {
    for (int i = tid; i < k; i += NT) out[i] = i < n ? i : -1;
    return;
  }
  int L, Lp;
  run_shape<NT, V>(n, &L, &Lp);
  K* keys = reinterpret_cast<K*>(dsm);
  int* hflat = &hist[0][0];
  const int cp = lane & (RunCopies<NT>::n - 1);
  for (int i = tid; i < RunCopies<NT>::n * 256; i += NT) hflat[i] = 0;
  __syncthreads();

  // rows that try the sampled threshold first take their first-digit
  // histogram only if they fall back to the full radix path
  // (long rows only: on short rows the two small selects cost more than the
  // radix passes they save)
  const bool sampled = KO::bits == 16 && NT >= 512 && n >= 2 * k && n > 4 * NT;
  const bool hist_in_load = !sampled;
  // ---- stage the row as keys (16-byte loads where aligned) + first-digit histogram
  const T* srow = score + static_cast<size_t>(row) * ld;
  int done = 0;
  if ((reinterpret_cast<uintptr_t>(srow) & 15) == 0) {
    const int nvec = n / V;
#pragma unroll 2
    for (int g = tid; g < nvec; g += NT) {
      const uint4 u = reinterpret_cast<const uint4*>(srow)[g];
      const T* e = reinterpret_cast<const T*>(&u);
      K kk[V];
#pragma unroll
      for (int q = 0; q < V; ++q) {
        kk[q] = KO::get(e[q]);
        if (hist_in_load) atomicAdd(&hist[cp][static_cast<uint32_t>(kk[q]) >> top], 1);
      }
      const int i = g * V;
      const int t = i / L;
      *reinterpret_cast<uint4*>(keys + static_cast<size_t>(t) * Lp + (i - t * L)) =
          *reinterpret_cast<const uint4*>(kk);
    }
    done = nvec * V;
  }
  for (int i = done + tid; i < n; i += NT) {
    const K key = KO::get(srow[i]);
    if (hist_in_load) atomicAdd(&hist[cp][static_cast<uint32_t>(key) >> top], 1);
    const int t = i / L;
    keys[static_cast<size_t>(t) * Lp + (i - t * L)] = key;
  }
  __syncthreads();

  const int cnt = max(0, min(L, n - tid * L));
  const K* run = keys + static_cast<size_t>(tid) * Lp;

  if constexpr (KO::bits == 16 && NT >= 512) {
    // ---- sampled threshold (long rows with n >= 2k): a radix select over 4 NT
    // evenly spaced keys gives T0, about 1.25 k + n / NT keys of the row lie
    // at or above it.  If at least k and at most kCandCap do, those candidates
    // are compacted in index order and the exact selection runs on them alone
    // (every key of the top k is >= T0 when at least k keys are); otherwise
    // the row takes the full radix path below.
    if (sampled) {
      constexpr int SPT = 4;                  // samples per thread
      constexpr int kSamples = SPT * NT;
      uint32_t sk[SPT];
#pragma unroll
      for (int q = 0; q < SPT; ++q) {
        const int pos = static_cast<int>(static_cast<long long>(tid * SPT + q) * n / kSamples);
        const int t = pos / L;
        sk[q] = keys[static_cast<size_t>(t) * Lp + (pos - t * L)];
      }
      int r = static_cast<int>(static_cast<long long>(5 * k) * kSamples / (4ll * n)) + 4;
      if (r > kSamples) r = kSamples;
      uint32_t T0;
      int unused;
      block_select16<NT, SPT>(sk, SPT, r, hflat, wsum, &sel_digit, &sel_above, &T0, &unused);
      int nge = 0;
      for (int j = 0; j < cnt; j += V) {
        const uint4 u = *reinterpret_cast<const uint4*>(run + j);
        const K* kk = reinterpret_cast<const K*>(&u);
#pragma unroll
        for (int q = 0; q < V; ++q) nge += (j + q < cnt && static_cast<uint32_t>(kk[q]) >= T0);
      }
      int tot;
      int cpos = block_excl_scan_nt<NT>(nge, wsum, &tot);
      if (tot >= k && tot <= kCandCap) {
        uint16_t* ckey = reinterpret_cast<uint16_t*>(dsm + cand_off);
        int32_t* cidx = reinterpret_cast<int32_t*>(dsm + cand_off + kCandCap * 2);
        const int base = tid * L;
        for (int j = 0; j < cnt; j += V) {
          const uint4 u = *reinterpret_cast<const uint4*>(run + j);
          const K* kk = reinterpret_cast<const K*>(&u);
#pragma unroll
          for (int q = 0; q < V; ++q) {
            const uint32_t key = kk[q];
            if (j + q < cnt && key >= T0) {
              ckey[cpos] = static_cast<uint16_t>(key);
              cidx[cpos] = base + j + q;
              ++cpos;
            }
          }
        }
        __syncthreads();
        // exact selection among the tot candidates (index order): thread t owns
        // candidates [t cpt, t cpt + cpt)
        constexpr int CPT = kCandCap / NT;
        const int cpt = (tot + NT - 1) / NT;
        const int c0 = tid * cpt;
        const int cc = max(0, min(cpt, tot - c0));
        uint32_t ck[CPT];
#pragma unroll
        for (int q = 0; q < CPT; ++q) ck[q] = q < cc ? ckey[c0 + q] : 0u;
        uint32_t Kf;
        int kremf;
        block_select16<NT, CPT>(ck, cc, k, hflat, wsum, &sel_digit, &sel_above, &Kf, &kremf);
        int n_gt = 0, n_eq = 0;
#pragma unroll
        for (int q = 0; q < CPT; ++q) {
          n_gt += q < cc && ck[q] > Kf;
          n_eq += q < cc && ck[q] == Kf;
        }
        int tg, te;
        const int gt_before = block_excl_scan_nt<NT>(n_gt, wsum, &tg);
        int eq_seen = block_excl_scan_nt<NT>(n_eq, wsum, &te);
        int pos = gt_before + min(eq_seen, kremf);
#pragma unroll
        for (int q = 0; q < CPT; ++q) {
          if (q < cc) {
            if (ck[q] > Kf) {
              out[pos++] = cidx[c0 + q];
            } else if (ck[q] == Kf) {
              if (eq_seen < kremf) out[pos++] = cidx[c0 + q];
              ++eq_seen;
            }
          }
        }
        return;
      }
      // fall back to the full radix path: take its first-digit histogram now
      for (int i = tid; i < RunCopies<NT>::n * 256; i += NT) hflat[i] = 0;
      __syncthreads();
      for (int j = 0; j < cnt; j += V) {
        const uint4 u = *reinterpret_cast<const uint4*>(run + j);
        const K* kk = reinterpret_cast<const K*>(&u);
#pragma unroll
        for (int q = 0; q < V; ++q)
          if (j + q < cnt) atomicAdd(&hist[cp][static_cast<uint32_t>(kk[q]) >> top], 1);
      }
      __syncthreads();
    }
  }
  uint32_t prefix = 0, pmask = 0;
  int krem = k;
#pragma unroll 1
  for (int shift = top; shift >= 0; shift -= 8) {
    if (shift != top) {
      for (int i = tid; i < RunCopies<NT>::n * 256; i += NT) hflat[i] = 0;
      __syncthreads();
      for (int j = 0; j < cnt; j += V) {
        const uint4 u = *reinterpret_cast<const uint4*>(run + j);
        const K* kk = reinterpret_cast<const K*>(&u);
#pragma unroll
        for (int q = 0; q < V; ++q) {
          const uint32_t key = kk[q];
          if (j + q < cnt && (key & pmask) == prefix) atomicAdd(&hist[cp][(key >> shift) & 0xFFu], 1);
        }
      }
      __syncthreads();
    }
    // thread t owns digits 255 - DPT t - q (descending), summed over the copies
    int cq[DPT], csum = 0;
#pragma unroll
    for (int q = 0; q < DPT; ++q) {
      const int d = 255 - DPT * tid - q;
      int c = 0;
      if (d >= 0) {
#pragma unroll
        for (int c2 = 0; c2 < RunCopies<NT>::n; ++c2) c += hist[c2][d];
      }
      cq[q] = c;
      csum += c;
    }
    int tot;
    int above = block_excl_scan_nt<NT>(csum, wsum, &tot);
#pragma unroll
    for (int q = 0; q < DPT; ++q) {
      if (above < krem && krem <= above + cq[q]) {
        sel_digit = 255 - DPT * tid - q;
        sel_above = above;
      }
      above += cq[q];
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(sel_digit) << shift;
    pmask |= 0xFFu << shift;
    krem -= sel_above;
  }
  // ---- threshold key K = prefix: every key > K, and the first krem keys == K
  int n_gt = 0, n_eq = 0;
  for (int j = 0; j < cnt; j += V) {
    const uint4 u = *reinterpret_cast<const uint4*>(run + j);
    const K* kk = reinterpret_cast<const K*>(&u);
#pragma unroll
    for (int q = 0; q < V; ++q) {
      const uint32_t key = kk[q];
      const bool ok = j + q < cnt;
      n_gt += ok && key > prefix;
      n_eq += ok && key == prefix;
    }
  }
  int tot_gt, tot_eq;
  const int gt_before = block_excl_scan_nt<NT>(n_gt, wsum, &tot_gt);
  int eq_seen = block_excl_scan_nt<NT>(n_eq, wsum, &tot_eq);
  int pos = gt_before + min(eq_seen, krem);
  const int base = tid * L;
  for (int j = 0; j < cnt; j += V) {
    const uint4 u = *reinterpret_cast<const uint4*>(run + j);
    const K* kk = reinterpret_cast<const K*>(&u);
#pragma unroll
    for (int q = 0; q < V; ++q) {
      const uint32_t key = kk[q];
      if (j + q < cnt) {
        if (key > prefix) {
          out[pos++] = base + j + q;
        } else if (key == prefix) {
          if (eq_seen < krem) out[pos++] = base + j + q;
          ++eq_seen;
        }
      }
    }
  }
}

// keys region, then (16-bit keys) the candidate buffer of the sampled path
template <typename T, int NT>
size_t run_keys_bytes(int S) {
  using K = typename KeyOf<T>::K;
  constexpr int V = 16 / sizeof(K);
  int L, Lp;
  run_shape<NT, V>(S, &L, &Lp);
  return (static_cast<size_t>(NT) * (L + V) * sizeof(K) + 15) & ~static_cast<size_t>(15);
}
template <typename T, int NT>
size_t run_smem_bytes(int S) {
  return run_keys_bytes<T, NT>(S) + (KeyOf<T>::bits == 16 && NT >= 512 ? static_cast<size_t>(kCandCap) * 6 : 0);
}

template <typename T, int NT>
int launch_topk_run(const T* score, long long rows, int T_chunk, int S, int ld, int k, int m, int row0,
                    const int32_t* q_pos0, int32_t* idx, cudaStream_t st) {
  const size_t bytes = run_smem_bytes<T, NT>(S);
  static int attr = -1;
  if (attr < static_cast<int>(bytes)) {
    cudaError_t e = cudaFuncSetAttribute(topk_run_kernel<T, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kTopkSmemMax));
    if (e != cudaSuccess) return set_cuda_error(e);
    attr = static_cast<int>(kTopkSmemMax);
  }
  topk_run_kernel<T, NT><<<static_cast<unsigned>(rows), NT, bytes, st>>>(
      score, T_chunk, S, ld, k, m, row0, q_pos0, idx, static_cast<int>(run_keys_bytes<T, NT>(S)));
  return check_launch();
}

// ---------------------------------------------------------------------------
// Multi-CTA select for a few long BF16 rows (decode: 32 rows of 262144 scores).
// A row is cut into chunks of kMcChunk keys, one CTA per (row, chunk), and the
// radix select runs as three launches that meet through a caller workspace:
//   K1  11-bit histogram of the high key bits      -> ws hist1[row][2048]
//   K2  threshold bin b1 (every CTA scans hist1),
//       5-bit histogram of the keys in bin b1       -> ws hist2[row][32]
//       and per chunk: its keys above bin b1 and its own 5-bit histogram of
//       bin b1                                     -> ws chunk[row][c][33]
//   K3  exact threshold key K = (b1, b2) and the count krem of keys == K to
//       take (every CTA scans hist2); the counts of keys > K and == K in the
//       earlier chunks follow from their K2 records, which give the chunk's
//       output offset; then in-order compaction over per-thread runs.
// The histograms are cleared by a memset at the start of every call.  The
// union of per-chunk results is the exact row result with the same tie rule.
// ---------------------------------------------------------------------------
constexpr int kMcThreads = 256;
constexpr int kMcWarps = kMcThreads / 32;
constexpr int kMcChunk = 8192;
constexpr int kMcHist1 = 2048;
constexpr int kMcHist2 = 32;
constexpr int kMcRowsMax = 512;     // more rows than this use one CTA per row
constexpr int kMcMinS = 16384;      // shorter rows use one CTA per row

struct McLayout {
  int C;            // chunks per row
  size_t row_ints;  // ints per row
  // per row: hist1[2048] hist2[32] state[4] chunk[C][1 + 32] (keys above bin
  // b1, then the chunk's 5-bit histogram of bin b1)
  static constexpr int kHist2 = kMcHist1, kState = kMcHist1 + kMcHist2, kCnt = kMcHist1 + kMcHist2 + 4;
  static constexpr int kChunkInts = 1 + kMcHist2;
  __host__ __device__ McLayout(int S)
      : C((S + kMcChunk - 1) / kMcChunk),
        row_ints(kCnt + kChunkInts * static_cast<size_t>((S + kMcChunk - 1) / kMcChunk)) {}
};

__device__ __forceinline__ int mc_row_n(int row, int T_chunk, int S, int m, int row0, const int32_t* q_pos0) {
  const int bi = row / T_chunk;
  const int r = row - bi * T_chunk;
  long long nv = (static_cast<long long>(q_pos0[bi]) + row0 + r + 1) / m;
  if (nv > S) nv = S;
  if (nv < 0) nv = 0;
  return static_cast<int>(nv);
}

// Descending bin search over a shared histogram of NB bins: returns (bin, count
// of keys in higher bins) for the bin holding the krem-th largest key.
template <int NB>
__device__ __forceinline__ void mc_find_bin(const int* h, int krem, int* wsum, int* out_bin, int* out_above) {
  constexpr int PER = (NB + kMcThreads - 1) / kMcThreads;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int c[PER], tot = 0;
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int d = NB - 1 - PER * tid - q;
    c[q] = d >= 0 ? h[d] : 0;
    tot += c[q];
  }
  const int inc = warp_incl_scan(tot);
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  int above = inc - tot;
#pragma unroll
  for (int w = 0; w < kMcWarps; ++w) above += (w < warp) ? wsum[w] : 0;
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    if (above < krem && krem <= above + c[q]) {
      *out_bin = NB - 1 - PER * tid - q;
      *out_above = above;
    }
    above += c[q];
  }
  __syncthreads();
}

// Keys [i, i + 8) of a row as order-preserving keys (valid where < i1): one
// 16-byte load when the row start is 16-byte aligned and the load stays inside
// the row's ld elements, else element loads.
__device__ __forceinline__ void mc_load8(const __nv_bfloat16* srow, int i, int i1, int ld, bool aligned,
                                         uint32_t (&kk)[8]) {
  using KO = KeyOf<__nv_bfloat16>;
  if (aligned && i + 8 <= ld) {
    const uint4 u = *reinterpret_cast<const uint4*>(srow + i);
    const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&u);
#pragma unroll
    for (int q = 0; q < 8; ++q) kk[q] = KO::get(e[q]);
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) kk[q] = i + q < i1 ? static_cast<uint32_t>(KO::get(srow[i + q])) : 0u;
  }
}
// thread t of a chunk owns keys [i0 + kMcRun t, i0 + kMcRun (t + 1))
constexpr int kMcRun = kMcChunk / kMcThreads;   // 32

__global__ void __launch_bounds__(kMcThreads) topk_mc_hist1(const __nv_bfloat16* __restrict__ score, int T_chunk,
                                                            int S, int ld, int k, int m, int row0,
                                                            const int32_t* __restrict__ q_pos0, int* __restrict__ ws) {
  using KO = KeyOf<__nv_bfloat16>;
  __shared__ int h[kMcHist1];
  const McLayout L(S);
  const int row = blockIdx.x / L.C, c = blockIdx.x % L.C;
  const int n = mc_row_n(row, T_chunk, S, m, row0, q_pos0);
  if (n <= k) return;
  const int i0 = c * kMcChunk, i1 = min(n, i0 + kMcChunk);
  if (i0 >= i1) return;
  for (int i = threadIdx.x; i < kMcHist1; i += kMcThreads) h[i] = 0;
  __syncthreads();
  const __nv_bfloat16* srow = score + static_cast<size_t>(row) * ld;
  const bool al = (reinterpret_cast<uintptr_t>(srow) & 15) == 0;
  const int r0 = i0 + kMcRun * threadIdx.x;
#pragma unroll
  for (int g = 0; g < kMcRun / 8; ++g) {
    const int b = r0 + 8 * g;
    if (b < i1) {
      uint32_t kk[8];
      mc_load8(srow, b, i1, ld, al, kk);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (b + q < i1) atomicAdd(&h[kk[q] >> 5], 1);
    }
  }
  __syncthreads();
  int* g = ws + static_cast<size_t>(row) * L.row_ints;
  for (int i = threadIdx.x; i < kMcHist1; i += kMcThreads)
    if (h[i]) atomicAdd(&g[i], h[i]);
}

__global__ void __launch_bounds__(kMcThreads) topk_mc_hist2(const __nv_bfloat16* __restrict__ score, int T_chunk,
                                                            int S, int ld, int k, int m, int row0,
                                                            const int32_t* __restrict__ q_pos0, int* __restrict__ ws) {
  using KO = KeyOf<__nv_bfloat16>;
  __shared__ int h[kMcHist1];
  __shared__ int h2[kMcHist2];
  __shared__ int wsum[kMcWarps];
  __shared__ int s_bin, s_above;
  const McLayout L(S);
  const int row = blockIdx.x / L.C, c = blockIdx.x % L.C;
  const int n = mc_row_n(row, T_chunk, S, m, row0, q_pos0);
  if (n <= k) return;
  int* g = ws + static_cast<size_t>(row) * L.row_ints;
  for (int i = threadIdx.x; i < kMcHist1; i += kMcThreads) h[i] = g[i];
  if (threadIdx.x < kMcHist2) h2[threadIdx.x] = 0;
  __syncthreads();
  mc_find_bin<kMcHist1>(h, k, wsum, &s_bin, &s_above);
  const int b1 = s_bin;
  if (c == 0 && threadIdx.x == 0) {
    g[McLayout::kState + 0] = b1;
    g[McLayout::kState + 1] = s_above;
  }
  const int i0 = c * kMcChunk, i1 = min(n, i0 + kMcChunk);
  const __nv_bfloat16* srow = score + static_cast<size_t>(row) * ld;
  const bool al = (reinterpret_cast<uintptr_t>(srow) & 15) == 0;
  const int r0 = i0 + kMcRun * threadIdx.x;
  int n_above = 0;   // this thread's keys above bin b1
#pragma unroll
  for (int g = 0; g < kMcRun / 8; ++g) {
    const int b = r0 + 8 * g;
    if (b < i1) {
      uint32_t kk[8];
      mc_load8(srow, b, i1, ld, al, kk);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int bin = static_cast<int>(kk[q] >> 5);
        if (b + q < i1) {
          n_above += bin > b1;
          if (bin == b1) atomicAdd(&h2[kk[q] & 31], 1);
        }
      }
    }
  }
  n_above = __reduce_add_sync(0xffffffffu, n_above);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = n_above;
  __syncthreads();
  int* rec = g + McLayout::kCnt + static_cast<size_t>(c) * McLayout::kChunkInts;
  if (threadIdx.x < kMcHist2) {
    const int v = h2[threadIdx.x];
    rec[1 + threadIdx.x] = v;
    if (v) atomicAdd(&g[McLayout::kHist2 + threadIdx.x], v);
  }
  if (threadIdx.x == 0) {
    int a = 0;
#pragma unroll
    for (int w = 0; w < kMcWarps; ++w) a += wsum[w];
    rec[0] = a;
  }
}

__global__ void __launch_bounds__(kMcThreads, 4) topk_mc_emit(const __nv_bfloat16* __restrict__ score, int T_chunk,
                                                           int S, int ld, int k, int m, int row0,
                                                           const int32_t* __restrict__ q_pos0,
                                                           const int* __restrict__ ws, int32_t* __restrict__ idx) {
  __shared__ int wsum[kMcWarps];
  __shared__ int h2s[kMcHist2];
  __shared__ int s_bin, s_above, s_gt, s_eq;
  const McLayout L(S);
  const int row = blockIdx.x / L.C, c = blockIdx.x % L.C;
  const int n = mc_row_n(row, T_chunk, S, m, row0, q_pos0);
  int32_t* out = idx + static_cast<size_t>(row) * k;
  const int i0 = c * kMcChunk;
  if (n <= k) {
    // every visible entry, then -1 pads; chunk c covers output slots [i0, i0 + kMcChunk)
    const int hi = c == L.C - 1 ? k : min(k, i0 + kMcChunk);   // the last chunk also covers slots >= S
    for (int i = i0 + threadIdx.x; i < hi; i += kMcThreads) out[i] = i < n ? i : -1;
    return;
  }
  const int i1 = min(n, i0 + kMcChunk);
  if (i0 >= i1) return;
  const int* g = ws + static_cast<size_t>(row) * L.row_ints;
  // threshold K = (b1, b2): b2 from the row's 5-bit histogram of bin b1
  if (threadIdx.x < kMcHist2) h2s[threadIdx.x] = g[McLayout::kHist2 + threadIdx.x];
  __syncthreads();
  const int b1 = g[McLayout::kState + 0];
  const int krem1 = k - g[McLayout::kState + 1];
  mc_find_bin<kMcHist2>(h2s, krem1, wsum, &s_bin, &s_above);
  const int b2 = s_bin;
  const uint32_t K = (static_cast<uint32_t>(b1) << 5) | static_cast<uint32_t>(b2);
  const int krem = krem1 - s_above;
  // keys > K and == K in the chunks before this one (lane l sums chunks l, l + 32, ...)
  if (threadIdx.x < 32) {
    int gt = 0, eq = 0;
    for (int cc = threadIdx.x; cc < c; cc += 32) {
      const int* rec = g + McLayout::kCnt + static_cast<size_t>(cc) * McLayout::kChunkInts;
      int a = rec[0];
      for (int bb = b2 + 1; bb < kMcHist2; ++bb) a += rec[1 + bb];
      gt += a;
      eq += rec[1 + b2];
    }
    gt = __reduce_add_sync(0xffffffffu, gt);
    eq = __reduce_add_sync(0xffffffffu, eq);
    if (threadIdx.x == 0) {
      s_gt = gt;
      s_eq = eq;
    }
  }
  __syncthreads();
  const int gt_c = s_gt, eq_c = s_eq;
  // this thread's run, then its output position: every key > K before it in
  // the row, plus the keys == K before it that are taken (the first krem)
  const __nv_bfloat16* srow = score + static_cast<size_t>(row) * ld;
  const bool al = (reinterpret_cast<uintptr_t>(srow) & 15) == 0;
  const int r0 = i0 + kMcRun * threadIdx.x;
  // the run's 16-bit keys, two per register (key q in half q & 1 of kr[q / 2])
  uint32_t kr[kMcRun / 2];
#pragma unroll
  for (int gq = 0; gq < kMcRun / 8; ++gq) {
    uint32_t kk[8];
    const int b = r0 + 8 * gq;
    if (b < i1) {
      mc_load8(srow, b, i1, ld, al, kk);
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) kk[q] = 0u;
    }
#pragma unroll
    for (int q = 0; q < 8; q += 2) kr[4 * gq + q / 2] = kk[q] | (kk[q + 1] << 16);
  }
  auto key_at = [&](int q) -> uint32_t { return (kr[q >> 1] >> (16 * (q & 1))) & 0xFFFFu; };
  int n_gt = 0, n_eq = 0;
#pragma unroll
  for (int q = 0; q < kMcRun; ++q) {
    n_gt += r0 + q < i1 && key_at(q) > K;
    n_eq += r0 + q < i1 && key_at(q) == K;
  }
  int tg, te;
  const int gt_t = block_excl_scan_nt<kMcThreads>(n_gt, wsum, &tg);
  int eq_seen = eq_c + block_excl_scan_nt<kMcThreads>(n_eq, wsum, &te);
  int pos = gt_c + gt_t + min(eq_seen, krem);
#pragma unroll
  for (int q = 0; q < kMcRun; ++q) {
    const int i = r0 + q;
    if (i < i1) {
      const uint32_t key = key_at(q);
      if (key > K) {
        out[pos++] = i;
      } else if (key == K) {
        if (eq_seen < krem) out[pos++] = i;
        ++eq_seen;
      }
    }
  }
}

inline bool topk_use_multi(int score_dtype, long long rows, int S) {
  return score_dtype == CSA_BF16 && rows <= kMcRowsMax && S >= kMcMinS;
}

inline size_t topk_multi_bytes(long long rows, int S) {
  return static_cast<size_t>(rows) * McLayout(S).row_ints * sizeof(int);
}

int launch_topk_multi(const __nv_bfloat16* score, long long rows, int T_chunk, int S, int ld, int k, int m, int row0,
                      const int32_t* q_pos0, int32_t* idx, int* ws, cudaStream_t st) {
  const McLayout L(S);
  cudaError_t e = cudaMemsetAsync(ws, 0, topk_multi_bytes(rows, S), st);
  if (e != cudaSuccess) return set_cuda_error(e);
  const unsigned grid = static_cast<unsigned>(rows * L.C);
  topk_mc_hist1<<<grid, kMcThreads, 0, st>>>(score, T_chunk, S, ld, k, m, row0, q_pos0, ws);
  topk_mc_hist2<<<grid, kMcThreads, 0, st>>>(score, T_chunk, S, ld, k, m, row0, q_pos0, ws);
  topk_mc_emit<<<grid, kMcThreads, 0, st>>>(score, T_chunk, S, ld, k, m, row0, q_pos0, ws, idx);
  return check_launch();
}

template <typename T>
int launch_topk(const T* score, int B, int T_chunk, int S, int ld, int k, int m, int row0, const int32_t* q_pos0,
                int32_t* idx, cudaStream_t st) {
  const long long rows = static_cast<long long>(B) * T_chunk;
  using K = typename KeyOf<T>::K;
  const size_t keys_bytes = static_cast<size_t>(S) * sizeof(K);
  const unsigned grid = static_cast<unsigned>(rows);
  (void)keys_bytes;
  if (S <= 16384 && run_smem_bytes<T, 128>(S) <= kTopkSmemMax) {
    return launch_topk_run<T, 128>(score, rows, T_chunk, S, ld, k, m, row0, q_pos0, idx, st);
  } else if (run_smem_bytes<T, 512>(S) <= kTopkSmemMax) {
    return launch_topk_run<T, 512>(score, rows, T_chunk, S, ld, k, m, row0, q_pos0, idx, st);
  } else {
    topk_row_kernel<T, false><<<grid, kTopkThreads, 0, st>>>(score, T_chunk, S, ld, k, m, row0, q_pos0, idx);
  }
  return check_launch();
}

}  // namespace csa

using namespace csa;

extern "C" {

size_t topk_workspace_size(int B, int T_chunk, int S, int k) {
  (void)k;
  if (B <= 0 || T_chunk <= 0 || S <= 0) return 0;
  const long long rows = static_cast<long long>(B) * T_chunk;
  return topk_use_multi(CSA_BF16, rows, S) ? topk_multi_bytes(rows, S) : 0;
}

int topk_select(const void* score, int score_dtype, int B, int T_chunk, int S, int score_ld, int k, int m,
                int row0, const int32_t* q_pos0, int32_t* idx, void* workspace, size_t ws_bytes,
                csa_stream_t stream) {
  CSA_REQUIRE(score && idx && q_pos0, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE((reinterpret_cast<uintptr_t>(workspace) & 3) == 0, CSA_ERR_ALIGNMENT);
  CSA_REQUIRE(B >= 0 && T_chunk >= 0 && S >= 0 && score_ld >= S && k >= 1 && m >= 1 && row0 >= 0,
              CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(score_dtype == CSA_F32 || score_dtype == CSA_BF16, CSA_ERR_INVALID_ARG);
  const long long rows = static_cast<long long>(B) * T_chunk;
  if (rows == 0) return CSA_OK;
  CSA_REQUIRE(rows < (1ll << 31), CSA_ERR_UNSUPPORTED);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (topk_use_multi(score_dtype, rows, S) && workspace != nullptr && ws_bytes >= topk_multi_bytes(rows, S))
    return launch_topk_multi(static_cast<const __nv_bfloat16*>(score), rows, T_chunk, S, score_ld, k, m, row0,
                             q_pos0, idx, static_cast<int*>(workspace), st);
  if (score_dtype == CSA_F32)
    return launch_topk(static_cast<const float*>(score), B, T_chunk, S, score_ld, k, m, row0, q_pos0, idx, st);
  return launch_topk(static_cast<const __nv_bfloat16*>(score), B, T_chunk, S, score_ld, k, m, row0, q_pos0, idx,
                     st);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// topk_select_noalloc: the same selection for callers that may not allocate
// device memory.  An allocator-free caller (a real-time serving loop that
// must not block on the CUDA allocator, a host runtime that hands the library
// no memory of its own, code running where a cudaMalloc could implicitly
// synchronise the device) cannot provide the multi-CTA workspace.  This entry
// uses a fixed scratch array that lives in the library's own device image
// instead, so it allocates nothing, ever: no cudaMalloc, no cudaFree, no
// library routine that allocates.
//
// Limits and rules, in plain words:
//   * the scratch holds kNoAllocScratchBytes (1 MiB); a shape whose multi-CTA
//     histograms need more is rejected with CSA_ERR_UNSUPPORTED before any
//     work is queued (32 rows of 262,144 entries need about 402 KB);
//   * the scratch is one per device and per process: two calls that overlap
//     in time on the same device (different streams, or different host
//     threads) race on it and give wrong results;
//   * the first call on each device looks up the scratch's device address
//     (cudaGetSymbolAddress with that device current); make that first call
//     before any stream capture begins.  The address is cached for the life
//     of the process: after cudaDeviceReset the cached address is stale, so
//     a caller that resets a device must not call this entry on it again;
//   * shapes that need no scratch run the one-CTA-per-row kernel, as
//     topk_select does without a workspace.
// ---------------------------------------------------------------------------
namespace csa {

constexpr size_t kNoAllocScratchBytes = 1u << 20;
static __device__ __align__(256) uint8_t g_topk_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
static std::mutex g_noalloc_mu;
static void* g_noalloc_ptr[kNoAllocMaxDevices] = {nullptr};

// Device address of this device's scratch (set-up on first use per device).
static int noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_cuda_error(e);
  if (dev < 0 || dev >= kNoAllocMaxDevices) return CSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_topk_scratch);
    if (e != cudaSuccess) return set_cuda_error(e);
    if (p == nullptr) return CSA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return CSA_OK;
}

}  // namespace csa

extern "C" int topk_select_noalloc(const void* score, int score_dtype, int B, int T_chunk, int S, int score_ld,
                                   int k, int m, int row0, const int32_t* q_pos0, int32_t* idx,
                                   csa_stream_t stream) {
  CSA_REQUIRE(score && idx && q_pos0, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(B >= 0 && T_chunk >= 0 && S >= 0 && score_ld >= S && k >= 1 && m >= 1 && row0 >= 0,
              CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(score_dtype == CSA_F32 || score_dtype == CSA_BF16, CSA_ERR_INVALID_ARG);
  const long long rows = static_cast<long long>(B) * T_chunk;
  if (rows == 0) return CSA_OK;
  CSA_REQUIRE(rows < (1ll << 31), CSA_ERR_UNSUPPORTED);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!topk_use_multi(score_dtype, rows, S)) {
    if (score_dtype == CSA_F32)
      return launch_topk(static_cast<const float*>(score), B, T_chunk, S, score_ld, k, m, row0, q_pos0, idx, st);
    return launch_topk(static_cast<const __nv_bfloat16*>(score), B, T_chunk, S, score_ld, k, m, row0, q_pos0,
                       idx, st);
  }
  // the multi-CTA histograms must fit the fixed scratch; larger shapes are refused
  CSA_REQUIRE(topk_multi_bytes(rows, S) <= kNoAllocScratchBytes, CSA_ERR_UNSUPPORTED);
  void* scratch = nullptr;
  const int r = noalloc_scratch(&scratch);
  if (r != CSA_OK) return r;
  // launch_topk_multi clears the histogram region it uses (cudaMemsetAsync,
  // which allocates nothing) before its first kernel
  return launch_topk_multi(static_cast<const __nv_bfloat16*>(score), rows, T_chunk, S, score_ld, k, m, row0, q_pos0,
                           idx, static_cast<int*>(scratch), st);
}
