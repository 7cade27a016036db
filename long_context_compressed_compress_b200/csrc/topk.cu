// Per-query top-k selection over the lightning-indexer scores
// (cf-1.com/news/5231315 §3.1: each query picks its top-k compressed entries;
// §4.4: the scores are stored in BF16, which halves the selector's traffic).
//
// Radix select on order-preserving integer keys: a float's bit pattern is
// mapped so that unsigned integer order equals float order (+0 and -0 map to
// the same key).  8-bit digits are resolved from the top; each pass builds a
// 256-bin histogram of the candidates that still match the chosen prefix, and
// the bin holding the k-th largest key fixes the next digit.  After the last
// pass the threshold key K is exact: every key > K is selected, and the
// (k - #greater) keys == K with the smallest indices.  The final pass is an
// in-order compaction (block-wide prefix sums), so indices come out ascending
// and the result is bit-exact and independent of scheduling.
//
// One CTA per query row; the visible prefix of the row is staged in shared
// memory when it fits, otherwise every pass re-reads it from L2.
#include "common.cuh"

namespace csa {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;

__device__ __forceinline__ uint32_t key_of(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;                       // -0 == +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ uint32_t key_of(__nv_bfloat16 x) {
  uint32_t u = __bfloat16_as_ushort(x);
  if (u == 0x8000u) u = 0u;
  return (u & 0x8000u) ? (~u & 0xFFFFu) : (u | 0x8000u);
}

template <typename T> struct KeyBits;
template <> struct KeyBits<float> { static constexpr int bits = 32; };
template <> struct KeyBits<__nv_bfloat16> { static constexpr int bits = 16; };

// Block-wide exclusive scan of one int per thread (in thread order); also
// returns the block total.  Uses `scratch` (kTopkWarps + 1 ints).
__device__ __forceinline__ int block_excl_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int inc = warp_incl_scan(v);
  if (lane == 31) scratch[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kTopkWarps ? scratch[lane] : 0;
    const int wi = warp_incl_scan(w);
    if (lane < kTopkWarps) scratch[lane] = wi - w;
    if (lane == kTopkWarps - 1) scratch[kTopkWarps] = wi;
  }
  __syncthreads();
  const int res = scratch[warp] + inc - v;
  *total = scratch[kTopkWarps];
  __syncthreads();
  return res;
}

template <typename T, bool kSmem>
__global__ void __launch_bounds__(kTopkThreads) topk_row_kernel(const T* __restrict__ score, int T_chunk, int S,
                                                               int ld, int k, int m, int row0,
                                                               const int32_t* __restrict__ q_pos0,
                                                               int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ int hist[kTopkWarps][256];
  __shared__ int scratch[kTopkWarps + 2];
  __shared__ uint32_t sel_digit;
  __shared__ int sel_above;

  const int row = blockIdx.x;
  const int bi = row / T_chunk;
  const int r = row - bi * T_chunk;
  const long long p = static_cast<long long>(q_pos0[bi]) + row0 + r;
  long long nv = (p + 1) / m;
  if (nv > S) nv = S;
  if (nv < 0) nv = 0;
  const int n = static_cast<int>(nv);
  int32_t* out = idx + static_cast<size_t>(row) * k;
  if (n <= k) {
    for (int i = threadIdx.x; i < k; i += blockDim.x) out[i] = i < n ? i : -1;
    return;
  }
  const T* srow = score + static_cast<size_t>(row) * ld;
  uint32_t* keys = reinterpret_cast<uint32_t*>(dsm);
  if (kSmem) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) keys[i] = key_of(srow[i]);
  }
  auto key_at = [&](int i) -> uint32_t { return kSmem ? keys[i] : key_of(srow[i]); };

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t prefix = 0, pmask = 0;
  int krem = k;
  constexpr int kBits = KeyBits<T>::bits;
#pragma unroll 1
  for (int shift = kBits - 8; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < kTopkWarps * 256; i += blockDim.x) (&hist[0][0])[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const uint32_t key = key_at(i);
      const bool cand = (key & pmask) == prefix;
      const uint32_t dig = (key >> shift) & 0xFFu;
      // warp-aggregated increment of the per-warp histogram
      const unsigned act = __ballot_sync(__activemask(), cand);
      if (cand) {
        const unsigned peers = __match_any_sync(act, dig);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[warp][dig], __popc(peers));
      }
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits 255-8l .. 248-8l (descending); count per digit
      int cnt[8];
      int tot = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int d = 255 - (8 * lane + j);
        int c = 0;
        for (int w = 0; w < kTopkWarps; ++w) c += hist[w][d];
        cnt[j] = c;
        tot += c;
      }
      const int incl = warp_incl_scan(tot);
      int before = incl - tot;         // # candidates with a larger digit than this lane's first
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (before < krem && krem <= before + cnt[j]) {
          sel_digit = static_cast<uint32_t>(255 - (8 * lane + j));
          sel_above = before;
        }
        before += cnt[j];
      }
    }
    __syncthreads();
    prefix |= sel_digit << shift;
    pmask |= 0xFFu << shift;
    krem -= sel_above;
    __syncthreads();
  }
  // threshold key = prefix; take all keys > prefix, and the first `krem` keys == prefix.
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int i0 = min(n, static_cast<int>(threadIdx.x) * per);
  const int i1 = min(n, i0 + per);
  int n_gt = 0, n_eq = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = key_at(i);
    n_gt += key > prefix;
    n_eq += key == prefix;
  }
  int tot;
  const int eq_before = block_excl_scan(n_eq, scratch, &tot);
  const int eq_take = max(0, min(n_eq, krem - eq_before));
  const int pos0 = block_excl_scan(n_gt + eq_take, scratch, &tot);
  int o = pos0, eq_seen = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = key_at(i);
    bool take = key > prefix;
    if (key == prefix) { take = eq_seen < eq_take; ++eq_seen; }
    if (take) out[o++] = i;
  }
}

}  // namespace csa

using namespace csa;

extern "C" {

size_t topk_workspace_size(int B, int T_chunk, int S, int k) {
  (void)B; (void)T_chunk; (void)S; (void)k;
  return 0;
}

int topk_select(const void* score, int score_dtype, int B, int T_chunk, int S, int score_ld, int k, int m,
                int row0, const int32_t* q_pos0, int32_t* idx, void* workspace, size_t ws_bytes,
                csa_stream_t stream) {
  (void)workspace; (void)ws_bytes;
  CSA_REQUIRE(score && idx && q_pos0, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(B >= 0 && T_chunk >= 0 && S >= 0 && score_ld >= S && k >= 1 && m >= 1 && row0 >= 0,
              CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(score_dtype == CSA_F32 || score_dtype == CSA_BF16, CSA_ERR_INVALID_ARG);
  const long long rows = static_cast<long long>(B) * T_chunk;
  if (rows == 0) return CSA_OK;
  CSA_REQUIRE(rows < (1ll << 31), CSA_ERR_UNSUPPORTED);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t keys_bytes = static_cast<size_t>(S) * 4;
  const bool smem = keys_bytes <= 160 * 1024;
  const unsigned grid = static_cast<unsigned>(rows);
  if (score_dtype == CSA_F32) {
    if (smem) {
      cudaFuncSetAttribute(topk_row_kernel<float, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(keys_bytes));
      topk_row_kernel<float, true><<<grid, kTopkThreads, keys_bytes, st>>>(
          static_cast<const float*>(score), T_chunk, S, score_ld, k, m, row0, q_pos0, idx);
    } else {
      topk_row_kernel<float, false><<<grid, kTopkThreads, 0, st>>>(static_cast<const float*>(score), T_chunk, S,
                                                                    score_ld, k, m, row0, q_pos0, idx);
    }
  } else {
    if (smem) {
      cudaFuncSetAttribute(topk_row_kernel<__nv_bfloat16, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(keys_bytes));
      topk_row_kernel<__nv_bfloat16, true><<<grid, kTopkThreads, keys_bytes, st>>>(
          static_cast<const __nv_bfloat16*>(score), T_chunk, S, score_ld, k, m, row0, q_pos0, idx);
    } else {
      topk_row_kernel<__nv_bfloat16, false><<<grid, kTopkThreads, 0, st>>>(
          static_cast<const __nv_bfloat16*>(score), T_chunk, S, score_ld, k, m, row0, q_pos0, idx);
    }
  }
  return check_launch();
}

}  // extern "C"
