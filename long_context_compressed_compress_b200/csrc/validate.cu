// Bounds check of selected-entry indices, the check mode of the layer drivers
// (cf-1.com/news/5231315 §3.1: each query attends to its top-k visible
// compressed entries).  It runs between the selection and the attention when
// the drivers' check mode is on, and reports a bad index in a status word
// instead of letting the attention gather from outside the visible entries.
//
// Row r of a chunk (position p = q_pos0[b] + row0 + r) sees n = min(S, (p+1)/m)
// entries.  A valid idx row holds entries in [0, n), strictly ascending, then
// -1 padding to k.  One warp checks a row; each lane compares its entry with
// the next one.  A violation writes CSA_ERR_INVALID_ARG | site << 8 to the
// status word (first one kept): site 1 an entry outside [-1, n), site 2 two
// valid entries out of order, site 3 a valid entry after the padding began.
#include "common.cuh"

namespace csa {

__global__ void __launch_bounds__(256) validate_idx_kernel(const int32_t* __restrict__ idx, int B, int T_chunk,
                                                           int k, int S, int m, int row0,
                                                           const int32_t* __restrict__ q_pos0,
                                                           int* __restrict__ status) {
  const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<long long>(B) * T_chunk) return;
  const int bi = static_cast<int>(row / T_chunk);
  const long long p = static_cast<long long>(q_pos0[bi]) + row0 + (row - static_cast<long long>(bi) * T_chunk);
  long long nv = (p + 1) / m;
  if (nv > S) nv = S;
  if (nv < 0) nv = 0;
  const int32_t* r = idx + row * k;
  int site = 0;
  for (int i = lane; i < k; i += 32) {
    const int v = r[i];
    if (v < -1 || v >= nv) {
      site = 1;
    } else if (i + 1 < k) {
      const int w = r[i + 1];
      if (v >= 0 && w >= 0 && w <= v) site = site ? site : 2;
      if (v == -1 && w >= 0) site = site ? site : 3;
    }
  }
  const unsigned bad = __ballot_sync(0xffffffffu, site != 0);
  if (bad && lane == __ffs(bad) - 1) atomicCAS(status, 0, CSA_ERR_INVALID_ARG | (site << 8));
}

}  // namespace csa

using namespace csa;

extern "C" int csa_validate_indices(const int32_t* idx, int B, int T_chunk, int k, int S, int m, int row0,
                                    const int32_t* q_pos0, int32_t* status, csa_stream_t stream) {
  CSA_REQUIRE(idx && q_pos0 && status, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(B >= 0 && T_chunk >= 0 && k >= 1 && S >= 0 && m >= 1 && row0 >= 0, CSA_ERR_INVALID_ARG);
  if (B == 0 || T_chunk == 0) return CSA_OK;
  const long long rows = static_cast<long long>(B) * T_chunk;
  const long long grid = (rows + 7) / 8;
  CSA_REQUIRE(grid < (1ll << 31), CSA_ERR_UNSUPPORTED);
  validate_idx_kernel<<<static_cast<unsigned>(grid), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      idx, B, T_chunk, k, S, m, row0, q_pos0, reinterpret_cast<int*>(status));
  return check_launch();
}
