// Attention with raw window and sink on CUDA cores (fp32 arithmetic).
//
// This is the fp32 path of sparse_attn_fwd / hca_dense_attn_fwd (the tensor
// cores have no fp32 kind, and the fp32 workload asks for 1e-5 relative
// agreement), and the whole of swa_sink_merge (cf-1.com/news/5231315 §3.3:
// the raw-window branch and the learnable sink enter the same softmax
// denominator as the compressed branch).
//
// CTA = (query row, group of 8 heads); warp = one head; lane = D/32 dims of
// q and of the running output.  Keys are staged 64 at a time in shared memory
// as fp32; each key's logit is a warp all-reduce and the softmax is the usual
// online (running max, running sum) form.
#include "common.cuh"

namespace csa {

enum AttnMode : int { kModeSparse = 0, kModeDense = 1, kModeWindow = 2 };
constexpr int kSimtHeads = 8;
constexpr int kSimtKeys = 64;

template <typename T, int D>
__global__ void __launch_bounds__(256) attn_simt_kernel(
    const T* __restrict__ q, const T* __restrict__ kv_c, const int32_t* __restrict__ idx,
    const T* __restrict__ kv_raw, const float* __restrict__ sink, float tau, int W, int Tq, int row0,
    int T_chunk, int H, int kv_bstride, int k, int S, int m, int raw_cap, const int32_t* __restrict__ q_pos0,
    T* __restrict__ out, float* __restrict__ lse, int mode, const T* __restrict__ o_c,
    const float* __restrict__ lse_c) {
  constexpr int DL = D / 32;
  __shared__ float keys[kSimtKeys][D];
  __shared__ const T* rowptr[kSimtKeys];
  const int ngroups = (H + kSimtHeads - 1) / kSimtHeads;
  const int hg = blockIdx.x % ngroups;
  const int row = blockIdx.x / ngroups;
  const int bi = row / T_chunk;
  const int r = row - bi * T_chunk;
  const int t = row0 + r;
  const long long p = static_cast<long long>(q_pos0[bi]) + t;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = hg * kSimtHeads + warp;
  const bool hok = h < H;

  float qv[DL], acc[DL];
  const size_t qoff = ((static_cast<size_t>(bi) * Tq + t) * H + (hok ? h : 0)) * D;
#pragma unroll
  for (int i = 0; i < DL; ++i) {
    qv[i] = to_f(q[qoff + lane + 32 * i]) * tau;
    acc[i] = 0.f;
  }
  float mrun = -INFINITY, lsum = 0.f;

  // key list: [compressed entries][window rows]
  int n_ent = 0;
  if (mode == kModeSparse) n_ent = k;
  else if (mode == kModeDense) {
    long long v = (p + 1) / m;
    n_ent = static_cast<int>(v < S ? v : S);
  }
  const long long jlo = p - W + 1 > 0 ? p - W + 1 : 0;
  const int n_win = W > 0 ? static_cast<int>(p - jlo + 1) : 0;
  const int n_all = n_ent + n_win;
  const int32_t* irow = idx + static_cast<size_t>(row) * k;

  for (int base = 0; base < n_all; base += kSimtKeys) {
    const int cnt = min(kSimtKeys, n_all - base);
    __syncthreads();
    if (threadIdx.x < cnt) {
      const int j = base + threadIdx.x;
      const T* ptr = nullptr;
      if (j < n_ent) {
        const int s = mode == kModeSparse ? irow[j] : j;
        if (s >= 0) ptr = kv_c + (static_cast<size_t>(bi) * kv_bstride + s) * D;
      } else {
        const long long tok = jlo + (j - n_ent);
        ptr = kv_raw + (static_cast<size_t>(bi) * raw_cap + static_cast<size_t>(tok % raw_cap)) * D;
      }
      rowptr[threadIdx.x] = ptr;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < cnt * D; e += blockDim.x) {
      const int kk = e / D, d = e - kk * D;
      const T* ptr = rowptr[kk];
      keys[kk][d] = ptr ? to_f(ptr[d]) : 0.f;
    }
    __syncthreads();
    if (hok) {
      for (int kk = 0; kk < cnt; ++kk) {
        if (rowptr[kk] == nullptr) continue;
        float part = 0.f;
#pragma unroll
        for (int i = 0; i < DL; ++i) part = fmaf(qv[i], keys[kk][lane + 32 * i], part);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        const float l = part;
        if (l > mrun) {
          const float sc = expf(mrun - l);
          lsum *= sc;
#pragma unroll
          for (int i = 0; i < DL; ++i) acc[i] *= sc;
          mrun = l;
        }
        const float pe = expf(l - mrun);
        lsum += pe;
#pragma unroll
        for (int i = 0; i < DL; ++i) acc[i] = fmaf(pe, keys[kk][lane + 32 * i], acc[i]);
      }
    }
  }
  if (!hok) return;
  const size_t ooff = qoff;
  const size_t lrow = (static_cast<size_t>(bi) * Tq + t) * H + h;
  float res[DL];
  if (mode != kModeWindow) {
    // out = acc / (lsum + e^{sigma - M}) with M = max(mrun, sigma)
    const float sg = sink ? sink[h] : -INFINITY;
    float denom, scale;
    if (mrun == -INFINITY && sg == -INFINITY) { denom = 1.f; scale = 0.f; }
    else if (sg > mrun) { scale = expf(mrun - sg); denom = lsum * scale + 1.f; }
    else { scale = 1.f; denom = lsum + expf(sg - mrun); }
#pragma unroll
    for (int i = 0; i < DL; ++i) res[i] = __fdiv_rn(acc[i] * scale, denom);
    if (lse && lane == 0) lse[lrow] = mrun == -INFINITY ? -INFINITY : mrun + logf(lsum);
  } else {
    // merge (o_c, L_c) with the window branch (o_w, L_w) and the sink
    const float lw = mrun == -INFINITY ? -INFINITY : mrun + logf(lsum);
    const float lc = lse_c[lrow];
    const float sg = sink ? sink[h] : -INFINITY;
    float M = fmaxf(fmaxf(lc, lw), sg);
    if (M == -INFINITY) M = 0.f;
    const float ec = expf(lc - M), ew = expf(lw - M), es = expf(sg - M);
    const float denom = ec + ew + es;
#pragma unroll
    for (int i = 0; i < DL; ++i) {
      const float ow = lsum > 0.f ? acc[i] / lsum : 0.f;
      const float oc = to_f(o_c[ooff + lane + 32 * i]);
      res[i] = __fdiv_rn(ec * oc + ew * ow, denom > 0.f ? denom : 1.f);
    }
  }
#pragma unroll
  for (int i = 0; i < DL; ++i) out[ooff + lane + 32 * i] = static_cast<T>(res[i]);
}

int launch_attn_simt(const void* q, const void* kv_c, const int32_t* idx, const void* kv_raw, const float* sink,
                     float tau, int W, int B, int Tq, int row0, int T_chunk, int H, int D, int kv_bstride, int k,
                     int S, int m, int raw_cap, const int32_t* q_pos0, void* out, float* lse, int dtype, int mode,
                     const void* o_c, const float* lse_c, cudaStream_t st) {
  const long long rows = static_cast<long long>(B) * T_chunk;
  if (rows == 0 || H == 0) return CSA_OK;
  const long long grid = rows * ((H + kSimtHeads - 1) / kSimtHeads);
  CSA_REQUIRE(grid < (1ll << 31), CSA_ERR_UNSUPPORTED);
#define CSA_SIMT(TT, DD)                                                                                    \
  attn_simt_kernel<TT, DD><<<static_cast<unsigned>(grid), 256, 0, st>>>(                                   \
      static_cast<const TT*>(q), static_cast<const TT*>(kv_c), idx, static_cast<const TT*>(kv_raw), sink,  \
      tau, W, Tq, row0, T_chunk, H, kv_bstride, k, S, m, raw_cap, q_pos0, static_cast<TT*>(out), lse, mode, \
      static_cast<const TT*>(o_c), lse_c)
  if (dtype == CSA_F32) {
    if (D == 64) CSA_SIMT(float, 64); else CSA_SIMT(float, 128);
  } else {
    if (D == 64) CSA_SIMT(__nv_bfloat16, 64); else CSA_SIMT(__nv_bfloat16, 128);
  }
#undef CSA_SIMT
  return check_launch();
}

}  // namespace csa

using namespace csa;

extern "C" int swa_sink_merge(const void* o_c, const float* lse_c, const void* q, const void* kv_raw,
                              const float* sink, float tau, int W, int B, int T, int row0, int T_chunk, int H,
                              int D, int raw_cap, const int32_t* q_pos0, void* out, int dtype,
                              csa_stream_t stream) {
  CSA_REQUIRE(o_c && lse_c && q && kv_raw && q_pos0 && out, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(B >= 0 && T >= 0 && row0 >= 0 && T_chunk >= 0 && row0 + T_chunk <= T, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(H >= 0 && W >= 0 && raw_cap >= 1 && raw_cap >= W, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(dtype == CSA_F32 || dtype == CSA_BF16, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(D == 64 || D == 128, CSA_ERR_UNSUPPORTED);
  CSA_REQUIRE(aligned16(q) && aligned16(kv_raw) && aligned16(o_c) && aligned16(out), CSA_ERR_ALIGNMENT);
  return launch_attn_simt(q, nullptr, nullptr, kv_raw, sink, tau, W, B, T, row0, T_chunk, H, D, 0, 0, 0, 1,
                          raw_cap, q_pos0, out, nullptr, dtype, kModeWindow, o_c, lse_c,
                          reinterpret_cast<cudaStream_t>(stream));
}
