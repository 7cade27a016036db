// Entry points of the attention steps: CSA sparse attention over the top-k
// entries (cf-1.com/news/5231315 §3.1) and HCA dense attention over every
// visible entry (§3.2), both fused with the 128-token raw window and the sink
// (§3.3).  bf16 runs on the tcgen05 kernel (attn_tc.cu); fp32 runs on CUDA
// cores in fp32 (attn_simt.cu), since the tensor cores have no fp32 kind.
#include "common.cuh"

namespace csa {
int launch_attn_tc(const void* q, const void* kv_c, const int32_t* idx, const void* kv_raw, const float* sink,
                   float tau, int W, int B, int Tq, int row0, int T_chunk, int H, int kv_bstride, int k, int S, int m,
                   int raw_cap, const int32_t* q_pos0, void* out, float* lse, int sparse, int* status,
                   cudaStream_t st);
int launch_attn_simt(const void* q, const void* kv_c, const int32_t* idx, const void* kv_raw, const float* sink,
                     float tau, int W, int B, int Tq, int row0, int T_chunk, int H, int D, int kv_bstride, int k,
                     int S, int m, int raw_cap, const int32_t* q_pos0, void* out, float* lse, int dtype, int mode,
                     const void* o_c, const float* lse_c, cudaStream_t st);
}

using namespace csa;

namespace {
int check_attn_args(const void* q, const void* kv_c, const void* kv_raw, const int32_t* q_pos0, const void* out,
                    int W, int B, int T, int row0, int T_chunk, int H, int D, int raw_cap, int dtype) {
  CSA_REQUIRE(q && kv_c && q_pos0 && out, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(W == 0 || kv_raw != nullptr, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(B >= 0 && T >= 0 && row0 >= 0 && T_chunk >= 0 && row0 + T_chunk <= T, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(H >= 0 && W >= 0, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(W == 0 || raw_cap >= W, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(dtype == CSA_F32 || dtype == CSA_BF16, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(D == 64 || D == 128, CSA_ERR_UNSUPPORTED);
  CSA_REQUIRE(aligned16(q) && aligned16(kv_c) && aligned16(out) && (!kv_raw || aligned16(kv_raw)),
              CSA_ERR_ALIGNMENT);
  return CSA_OK;
}
}  // namespace

extern "C" int sparse_attn_fwd(const void* q, const void* kv_c, const int32_t* idx, const void* kv_raw,
                               const float* sink, float tau, int W, int B, int T, int row0, int T_chunk, int H,
                               int D, int kv_bstride, int k, int raw_cap, const int32_t* q_pos0, void* out,
                               float* lse, int dtype, int32_t* status, csa_stream_t stream) {
  int st = check_attn_args(q, kv_c, kv_raw, q_pos0, out, W, B, T, row0, T_chunk, H, D, raw_cap, dtype);
  if (st != CSA_OK) return st;
  CSA_REQUIRE(idx != nullptr && k >= 1 && kv_bstride >= 1, CSA_ERR_INVALID_ARG);
  if (dtype == CSA_BF16) {
    CSA_REQUIRE(D == 128, CSA_ERR_UNSUPPORTED);
    return launch_attn_tc(q, kv_c, idx, kv_raw, sink, tau, W, B, T, row0, T_chunk, H, kv_bstride, k, 0, 1, raw_cap,
                          q_pos0, out, lse, 1, status_word(status), reinterpret_cast<cudaStream_t>(stream));
  }
  return launch_attn_simt(q, kv_c, idx, kv_raw, sink, tau, W, B, T, row0, T_chunk, H, D, kv_bstride, k, 0, 1,
                          raw_cap, q_pos0, out, lse, dtype, 0, nullptr, nullptr,
                          reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int hca_dense_attn_fwd(const void* q, const void* kv_c, const void* kv_raw, const float* sink,
                                  float tau, int W, int B, int T, int row0, int T_chunk, int H, int D,
                                  int kv_bstride, int S, int m, int raw_cap, const int32_t* q_pos0, void* out,
                                  float* lse, int dtype, int32_t* status, csa_stream_t stream) {
  int st = check_attn_args(q, kv_c, kv_raw, q_pos0, out, W, B, T, row0, T_chunk, H, D, raw_cap, dtype);
  if (st != CSA_OK) return st;
  CSA_REQUIRE(S >= 0 && kv_bstride >= S && m >= 1, CSA_ERR_INVALID_ARG);
  if (dtype == CSA_BF16) {
    CSA_REQUIRE(D == 128, CSA_ERR_UNSUPPORTED);
    return launch_attn_tc(q, kv_c, nullptr, kv_raw, sink, tau, W, B, T, row0, T_chunk, H, kv_bstride > 0 ? kv_bstride : 1,
                          0, S, m, raw_cap, q_pos0, out, lse, 0, status_word(status),
                          reinterpret_cast<cudaStream_t>(stream));
  }
  return launch_attn_simt(q, kv_c, nullptr, kv_raw, sink, tau, W, B, T, row0, T_chunk, H, D, kv_bstride, 0, S,
                          m, raw_cap, q_pos0, out, lse, dtype, 1, nullptr, nullptr,
                          reinterpret_cast<cudaStream_t>(stream));
}
