// Grouped output projection (cf-1.com/news/5231315 §3.4: with many query heads
// the heads are split into groups, each group's concatenated outputs are
// projected down, and the concatenation is projected to the model dimension)
// as two launches of one dense bf16 GEMM on tcgen05:
//   y   = o . blockdiag(w1[0], ..., w1[g-1])^T     (block-diagonal: output
//                                                    tile n reads only its
//                                                    group's K range of o)
//   out = y . w2^T
// C [M x N] = A [M x K] . B[N x K]^T, both operands K-major bf16, fp32
// accumulation in TMEM, bf16 result.
//
// CTA tile 128 x 256, K blocks of 64 (one 128-byte swizzle atom per row),
// four stages of TMA loads.  Warp 0: TMA producer; warp 1: TMEM allocation and
// the MMA issuer (M = 128, N = 256, K = 16 per instruction); warps 2-5: the
// epilogue (TMEM lane quarter = warp % 4, one output row per thread).  All
// waits are bounded in time; a wait that gives up records CSA_ERR_TIMEOUT and
// every role leaves, so the kernel returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace csa {
namespace gm {

constexpr int BM = 128, BN = 256, BK = 64, kStages = 4;
constexpr int kABytes = BM * BK * 2;   // 16 KB
constexpr int kBBytes = BN * BK * 2;   // 32 KB
constexpr int kThreads = 6 * 32;

struct __align__(1024) Smem {
  uint8_t a[kStages][kABytes];
  uint8_t b[kStages][kBBytes];
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full;
  uint32_t tmem;
  int abort_flag;
};

struct Maps {
  CUtensorMap a;   // [M, lda] bf16, box 64 x 128
  CUtensorMap b;   // [N, ldb] bf16, box 64 x 256
};

struct Args {
  __nv_bfloat16* c;
  int ldc, M, N, K;
  int group_k;        // > 0: output tile n reads A columns [(n0 / group_n) group_k, + group_k)
  int group_n;        // output columns per group
  int* status;
  unsigned long long wait_ns;
};

__device__ __forceinline__ bool gwait(uint64_t* bar, uint32_t parity, const Args& a, volatile int* abort_flag,
                                      int site) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_ns() - t0 > a.wait_ns) break;
  }
  atomicCAS(a.status, 0, CSA_ERR_TIMEOUT | (site << 8));
  *abort_flag = 1;
  return false;
}

__device__ __forceinline__ uint64_t desc_k(uint32_t base, int j) {
  return make_sdesc(base + 32 * j, 16, 1024, kLayoutSw128);
}

__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ Args args,
                                                           const __grid_constant__ Maps maps) {
  extern __shared__ __align__(1024) uint8_t gm_smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(gm_smem_raw) + 1023) &
                                      ~static_cast<uintptr_t>(1023));
  const Args& a = args;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;
  // N tiles vary fastest: the CTAs sharing an A row block (every N tile of a
  // group, or of the whole row) run together and read it once from DRAM
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int a_k0 = a.group_k > 0 ? (n0 / a.group_n) * a.group_k : 0;
  const int nk = (a.group_k > 0 ? a.group_k : a.K) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.acc_full, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem, BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem;

  if (warp == 0) {
    // ---- TMA producer
    if (lane == 0) {
      int armed = -1;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kStages;
        if (kb >= kStages && !gwait(&sm.empty[s], ((kb / kStages) - 1) & 1, a, abort_flag, 1)) break;
        mbar_arrive_expect_tx(&sm.full[s], kABytes + kBBytes);
        tma_load_2d(smem_u32(sm.a[s]), reinterpret_cast<uint64_t>(&maps.a), a_k0 + kb * BK, m0, &sm.full[s]);
        tma_load_2d(smem_u32(sm.b[s]), reinterpret_cast<uint64_t>(&maps.b), kb * BK, n0, &sm.full[s]);
        armed = kb;
      }
      if (*abort_flag && armed >= 0) {
        // copies still in flight land within microseconds
        const uint64_t t0 = global_ns();
        while (!mbar_try_wait(&sm.full[armed % kStages], (armed / kStages) & 1))
          if (global_ns() - t0 > 1000000ull) break;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(BM, BN, 0, 0);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kStages;
        if (!gwait(&sm.full[s], (kb / kStages) & 1, a, abort_flag, 2)) break;
        tc_fence_after();
        const uint32_t ab = smem_u32(sm.a[s]), bb = smem_u32(sm.b[s]);
#pragma unroll
        for (int j = 0; j < BK / 16; ++j) mma_bf16(tmem, desc_k(ab, j), desc_k(bb, j), idesc, (kb | j) ? 1u : 0u);
        tc_commit(&sm.empty[s]);
      }
      // the epilogue waits for every MMA (also after an abort, so TMEM is
      // released only when the tensor pipe is done with it)
      tc_commit(&sm.acc_full);
    }
    __syncwarp();
  } else {
    // ---- epilogue: thread = output row
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    bool ok = mbar_try_wait(&sm.acc_full, 0);
    if (!ok) {
      const uint64_t t0 = global_ns();
      while (!(ok = mbar_try_wait(&sm.acc_full, 0)))
        if (global_ns() - t0 > a.wait_ns + 1000000ull) break;
      if (!ok) atomicCAS(a.status, 0, CSA_ERR_TIMEOUT | (3 << 8));
    }
    ok = __all_sync(0xffffffffu, ok) && !*abort_flag;
    if (ok) {
      tc_fence_after();
      const int row = m0 + r;
      __nv_bfloat16* crow = a.c + static_cast<size_t>(row) * a.ldc + n0;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_addr + c0, v);
        tmem_ld_wait();
        if (row < a.M) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
            w[e] = *reinterpret_cast<uint32_t*>(&h);
          }
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            *reinterpret_cast<uint4*>(crow + c0 + 8 * q4) = make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2],
                                                                       w[4 * q4 + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

}  // namespace gm

namespace {
PFN_cuTensorMapEncodeTiled_v12000 gm_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2D bf16 map over [rows, cols] (row stride ld elements), box 64 x box_rows, 128-byte swizzle.
bool gm_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows) {
  auto enc = gm_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// C [M, N] (ldc) = A [M, K_a] (lda) . B [N, K_b] (ldb)^T over K (or, grouped,
// over each output group's K range of A).
int gm_launch(const void* A, int lda, int K_a, const void* B, int ldb, int K_b, void* C, int ldc, int M, int N,
              int K, int group_k, int group_n, int* status, cudaStream_t st) {
  using namespace gm;
  gm::Maps maps;
  if (!gm_map(&maps.a, A, static_cast<uint64_t>(M), static_cast<uint64_t>(K_a), static_cast<uint64_t>(lda), BM) ||
      !gm_map(&maps.b, B, static_cast<uint64_t>(N), static_cast<uint64_t>(K_b), static_cast<uint64_t>(ldb), BN))
    return CSA_ERR_CUDA;
  gm::Args a;
  a.c = static_cast<__nv_bfloat16*>(C);
  a.ldc = ldc; a.M = M; a.N = N; a.K = K;
  a.group_k = group_k; a.group_n = group_n;
  a.status = status;
  a.wait_ns = wait_limit_ns();
  const size_t smem = sizeof(Smem) + 1024;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return set_cuda_error(e);
    attr_set = true;
  }
  CSA_REQUIRE((M + BM - 1) / BM < 65536, CSA_ERR_UNSUPPORTED);
  dim3 grid(N / BN, (M + BM - 1) / BM);
  gemm_kernel<<<grid, kThreads, smem, st>>>(a, maps);
  return check_launch();
}
}  // namespace

}  // namespace csa

using namespace csa;

extern "C" int grouped_out_proj(const void* o, int M, int H, int D, int groups, int d_g, const void* w1,
                                const void* w2, int d_model, void* y, void* out, int32_t* status,
                                csa_stream_t stream) {
  CSA_REQUIRE(o && w1 && w2 && y && out, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(M >= 0 && H > 0 && D > 0 && groups > 0 && d_g > 0 && d_model > 0, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(H % groups == 0, CSA_ERR_INVALID_ARG);
  const long long kg = static_cast<long long>(H / groups) * D;   // K of one group
  const long long ny = static_cast<long long>(groups) * d_g;     // y columns = K of the second product
  CSA_REQUIRE(kg % gm::BK == 0 && d_g % gm::BN == 0 && ny % gm::BK == 0 && d_model % gm::BN == 0,
              CSA_ERR_UNSUPPORTED);
  CSA_REQUIRE(static_cast<long long>(H) * D < (1ll << 31) && ny < (1ll << 31), CSA_ERR_UNSUPPORTED);
  CSA_REQUIRE(aligned16(o) && aligned16(w1) && aligned16(w2) && aligned16(y) && aligned16(out), CSA_ERR_ALIGNMENT);
  if (M == 0) return CSA_OK;
  int* st_word = status_word(status);
  CSA_REQUIRE(st_word != nullptr, CSA_ERR_CUDA);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int HD = H * D;
  // y = o . blockdiag(w1)^T: w1 is [groups * d_g, kg]; output tile n (group
  // n0 / d_g) reads o's columns [group * kg, + kg)
  int r = gm_launch(o, HD, HD, w1, static_cast<int>(kg), static_cast<int>(kg), y, static_cast<int>(ny), M,
                    static_cast<int>(ny), static_cast<int>(kg), static_cast<int>(kg), d_g, st_word, st);
  if (r != CSA_OK) return r;
  // out = y . w2^T
  return gm_launch(y, static_cast<int>(ny), static_cast<int>(ny), w2, static_cast<int>(ny), static_cast<int>(ny), out,
                   d_model, M, d_model, static_cast<int>(ny), 0, 0, st_word, st);
}
