// Lightning-indexer score on tcgen05 block-scaled FP4 MMA
// (cf-1.com/news/5231315 §3.4: the indexer is low-rank and low-precision, its
// QK runs in FP4; §4.4: index scores are stored in BF16).
//
//   score[t, s] = sum_h w[t,h] * ReLU( qhat[t,h,:] . khat[s,:] )
//
// The contraction runs "entries x (token, head)": the MMA's M = 128 compressed
// entries, N (token, head) pairs (N/HI tokens x HI heads; N = 112 for prefill
// chunks, 16 for decode chunks), K = 64 FP4 values (one MMA; DI = 32 is
// zero-padded).  The accumulator tile lives in
// TMEM with one entry per lane, so each epilogue thread owns one entry and the
// HI heads of a token sit in adjacent columns of its own lane: the weighted
// ReLU head-sum needs no cross-thread reduction, and the 32 threads of a warp
// store 32 consecutive scores of a token row (coalesced).  Block scales (UE4M3,
// one per 16 values) go smem -> TMEM with tcgen05.cp; the global scales are
// folded into w.  Operands are staged with cp.async into the canonical
// no-swizzle K-major layout (8 rows x 16 B core matrices).
//
// A CTA owns one tile of N (token, head) rows and up to kTilesPerCta entry
// tiles, streamed through a ring of shared-memory stages.  Work above the
// causal limit (entries no query of the tile can see) is never launched.
#include "common.cuh"

namespace csa {

constexpr int kIdxThreads = 128;
// entry tiles per CTA and shared-memory stages: the narrow (decode) tile
// streams more tiles per CTA through a deeper ring
template <int NQ> struct IdxShape {
  static constexpr int tiles = NQ > 16 ? 8 : 16;
  static constexpr int stages = NQ > 16 ? 2 : 4;
};
// The narrow tile double-buffers its accumulator (the MMA of tile j+1 runs
// during the epilogue of tile j); the wide one cannot without halving the
// CTAs that share an SM's TMEM.
template <int NQ> struct IdxAcc { static constexpr int bufs = NQ <= 16 ? 2 : 1; };
// TMEM columns: accumulators and key scales (SFA, 4 columns) bufs times each,
// query scales (SFB) 4, rounded to a power of two
template <int NQ> struct IdxTmem {
  static constexpr int used = IdxAcc<NQ>::bufs * (NQ + 4) + 4;
  static constexpr uint32_t cols = used <= 32 ? 32 : (used <= 64 ? 64 : (used <= 128 ? 128 : 256));
};
// shared-memory floor per CTA so that no more CTAs share an SM than its 512
// TMEM columns hold (a CTA waiting in tcgen05.alloc would only idle)
template <int NQ> struct IdxFloor {
  static constexpr size_t bytes = IdxTmem<NQ>::cols == 256   ? 96 * 1024
                                  : IdxTmem<NQ>::cols == 128 ? 48 * 1024
                                  : IdxTmem<NQ>::cols == 64  ? 27 * 1024
                                                             : 0;
};

template <int NS>
struct __align__(128) IdxSmem {
  uint8_t qB[128 * 32];
  uint8_t kA[NS][128 * 32];
  uint8_t sfa[NS][512];
  uint8_t sfb[512];
  float w[128];
  uint64_t mbar[2];
  uint32_t tmem;
  int abort_flag;
};

// Canonical no-swizzle K-major placement: 8-row x 16-byte core matrices,
// row groups 256 B apart, the two 16-byte K chunks of a row 128 B apart.
__device__ __forceinline__ uint32_t cm_off(int r, int c16) { return (r >> 3) * 256 + c16 * 128 + (r & 7) * 16; }
// Scale-factor placement for tcgen05.cp 32x128b: row r -> 16-byte line r % 32,
// 4-byte word r / 32 of that line, byte j = block index along K.
__device__ __forceinline__ uint32_t sf_off(int r) { return (r & 31) * 16 + (r >> 5) * 4; }

// NQ = MMA N: 128 (token, head) columns for prefill chunks, 16 for decode
// (a chunk of at most 16 / HI query tokens): the narrow tile needs 32 TMEM
// columns and little shared memory, so many CTAs share an SM and keep enough
// key loads in flight to stream the whole NVFP4 key cache from HBM.
template <int HI, typename TS, int NQ>
__global__ void __launch_bounds__(kIdxThreads) indexer_kernel(
    const uint8_t* __restrict__ q_fp4, const uint8_t* __restrict__ q_sf, const uint8_t* __restrict__ k_fp4,
    const uint8_t* __restrict__ k_sf, const float* __restrict__ w, float gscale, int T, int row0, int T_chunk,
    int S, int k_bstride, int DI, int m, const int32_t* __restrict__ q_pos0, TS* __restrict__ score, int ld,
    int n_qtiles, int n_chunks, int* __restrict__ status, unsigned long long wait_ns) {
  constexpr int TQ = NQ / HI;
  constexpr uint32_t kIdxTmemCols = IdxTmem<NQ>::cols;
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  constexpr int NS = IdxShape<NQ>::stages;
  constexpr int kTilesPerCta = IdxShape<NQ>::tiles;
  IdxSmem<NS>& sm = *reinterpret_cast<IdxSmem<NS>*>(dsm_raw);
  const int tid = threadIdx.x, warp = tid >> 5;

  int blk = blockIdx.x;
  const int ch = blk % n_chunks; blk /= n_chunks;
  const int qt = blk % n_qtiles;
  const int bi = blk / n_qtiles;
  const int tq0 = qt * TQ;
  const int ntok = min(TQ, T_chunk - tq0);
  const long long pbase = static_cast<long long>(q_pos0[bi]) + row0 + tq0;
  long long vis_last = (pbase + ntok - 1 + 1) / m;
  if (vis_last > S) vis_last = S;
  const int n_et = static_cast<int>((vis_last + 127) / 128);
  const int et0 = ch * kTilesPerCta;
  const int et1 = min(n_et, et0 + kTilesPerCta);
  if (et0 >= et1) return;  // uniform: nothing visible for this CTA
  const int ntiles = et1 - et0;

  if (warp == 0) {
    tmem_alloc(&sm.tmem, kIdxTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&sm.mbar[0], 1);
    mbar_init(&sm.mbar[1], 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  const int dbytes = DI / 2;       // packed bytes per row (16 or 32)
  const int sfn = DI / 16;         // scale bytes per row (2 or 4)

  // ---- q tile (B operand), SFB and folded weights: row n = t * HI + h
  {
    const int n = tid;
    const int t = n / HI;
    const bool ok = n < NQ && t < ntok;
    const size_t qrow = (static_cast<size_t>(bi) * T + row0 + tq0) * HI + n;
    const uint8_t* src = q_fp4 + (ok ? qrow : 0) * dbytes;
    cp_async16(smem_u32(sm.qB + cm_off(n, 0)), src, ok ? 16u : 0u);
    cp_async16(smem_u32(sm.qB + cm_off(n, 1)), src + (dbytes > 16 ? 16 : 0), (ok && dbytes > 16) ? 16u : 0u);
    uint32_t sfw = 0;
    if (ok) {
      const uint8_t* sp = q_sf + qrow * sfn;
      for (int j = 0; j < sfn; ++j) sfw |= static_cast<uint32_t>(sp[j]) << (8 * j);
    }
    *reinterpret_cast<uint32_t*>(sm.sfb + sf_off(n)) = sfw;
    sm.w[n] = ok ? w[qrow] * gscale : 0.f;
  }
  auto load_k_tile = [&](int et, int stage) {
    const int r = tid;
    const int s = et * 128 + r;
    const bool ok = s < S;
    const size_t krow = static_cast<size_t>(bi) * k_bstride + (ok ? s : 0);
    const uint8_t* src = k_fp4 + krow * dbytes;
    cp_async16(smem_u32(sm.kA[stage] + cm_off(r, 0)), src, ok ? 16u : 0u);
    cp_async16(smem_u32(sm.kA[stage] + cm_off(r, 1)), src + (dbytes > 16 ? 16 : 0),
               (ok && dbytes > 16) ? 16u : 0u);
    if (sfn == 4) {
      // the row's four scale bytes as one asynchronous 4-byte copy
      cp_async4(smem_u32(sm.sfa[stage] + sf_off(r)), k_sf + krow * 4, ok ? 4u : 0u);
    } else {
      uint32_t sfw = 0;
      if (ok) {
        const uint8_t* sp = k_sf + krow * sfn;
        for (int j = 0; j < sfn; ++j) sfw |= static_cast<uint32_t>(sp[j]) << (8 * j);
      }
      *reinterpret_cast<uint32_t*>(sm.sfa[stage] + sf_off(r)) = sfw;
    }
  };
#pragma unroll
  for (int p = 0; p < NS; ++p) {
    if (p < ntiles) load_k_tile(et0 + p, p);
    cp_async_commit();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem;
  constexpr int NB = IdxAcc<NQ>::bufs;
  // per buffer b: accumulator at b NQ, key scales at NB NQ + 4 b; query scales last
  const uint32_t t_sfa0 = tmem + NB * NQ, t_sfb = tmem + NB * NQ + 4 * NB;
  constexpr uint32_t idesc = idesc_nvfp4(128, NQ);
  const uint64_t bdesc = make_sdesc(smem_u32(sm.qB), 128, 256, kLayoutNone);
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  // the narrow tile keeps its NQ folded weights in registers
  float wr[NQ <= 16 ? NQ : 1];
  if constexpr (NQ <= 16) {
#pragma unroll
    for (int c = 0; c < NQ; ++c) wr[c] = sm.w[c];
  }
  // MMA of tile j (thread 0): scales to TMEM, block-scaled FP4 MMA, commit
  auto issue_mma = [&](int j) {
    if (tid == 0) {
      tc_fence_after();
      if (j == 0) tmem_cp_32x128b_x4(t_sfb, make_sdesc(smem_u32(sm.sfb), 128, 128, kLayoutNone));
      const int stage = j % NS;
      const uint32_t t_sfa = t_sfa0 + 4 * (j % NB);
      tmem_cp_32x128b_x4(t_sfa, make_sdesc(smem_u32(sm.sfa[stage]), 128, 128, kLayoutNone));
      const uint64_t adesc = make_sdesc(smem_u32(sm.kA[stage]), 128, 256, kLayoutNone);
      mma_nvfp4(tmem + (j % NB) * NQ, adesc, bdesc, idesc, t_sfa, t_sfb, 0u);
      tc_commit(&sm.mbar[j % NB]);
    }
  };
  if constexpr (NB == 2) {
    cp_async_wait<NS - 1>();
    fence_proxy_async();
    __syncthreads();
    issue_mma(0);
  }

  for (int j = 0; j < ntiles; ++j) {
    const int stage = j % NS;
    if constexpr (NB == 2) {
      // tile j+1's keys are in (groups 0 .. j+1 of NS + j committed); its MMA
      // goes into the other accumulator, whose epilogue (tile j-1) is done
      if (j + 1 < ntiles) {
        cp_async_wait<NS - 2>();
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (sm.abort_flag) break;
        issue_mma(j + 1);
      }
    } else {
      cp_async_wait<NS - 1>();
      fence_proxy_async();
      __syncthreads();
      if (sm.abort_flag) break;
      issue_mma(j);
    }
    if (!mbar_wait(&sm.mbar[j % NB], static_cast<uint32_t>((j / NB) & 1), status, wait_ns)) sm.abort_flag = 1;
    tc_fence_after();
    // the MMA has consumed this stage: prefetch NS tiles ahead into it
    if (j + NS < ntiles) load_k_tile(et0 + j + NS, stage);
    cp_async_commit();

    // ---- epilogue: this thread owns entry s; columns are (token, head) pairs
    const uint32_t t_acc = tmem + (j % NB) * NQ;
    const int s = (et0 + j) * 128 + tid;
    const bool s_ok = s < S;
    constexpr int CB = NQ % 32 == 0 ? 32 : 16;   // columns per TMEM load
#pragma unroll 1
    for (int c0 = 0; c0 < NQ; c0 += CB) {
      uint32_t v[CB];
      if constexpr (CB == 32) tmem_ld32(t_acc + lane_base + c0, v);
      else tmem_ld16(t_acc + lane_base + c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int tt = 0; tt < CB / HI; ++tt) {
        const int t = c0 / HI + tt;
        if constexpr (NQ <= 16) {
          if (t >= ntok) break;   // uniform: a decode chunk fills few of the tile's tokens
        }
        float acc = 0.f;
#pragma unroll
        for (int h = 0; h < HI; ++h) {
          const float wv = NQ <= 16 ? wr[(tt * HI + h) % (NQ <= 16 ? NQ : 1)] : sm.w[c0 + tt * HI + h];
          acc = fmaf(wv, fmaxf(__uint_as_float(v[tt * HI + h]), 0.f), acc);
        }
        const long long p = pbase + t;
        if (s_ok && (NQ <= 16 || t < ntok) && static_cast<long long>(m) * (s + 1) - 1 <= p)
          score[(static_cast<size_t>(bi) * T_chunk + tq0 + t) * ld + s] = static_cast<TS>(acc);
      }
    }
    tc_fence_before();
  }
  cp_async_wait<0>();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kIdxTmemCols);
}

}  // namespace csa

using namespace csa;

extern "C" int indexer_score(const uint8_t* q_fp4, const uint8_t* q_sf, float q_gscale, const uint8_t* k_fp4,
                             const uint8_t* k_sf, float k_gscale, const float* w, int B, int T, int row0,
                             int T_chunk, int S, int k_bstride, int HI, int DI, int m, const int32_t* q_pos0,
                             void* score, int score_dtype, int score_ld, int32_t* status_out,
                             csa_stream_t stream) {
  CSA_REQUIRE(q_fp4 && q_sf && k_fp4 && k_sf && w && q_pos0 && score, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(B >= 0 && T >= 0 && row0 >= 0 && T_chunk >= 0 && row0 + T_chunk <= T, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(S >= 0 && k_bstride >= S && m >= 1 && score_ld >= S, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(q_gscale > 0.f && k_gscale > 0.f, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(score_dtype == CSA_F32 || score_dtype == CSA_BF16, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(DI == 32 || DI == 64, CSA_ERR_UNSUPPORTED);
  CSA_REQUIRE(HI == 1 || HI == 2 || HI == 4 || HI == 8, CSA_ERR_UNSUPPORTED);
  CSA_REQUIRE(aligned16(q_fp4) && aligned16(k_fp4), CSA_ERR_ALIGNMENT);
  CSA_REQUIRE(DI != 64 || (reinterpret_cast<uintptr_t>(k_sf) & 3) == 0, CSA_ERR_ALIGNMENT);
  if (B == 0 || T_chunk == 0 || S == 0) return CSA_OK;
  // N = 16 for decode-sized chunks; N = 112 (TMEM 128 columns, four CTAs per
  // SM) for prefill chunks
  const bool narrow = T_chunk * HI <= 16;
  constexpr int kWide = 112;
  const int TQ = (narrow ? 16 : kWide) / HI;
  const int n_qtiles = (T_chunk + TQ - 1) / TQ;
  const int n_et = (S + 127) / 128;
  const int tiles_per_cta = narrow ? IdxShape<16>::tiles : IdxShape<kWide>::tiles;
  const int n_chunks = (n_et + tiles_per_cta - 1) / tiles_per_cta;
  const long long grid = static_cast<long long>(B) * n_qtiles * n_chunks;
  CSA_REQUIRE(grid < (1ll << 31), CSA_ERR_UNSUPPORTED);
  const size_t smem_min = (narrow ? sizeof(IdxSmem<IdxShape<16>::stages>) : sizeof(IdxSmem<IdxShape<kWide>::stages>)) + 1024;
  const size_t floor_b = narrow ? IdxFloor<16>::bytes : IdxFloor<kWide>::bytes;
  const size_t smem = smem_min > floor_b ? smem_min : floor_b;
  const float g = q_gscale * k_gscale;
  int* status = status_word(status_out);
  CSA_REQUIRE(status != nullptr, CSA_ERR_CUDA);
  const unsigned long long wait_ns = wait_limit_ns();
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#define CSA_IDX_LAUNCH_NQ(HIV, TS, NQV)                                                                        \
  do {                                                                                                         \
    cudaFuncSetAttribute(indexer_kernel<HIV, TS, NQV>, cudaFuncAttributeMaxDynamicSharedMemorySize,            \
                         static_cast<int>(smem));                                                              \
    indexer_kernel<HIV, TS, NQV><<<static_cast<unsigned>(grid), kIdxThreads, smem, st>>>(                      \
        q_fp4, q_sf, k_fp4, k_sf, w, g, T, row0, T_chunk, S, k_bstride, DI, m, q_pos0, static_cast<TS*>(score), \
        score_ld, n_qtiles, n_chunks, status, wait_ns);                                                                 \
  } while (0)
#define CSA_IDX_LAUNCH(HIV, TS)                                 \
  do {                                                          \
    if (narrow) CSA_IDX_LAUNCH_NQ(HIV, TS, 16);                 \
    else CSA_IDX_LAUNCH_NQ(HIV, TS, kWide);                     \
  } while (0)
#define CSA_IDX_DT(HIV)                                                \
  do {                                                                 \
    if (score_dtype == CSA_F32) CSA_IDX_LAUNCH(HIV, float);            \
    else CSA_IDX_LAUNCH(HIV, __nv_bfloat16);                           \
  } while (0)
  switch (HI) {
    case 1: CSA_IDX_DT(1); break;
    case 2: CSA_IDX_DT(2); break;
    case 4: CSA_IDX_DT(4); break;
    default: CSA_IDX_DT(8); break;
  }
#undef CSA_IDX_DT
#undef CSA_IDX_LAUNCH
#undef CSA_IDX_LAUNCH_NQ
  return check_launch();
}
