// bf16 attention on tcgen05 with TMEM accumulators: CSA sparse attention over
// the top-k entries (cf-1.com/news/5231315 §3.1), HCA dense attention over all
// visible entries (§3.2), both with the 128-token raw window and the sink in
// the softmax denominator (§3.3).
//
// Orientation.  MQA shares one K=V row between all heads, so a KV tile is the
// operand every head reuses.  The kernel puts KV rows on the MMA's M side:
//   S^T [128 KV rows x N] = KV [128 x D] . Q^T        (A = KV, K-major; B = Q)
//   O^T [D x N]          += V^T [D x 128] . P^T       (A = the same KV tile read
//                                                       MN-major; B = P^T)
// N = (query tokens sharing the KV set) x heads: one token for CSA (each has
// its own top-k set), 128/H tokens for HCA.  With H = 64 this keeps M = 128
// (full tcgen05 rate) where the transposed form would need M = 64.
//
// Roles (one CTA per SM, persistent over work units):
//   producer warp (1): gathers the unit's KV rows (top-k entries or every
//     visible entry, then the raw-window tokens) into 128-row tiles with TMA
//     tile::gather4 (four rows per instruction, one 4-row group per lane, the
//     128-byte swizzle applied by the TMA unit); Q arrives by a 2D TMA load.
//     Completion is tracked by mbarrier transaction bytes.  The compressed
//     part of the row list is padded to a multiple of 4 rows (masked rows,
//     zero-filled by out-of-range coordinates) so a group never mixes sources.
//   MMA warp (1): issues QK(i+1) before PV(i) so the tensor core works on the
//     next tile while the softmax runs.
//   softmax warpgroups (4 warps each): thread = TMEM lane = KV row of S^T
//     and dim row of O^T; a warpgroup owns 16 (N = 64) or 32 (N = 128) columns.  Column maxima are warp
//     redux.sync.max + a 4-warp exchange; running maxima are raised only when a
//     tile exceeds them by 2^8 (then O^T and the row sums are rescaled), row
//     sums stay per thread until the unit's end.  P^T goes to shared memory as
//     bf16 (MN-major, swizzled) for the PV MMA.
// All waits are bounded; a wait that gives up sets the device status word and
// an abort flag that every role polls, so the kernel always returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

// Compile-time event trace for pipeline analysis (debug builds only):
// globaltimer stamps of each role's per-tile events in CTA 0.
#ifdef CSA_TRACE
__device__ unsigned long long* g_csa_trace;
#define CSA_TR(unit, tile, ev)                                                                   \
  do {                                                                                           \
    if (blockIdx.x == 0 && g_csa_trace != nullptr && (unit) < 64 && (tile) < 16) {               \
      unsigned long long t_;                                                                     \
      asm volatile("mov.u64 %0, %%clock64;" : "=l"(t_));                                         \
      g_csa_trace[((unit) * 16 + (tile)) * 8 + (ev)] = t_;                                        \
    }                                                                                            \
  } while (0)
extern "C" int csa_debug_set_trace(void* p) {
  return cudaMemcpyToSymbol(g_csa_trace, &p, sizeof(p)) == cudaSuccess ? 0 : 4;
}
#else
#define CSA_TR(unit, tile, ev) do { } while (0)
#endif

namespace csa {

constexpr int kTcTile = 128;   // KV rows per tile
constexpr int kTcDim = 128;    // head dim

// NB = number of 64-column blocks of N; each softmax warpgroup owns kCW columns.
template <int NB>
struct TcCfg {
  static constexpr int N = 64 * NB;                       // MMA N (token, head) columns
  static constexpr int kCW = NB == 1 ? 16 : 32;            // columns per softmax warpgroup
  static constexpr int kGroups = N / kCW;                  // softmax warpgroups
  static constexpr int kSoftWarps = 4 * kGroups;
  // Two producer warps: with 19 warps per CTA no SM sub-partition (16K
  // registers each) holds more than five, which leaves 96 registers per thread;
  // a sixth warp on a sub-partition would cap every thread at 80 and spill.
  // Two suffice for every tile kind: TMA loads contiguous tiles, and the
  // per-row gathers use loops with little address arithmetic per row.
  static constexpr int kProdWarps = 2;
  static constexpr int kThreads = 32 * (kSoftWarps + kProdWarps + 1);
  static constexpr int kStages = NB == 1 ? 4 : 2;
  static constexpr int kQBytes = N * kTcDim * 2;
  static constexpr int kKVBytes = kTcTile * kTcDim * 2;   // 32 KB
  static constexpr int kPBytes = kTcTile * N * 2;
  // S^T and P^T buffers: three for N = 64, so QK runs two tiles ahead of the
  // softmax and ahead of the PV of the tile before (the tensor pipe executes in
  // issue order); two for N = 128 (TMEM is full)
  static constexpr int kSBuf = NB == 1 ? 3 : 2;
  static constexpr uint32_t kOCol = kSBuf * N;             // O^T x2 after the S buffers
  static constexpr uint32_t kTmemCols = 512;               // 320 or 512 used
};

struct TcUnit {
  int b, r0, ntok, n_c, n_w, jlo, p0, nt, hoff;
  int n_all;   // leading rows valid for every token of the unit
  int n_cp;    // n_c rounded up to 4: window rows start here
};

struct TcMaps {
  CUtensorMap q;     // [B*Tq*H, 128] bf16, box 64 x H (one token)
  CUtensorMap kv;    // [B*kv_bstride, 128] bf16, box 64 x 128 (one tile half)
  CUtensorMap raw;   // [B*raw_cap, 128] bf16, box 64 x 128 (one tile half)
};

constexpr int kTcMaxIdxTiles = 8;   // top-k up to 1024 entries per query

template <int NB>
struct __align__(1024) TcSmem {
  using C = TcCfg<NB>;
  uint8_t q[2][C::kQBytes];
  uint8_t kv[C::kStages][C::kKVBytes];
  uint8_t p[C::kSBuf][C::kPBytes];
  uint64_t kv_full[C::kStages], kv_empty[C::kStages];
  uint64_t q_full[2], q_empty[2], o_full[2], o_empty[2];
  uint64_t s_full[C::kSBuf], s_free[C::kSBuf], p_full[C::kSBuf], p_empty[C::kSBuf];
  float xch[C::kGroups][4][C::kCW];
  float mcol[C::kGroups][C::kCW];
  float alpha[C::kGroups][C::kCW];
  float dlt[C::kGroups][C::kCW];
  float oscale[C::kGroups][C::kCW];   // output scales of a unit whose read-out is pending
  float sink_l2[128];      // sink logits in log2 units (-inf without a sink)
  TcUnit info[2];
  uint32_t tmem;
  int abort_flag;
};

struct TcArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* kv_c;
  const int32_t* idx;
  const __nv_bfloat16* kv_raw;
  const float* sink;
  const int32_t* q_pos0;
  __nv_bfloat16* out;
  float* lse;
  int* status;
  float scale_log2;      // tau * log2(e)
  int W, Tq, row0, T_chunk, H, kv_bstride, k, S, m, raw_cap;
  int G;                 // tokens per unit
  int hshift;            // log2(H)
  int sparse;            // 1: CSA (idx), 0: HCA (all visible entries)
  int units_per_b;
  int Hq;                // heads per token in q / out / lse / sink (H = heads per unit)
  int hsplit;            // units per token (Hq / H): few-token calls split the heads
  int n_units;
  int kv_rows, raw_rows; // rows of the kv / raw tensor maps (an index equal to them is out of range)
};

// Time-bounded wait shared by every role: returns false at once when another
// role has aborted, and aborts the CTA (recording the wait site) after kWaitNs.
__device__ __forceinline__ bool tc_wait_site(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag,
                                             int site) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_ns() - t0 > kWaitNs) break;
  }
  atomicCAS(status, 0, CSA_ERR_TIMEOUT | (site << 8));
  *abort_flag = 1;
  return false;
}
#define tc_wait(bar, parity, status, abort_flag) tc_wait_site(bar, parity, status, abort_flag, __LINE__)

__device__ __forceinline__ float redux_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ float fast_ex2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float fast_rcp(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float fast_lg2(float x) {
  float r;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
// d = a * b + c and x += y on pairs of floats (packed f32x2 pipe ops).
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                      float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void fadd2(float& x0, float& x1, float y0, float y1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%0, %1};\n\tmov.b64 rb, {%2, %3};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(x0), "+f"(x1)
      : "f"(y0), "f"(y1));
}
// Running-max sentinel for a column that has seen no valid row yet (finite, so
// every softmax argument stays finite; masked rows are -inf and give 0).
constexpr float kNoRowMax = -1e30f;
// Largest softmax argument (log2 units above the running max) taken without a
// group-wide max update; larger ones mark the unit for exact recomputation.
constexpr float kClampD = 64.0f;
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
// the two bf16 halves of a packed pair, widened exactly to fp32
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ bool bar_red_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// Descriptor of a K-major SW128 operand (rows of 128 B, 8-row atoms 1024 B):
// K-step j (16 bf16) of a [rows x 128] bf16 block lives in region j/4 at byte j%4*32.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t base, uint32_t region_bytes, int j) {
  return make_sdesc(base + (j >> 2) * region_bytes + (j & 3) * 32, 16, 1024, kLayoutSw128);
}
// Descriptor of an MN-major SW128 operand (K rows of 128 B = 64 MN values,
// 64-wide MN blocks `region_bytes` apart): K-step j = rows 16j..16j+15.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t base, uint32_t region_bytes, int j) {
  return make_sdesc(base + j * 2048, region_bytes, 1024, kLayoutSw128);
}
// byte offset of 16-byte chunk c (0..15 for a 256-byte row) of row r in a
// two-region SW128 block of `rows` rows
__device__ __forceinline__ uint32_t sw128_off(int r, int c, int rows) {
  return (c >> 3) * (rows * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

// Exact fallback for columns [col_begin, col_end) of one unit, on CUDA cores:
// warp w of nw takes every nw-th column (lane = 4 head dims), an online softmax in
// fp32 over the entries and window rows, then the sink, as the formula states.
// Used only for units whose fast path was inexact (a logit above the seeded
// max by more than 2^64, or every weight underflowing).
__device__ __noinline__ void tc_unit_exact(const TcArgs a, const TcUnit inf, const float* sink_l2, int col_begin,
                                           int col_end, int w, int nw) {
  const int lane = threadIdx.x & 31;
  for (int col = col_begin + w; col < col_end; col += nw) {
    const int g = col >> a.hshift;
    if (g >= inf.ntok) continue;
    const int h = inf.hoff + (col & (a.H - 1));
    const int p = inf.p0 + g;
    const size_t qrow = (static_cast<size_t>(inf.b) * a.Tq + a.row0 + inf.r0 + g) * a.Hq + h;
    float qv[4];
    {
      const uint2 u = *reinterpret_cast<const uint2*>(a.q + qrow * kTcDim + 4 * lane);
      const __nv_bfloat162 q01 = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
      const __nv_bfloat162 q23 = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
      qv[0] = __low2float(q01); qv[1] = __high2float(q01); qv[2] = __low2float(q23); qv[3] = __high2float(q23);
    }
    float m = -INFINITY, l = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
    auto visit = [&](const __nv_bfloat16* row) {
      const uint2 u = *reinterpret_cast<const uint2*>(row + 4 * lane);
      const __nv_bfloat162 k01 = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
      const __nv_bfloat162 k23 = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
      const float kv[4] = {__low2float(k01), __high2float(k01), __low2float(k23), __high2float(k23)};
      float dot = qv[0] * kv[0] + qv[1] * kv[1] + qv[2] * kv[2] + qv[3] * kv[3];
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      const float x = dot * a.scale_log2;
      const float mn = fmaxf(m, x);
      const float corr = exp2f(m - mn);
      const float pw = exp2f(x - mn);
      l = fmaf(l, corr, pw);
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] = fmaf(acc[e], corr, pw * kv[e]);
      m = mn;
    };
    if (a.sparse) {
      const int32_t* ir = a.idx + (static_cast<size_t>(inf.b) * a.T_chunk + inf.r0 + g) * a.k;
      for (int j = 0; j < inf.n_c; ++j)
        visit(a.kv_c + (static_cast<size_t>(inf.b) * a.kv_bstride + ir[j]) * kTcDim);
    } else {
      const int nv = min(a.S, (p + 1) / a.m);
      for (int e = 0; e < nv; ++e) visit(a.kv_c + (static_cast<size_t>(inf.b) * a.kv_bstride + e) * kTcDim);
    }
    if (a.W > 0)
      for (int j = max(0, p - a.W + 1); j <= p; ++j)
        visit(a.kv_raw + (static_cast<size_t>(inf.b) * a.raw_cap + (j % a.raw_cap)) * kTcDim);
    float scale = 0.f, lse_v = -INFINITY;
    if (l > 0.f) {
      const float sg = sink_l2[h];
      const float mx = fmaxf(m, sg);
      const float f = exp2f(m - mx);
      scale = __fdiv_rn(f, fmaf(l, f, exp2f(sg - mx)));
      lse_v = (m + log2f(l)) * 0.6931471805599453f;
    }
    const __nv_bfloat162 o01 = __floats2bfloat162_rn(acc[0] * scale, acc[1] * scale);
    const __nv_bfloat162 o23 = __floats2bfloat162_rn(acc[2] * scale, acc[3] * scale);
    uint2 ov;
    ov.x = *reinterpret_cast<const uint32_t*>(&o01);
    ov.y = *reinterpret_cast<const uint32_t*>(&o23);
    *reinterpret_cast<uint2*>(a.out + qrow * kTcDim + 4 * lane) = ov;
    if (a.lse != nullptr && lane == 0) a.lse[qrow] = lse_v;
  }
}

template <int NB>
__global__ void __launch_bounds__(TcCfg<NB>::kThreads, 1) attn_tc_kernel(const TcArgs args, const __grid_constant__ TcMaps maps) {
  using C = TcCfg<NB>;
  constexpr int N = C::N;
  extern __shared__ __align__(1024) uint8_t tc_smem_raw[];
  TcSmem<NB>& sm = *reinterpret_cast<TcSmem<NB>*>(
      (reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kProd0 = C::kSoftWarps;
  constexpr int kMmaWarp = C::kSoftWarps + C::kProdWarps;
  volatile int* abort_flag = &sm.abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&sm.kv_full[s], 32 * C::kProdWarps);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.q_full[s], 1);
      mbar_init(&sm.q_empty[s], 1 + 128 * C::kGroups);
      mbar_init(&sm.o_full[s], 1);
      mbar_init(&sm.o_empty[s], 128 * C::kGroups);
    }
    for (int s = 0; s < C::kSBuf; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.s_free[s], 128 * C::kGroups);
      mbar_init(&sm.p_full[s], 128 * C::kGroups);
      mbar_init(&sm.p_empty[s], 1);
    }
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  for (int h = threadIdx.x; h < 128; h += blockDim.x)
    sm.sink_l2[h] = (args.sink != nullptr && h < args.Hq) ? args.sink[h] * 1.4426950408889634f : -INFINITY;
  if (warp == kMmaWarp) {
    tmem_alloc(&sm.tmem, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem;

  if (warp >= kProd0 && warp < kMmaWarp) {
    // ===================================================================== producer
    const int pw = warp - kProd0;              // producer warp pw: tile rows [RW pw, RW pw + RW)
    constexpr int RW = kTcTile / C::kProdWarps;        // 64 rows per warp
    constexpr int NI = (RW + 31) / 32;                  // 32-row index chunks per warp
    static_assert(RW % 32 == 0, "each producer warp owns whole 32-row index chunks");
    const int cbase = (RW * pw) / 32;                   // first 32-row chunk of this warp's rows
    const uint64_t map_q = reinterpret_cast<uint64_t>(&maps.q);
    const uint64_t map_kv = reinterpret_cast<uint64_t>(&maps.kv);
    const uint64_t map_raw = reinterpret_cast<uint64_t>(&maps.raw);
    int it = 0, kvc = 0;
    for (int u = blockIdx.x; u < args.n_units; u += gridDim.x, ++it) {
      if (*abort_flag) break;
      const int slot = it & 1;
      if (it >= 2 && !tc_wait(&sm.q_empty[slot], ((it >> 1) - 1) & 1, args.status, abort_flag)) break;
      const int b = u / args.units_per_b;
      const int ul = u - b * args.units_per_b;
      const int r0 = (ul / args.hsplit) * args.G;
      const int hoff = (ul % args.hsplit) * args.H;
      const int ntok = min(args.G, args.T_chunk - r0);
      const int p0 = args.q_pos0[b] + args.row0 + r0;
      const int plast = p0 + ntok - 1;
      int n_c;
      const int32_t* irow = args.idx + (static_cast<size_t>(b) * args.T_chunk + r0) * args.k;
      // top-k indices of tile rows 32 (cbase + q) + lane of every entry tile
      // (the chunks holding this warp's rows), loaded up front
      int ir[kTcMaxIdxTiles][NI];
      if (args.sparse) {
        // Valid indices form a prefix (-1 pads the end).  Two round trips: lane
        // l tests the last index of 32-entry chunk l (the number of full chunks
        // f is a ballot count), then the warp counts chunk f.  This warp's own
        // tile rows are loaded alongside the first probe.
        const int Lp = 32 * lane + 31;
        const int vlast = Lp < args.k ? irow[Lp] : -1;
#pragma unroll
        for (int i = 0; i < kTcMaxIdxTiles; ++i)
#pragma unroll
          for (int q = 0; q < NI; ++q) {
            const int L = i * kTcTile + 32 * (cbase + q) + lane;
            ir[i][q] = L < args.k ? irow[L] : -1;
          }
        const int full = __popc(__ballot_sync(0xffffffffu, vlast >= 0));
        const int Lc = 32 * full + lane;
        const int vc = Lc < args.k ? irow[Lc] : -1;
        n_c = 32 * full + __popc(__ballot_sync(0xffffffffu, vc >= 0));
#pragma unroll
        for (int i = 0; i < kTcMaxIdxTiles; ++i)
#pragma unroll
          for (int q = 0; q < NI; ++q) ir[i][q] = ir[i][q] >= 0 ? ir[i][q] : 0;
      } else {
        n_c = min(args.S, (plast + 1) / args.m);
      }
      const int n_cp = (n_c + 3) & ~3;
      int jlo = 0, n_w = 0;
      if (args.W > 0) {
        jlo = max(0, p0 - args.W + 1);
        n_w = plast - jlo + 1;
      }
      const int n_rows = n_cp + n_w;
      const int nt = max(1, (n_rows + kTcTile - 1) / kTcTile);
      const int n_all = args.G > 1 ? min(n_c, (p0 + 1) / args.m) : (n_c == n_cp ? n_rows : n_c);
      if (pw == 0 && lane == 0) {
        sm.info[slot] = TcUnit{b, r0, ntok, n_c, n_w, jlo, p0, nt, hoff, n_all, n_cp};
        // ---- Q: per token one box of H rows (token-major, head-minor) per
        // 64-column half; only the unit's ntok tokens, so no box leaves q
        const int qrow0 = (b * args.Tq + args.row0 + r0) * args.Hq + hoff;
        mbar_arrive_expect_tx(&sm.q_full[slot], ntok * args.H * kTcDim * 2);
        for (int g = 0; g < ntok; ++g) {
          const uint32_t qd = smem_u32(sm.q[slot]) + g * args.H * 128;
          tma_load_2d(qd, map_q, 0, qrow0 + g * args.Hq, &sm.q_full[slot]);
          tma_load_2d(qd + N * 128, map_q, 64, qrow0 + g * args.Hq, &sm.q_full[slot]);
        }
      }
      // ---- KV tiles
      for (int i = 0; i < nt; ++i, ++kvc) {
        const int stage = kvc % C::kStages;
        const int use = kvc / C::kStages;
        if (use >= 1 && !tc_wait(&sm.kv_empty[stage], (use - 1) & 1, args.status, abort_flag)) break;
        if (pw == 0 && lane == 0) CSA_TR(it, i, 0);
        const int L0 = i * kTcTile;
        const uint32_t ks = smem_u32(sm.kv[stage]);
        // contiguous tiles (every row valid and consecutive in one tensor) take two TMA boxes
        const bool dense_entries = !args.sparse && L0 + kTcTile <= n_c;
        const int wj = jlo + (L0 - n_cp);
        const bool window_tile = L0 >= n_cp && L0 + kTcTile <= n_rows && (wj % args.raw_cap) + kTcTile <= args.raw_cap;
        if (dense_entries || window_tile) {
          if (pw == 0 && lane == 0) {
            const uint64_t map = dense_entries ? map_kv : map_raw;
            const int y = dense_entries ? b * args.kv_bstride + L0 : b * args.raw_cap + (wj % args.raw_cap);
            mbar_arrive_expect_tx(&sm.kv_full[stage], kTcTile * kTcDim * 2);
            tma_load_2d(ks, map, 0, y, &sm.kv_full[stage]);
            tma_load_2d(ks + kTcTile * 128, map, 64, y, &sm.kv_full[stage]);
          } else {
            mbar_arrive(&sm.kv_full[stage]);
          }
        } else if (args.sparse && L0 + kTcTile <= n_c) {
          // every row of the tile is a selected entry: lean issue loop (row base
          // pointer hoisted, one shuffle per row pair, swizzle term constant
          // after unrolling: tile row RW pw + 2 j + half has (row & 7) =
          // (2 j & 7) | half because RW pw is a multiple of 32)
          int tr[NI];
#pragma unroll
          for (int q = 0; q < NI; ++q) tr[q] = 0;
#pragma unroll
          for (int ii = 0; ii < kTcMaxIdxTiles; ++ii)
            if (ii == i) {
#pragma unroll
              for (int q = 0; q < NI; ++q) tr[q] = ir[ii][q];
            }
          const int half = lane >> 4, c = lane & 15;
          const __nv_bfloat16* rb = args.kv_c + static_cast<size_t>(b) * args.kv_bstride * kTcDim + c * 8;
          const uint32_t dbase = ks + (c >> 3) * (kTcTile * 128) + (RW * pw + half) * 128;
          const uint32_t cx = static_cast<uint32_t>((c & 7) ^ half);
#pragma unroll
          for (int j = 0; j < RW / 2; ++j) {
            const int s_g = __shfl_sync(0xffffffffu, tr[(2 * j) >> 5], (2 * j + half) & 31);
            const uint32_t dst = dbase + j * 256 + ((cx ^ static_cast<uint32_t>((2 * j) & 7)) << 4);
            cp_async16(dst, rb + static_cast<size_t>(s_g) * kTcDim, 16u);
          }
          cp_async_mbar_arrive(&sm.kv_full[stage]);
        } else if (!args.sparse) {
          // dense tile mixing entries, padding and window rows (or a tile the
          // window wraps in): each instruction moves two 256-byte rows (lanes
          // 0-15 / 16-31); the window's ring slots advance by one per row from
          // the tile's first window row (one modulo per tile, then wrap-arounds)
          const int half = lane >> 4, c = lane & 15;
          const int Lw0 = max(L0, n_cp);
          const int sw0 = n_w > 0 ? (jlo + (Lw0 - n_cp)) % args.raw_cap : 0;
          const __nv_bfloat16* kvb = args.kv_c + static_cast<size_t>(b) * args.kv_bstride * kTcDim + c * 8;
          const __nv_bfloat16* rwb = args.kv_raw + static_cast<size_t>(b) * args.raw_cap * kTcDim + c * 8;
#pragma unroll 8
          for (int j = 0; j < RW / 2; ++j) {
            const int rr = RW * pw + 2 * j + half;         // tile row
            const int L = L0 + rr;
            const __nv_bfloat16* src = kvb;
            uint32_t bytes = 0;
            if (L < n_c) {
              src = kvb + static_cast<size_t>(L) * kTcDim;
              bytes = 16;
            } else if (L >= n_cp && L < n_rows) {
              // the unit's window (W + G - 1 rows for G tokens) may exceed the
              // ring, so the slot can pass raw_cap more than once
              int slot = sw0 + (L - Lw0);
              while (slot >= args.raw_cap) slot -= args.raw_cap;
              src = rwb + static_cast<size_t>(slot) * kTcDim;
              bytes = 16;
            }
            cp_async16(ks + sw128_off(rr, c, kTcTile), src, bytes);
          }
          cp_async_mbar_arrive(&sm.kv_full[stage]);
        } else {
          // sparse tile past the selected entries: each instruction moves two
          // 256-byte rows (lanes 0-15 / 16-31)
          int tr[NI];
#pragma unroll
          for (int q = 0; q < NI; ++q) tr[q] = 0;
#pragma unroll
          for (int ii = 0; ii < kTcMaxIdxTiles; ++ii)
            if (ii == i) {
#pragma unroll
              for (int q = 0; q < NI; ++q) tr[q] = ir[ii][q];
            }
          const int half = lane >> 4, c = lane & 15;
#pragma unroll 8
          for (int j = 0; j < RW / 2; ++j) {
            const int rl = 2 * j + half;                   // row within this warp's RW rows
            const int trow = RW * pw + rl;                  // tile row: chunk trow / 32, lane trow % 32
            int s_g = 0;
#pragma unroll
            for (int q = 0; q < NI; ++q) {
              const int v = __shfl_sync(0xffffffffu, tr[q], trow & 31);
              if ((trow >> 5) - cbase == q) s_g = v;
            }
            const int rr = RW * pw + rl;                   // tile row
            const int L = L0 + rr;
            const __nv_bfloat16* src = args.kv_c;
            uint32_t bytes = 0;
            if (L < n_c) {
              const int s = args.sparse ? s_g : L;
              src = args.kv_c + (static_cast<size_t>(b) * args.kv_bstride + s) * kTcDim + c * 8;
              bytes = 16;
            } else if (L >= n_cp && L < n_rows) {
              const int jj = jlo + (L - n_cp);
              src = args.kv_raw + (static_cast<size_t>(b) * args.raw_cap + (jj % args.raw_cap)) * kTcDim + c * 8;
              bytes = 16;
            }
            cp_async16(ks + sw128_off(rr, c, kTcTile), src, bytes);
          }
          cp_async_mbar_arrive(&sm.kv_full[stage]);
        }
        if (pw == 0 && lane == 0) CSA_TR(it, i, 1);
      }
    }
    cp_async_wait<0>();
  } else if (warp == kMmaWarp) {
    // ===================================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, N, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(128, N, 1, 1);
      int it = 0, kvc = 0, gt = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < args.n_units && ok; u += gridDim.x, ++it) {
        const int slot = it & 1;
        if (!tc_wait(&sm.q_full[slot], (it >> 1) & 1, args.status, abort_flag)) break;
        const int nt = sm.info[slot].nt;
        const int ob = it & 1, ouse = it >> 1;
        const uint32_t qbase = smem_u32(sm.q[slot]);
        auto issue_qk = [&](int i) -> bool {
          const int stage = (kvc + i) % C::kStages;
          if (!tc_wait(&sm.kv_full[stage], ((kvc + i) / C::kStages) & 1, args.status, abort_flag)) return false;
          const int g = gt + i;
          const int sb = g % C::kSBuf, suse = g / C::kSBuf;
          if (suse >= 1 && !tc_wait(&sm.s_free[sb], (suse - 1) & 1, args.status, abort_flag)) return false;
          fence_proxy_async();
          tc_fence_after();
          CSA_TR(it, i, 2);
          const uint32_t kb = smem_u32(sm.kv[stage]);
#pragma unroll
          for (int j = 0; j < kTcDim / 16; ++j)
            mma_bf16(tmem + sb * N, desc_kmajor(kb, kTcTile * 128, j), desc_kmajor(qbase, N * 128, j), idesc_qk,
                     j > 0 ? 1u : 0u);
          tc_commit(&sm.s_full[sb]);
          return true;
        };
        // QK runs kSBuf - 1 tiles ahead: QK(i + kSBuf - 1) is issued before PV(i)
        constexpr int kAhead = C::kSBuf - 1;
        for (int i0 = 0; i0 < kAhead && i0 < nt; ++i0)
          if (!issue_qk(i0)) { ok = false; break; }
        if (!ok) break;
        for (int i = 0; i < nt; ++i) {
          if (i + kAhead < nt && !issue_qk(i + kAhead)) { ok = false; break; }
          const int g = gt + i;
          const int pb = g % C::kSBuf, puse = g / C::kSBuf;
          if (!tc_wait(&sm.p_full[pb], puse & 1, args.status, abort_flag)) { ok = false; break; }
          if (i == 0 && ouse >= 1 && !tc_wait(&sm.o_empty[ob], (ouse - 1) & 1, args.status, abort_flag)) {
            ok = false;
            break;
          }
          fence_proxy_async();
          tc_fence_after();
          CSA_TR(it, i, 3);
          const int stage = (kvc + i) % C::kStages;
          const uint32_t kb = smem_u32(sm.kv[stage]);
          const uint32_t pbase = smem_u32(sm.p[pb]);
#pragma unroll
          for (int j = 0; j < kTcTile / 16; ++j)
            mma_bf16(tmem + C::kOCol + ob * N, desc_mnmajor(kb, kTcTile * 128, j),
                     desc_mnmajor(pbase, kTcTile * 128, j), idesc_pv, (i > 0 || j > 0) ? 1u : 0u);
          tc_commit(&sm.kv_empty[stage]);
          tc_commit(&sm.p_empty[pb]);
        }
        if (!ok) break;
        tc_commit(&sm.o_full[ob]);
        tc_commit(&sm.q_empty[slot]);
        kvc += nt;
        gt += nt;
      }
    }
    __syncwarp();
  } else if (warp < C::kSoftWarps) {
    // ===================================================================== softmax
    constexpr int CW = C::kCW;
    const int wg = warp >> 2, wq = warp & 3;    // warpgroup wg owns columns [CW wg, CW wg + CW)
    const int row = wq * 32 + lane;             // TMEM lane: KV tile row / O^T dim row
    const int bar_id = 1 + wg;
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    const int col0 = CW * wg;
    const float sl2 = args.scale_log2;
    int it = 0, gt = 0;
    // A unit's O^T read-out is deferred until the next unit's first tile is
    // done, so the wait for its last PV overlaps useful work: the group's
    // column scales wait in sm.oscale, and these registers hold the rest.
    bool pend = false;
    int pend_ob = 0;
    uint32_t pend_par = 0, pend_cols = 0;   // o_full parity; columns with a token
    __nv_bfloat16* pend_out = nullptr;      // head dim `row` of the unit's first output row
    auto flush = [&]() -> bool {
      if (!tc_wait(&sm.o_full[pend_ob], pend_par, args.status, abort_flag)) return false;
      tc_fence_after();
      const uint32_t oaddr = tmem + lane_addr + C::kOCol + pend_ob * N + col0;
      uint32_t v[CW];
      tmem_ld16(oaddr, v);
      if constexpr (CW == 32) tmem_ld16(oaddr + 16, v + 16);
      tmem_ld_wait();
      if (threadIdx.x == 0) CSA_TR(it, 14, 2);
      // lane pairs trade half their columns so that each lane holds two
      // adjacent head dims of CW/2 columns: the even lane columns [0, CW/2)
      // at dims (d, d + 1), the odd lane columns [CW/2, CW) at (d - 1, d);
      // then one 4-byte bf16x2 store per column
      constexpr int HC = CW / 2;
      const bool odd = (lane & 1) != 0;
      __nv_bfloat16* pbase = pend_out - (odd ? 1 : 0);
#pragma unroll
      for (int j = 0; j < HC; ++j) {
        const float lo = __uint_as_float(v[j]) * sm.oscale[wg][j];
        const float hi = __uint_as_float(v[HC + j]) * sm.oscale[wg][HC + j];
        const float recv = __shfl_xor_sync(0xffffffffu, odd ? lo : hi, 1);
        const int c = odd ? HC + j : j;
        const uint32_t w = odd ? pack_bf16(recv, hi) : pack_bf16(lo, recv);
        if ((pend_cols >> c) & 1u)
          *reinterpret_cast<uint32_t*>(pbase + static_cast<size_t>(col0 + c) * kTcDim) = w;
      }
      tc_fence_before();
      mbar_arrive(&sm.o_empty[pend_ob]);
      pend = false;
      return true;
    };
    for (int u = blockIdx.x; u < args.n_units; u += gridDim.x, ++it) {
      const int slot = it & 1;
      if (!tc_wait(&sm.q_full[slot], (it >> 1) & 1, args.status, abort_flag)) break;
      const TcUnit inf = sm.info[slot];
      const int n_rows = inf.n_cp + inf.n_w;
      const int ob = it & 1, ouse = it >> 1;
      // this thread's row-sum partials of its CW columns; the running column
      // maxima (the same for every thread of the warpgroup) live in sm.mcol
      float lpart[CW];
      // The running max starts at the head's sink logit: the sink is part of
      // every denominator, so m >= sigma is a valid stabiliser from the first
      // row on, and a unit's first tile needs no exact max unless a logit
      // exceeds its sink by 2^8 (log2 units).  Without a sink, columns start
      // unset and the first valid rows fix their max exactly.
      bool allset = true;    // every column of this warpgroup has a running max
#pragma unroll
      for (int c = 0; c < CW; ++c) {
        const float sg = sm.sink_l2[inf.hoff + ((col0 + c) & (args.H - 1))];
        allset = allset && sg > -INFINITY;
      }
#pragma unroll
      for (int c = 0; c < CW; ++c) lpart[c] = 0.f;
      if (row < CW) {
        const float sg = sm.sink_l2[inf.hoff + ((col0 + row) & (args.H - 1))];
        sm.mcol[wg][row] = sg > -INFINITY ? sg : kNoRowMax;
      }
      named_bar_sync(bar_id, 128);
      bool ok = true;
      bool tainted = false;   // a clamped softmax argument in this thread (rare)
      for (int i = 0; i < inf.nt; ++i, ++gt) {
        const int sb = gt % C::kSBuf;
        if (!tc_wait(&sm.s_full[sb], (gt / C::kSBuf) & 1, args.status, abort_flag)) { ok = false; break; }
        tc_fence_after();
        if (threadIdx.x == 0) CSA_TR(it, i, 4);
        float s[CW];
        {
          uint32_t v[CW];
          tmem_ld16(tmem + lane_addr + sb * N + col0, v);
          if constexpr (CW == 32) tmem_ld16(tmem + lane_addr + sb * N + col0 + 16, v + 16);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < CW; ++c) s[c] = __uint_as_float(v[c]);
        }
        tc_fence_before();
        mbar_arrive(&sm.s_free[sb]);
        if (threadIdx.x == 0 && i < 8) CSA_TR(it, 8 + i, 0);
        // ---- masks (only tiles that reach past the rows every token sees):
        // padding rows, and for multi-token units per-token visibility
        if ((i + 1) * kTcTile > inf.n_all) {
          const int L = i * kTcTile + row;
          if (L >= n_rows || (L >= inf.n_c && L < inf.n_cp)) {
#pragma unroll
            for (int c = 0; c < CW; ++c) s[c] = -INFINITY;
          } else if (args.G > 1) {
            uint32_t vmask = 0;
            for (int g = 0; g < args.G; ++g) {
              const int p = inf.p0 + g;
              bool vis;
              if (L < inf.n_c) {
                vis = args.m * (L + 1) - 1 <= p;
              } else {
                const int j = inf.jlo + (L - inf.n_cp);
                vis = j <= p && j > p - args.W;
              }
              if (vis && g < inf.ntok) vmask |= 1u << g;
            }
#pragma unroll
            for (int c = 0; c < CW; ++c)
              if (!((vmask >> ((col0 + c) >> args.hshift)) & 1u)) s[c] = -INFINITY;
          }
        }
        // ---- d = s * scale_log2 - m in place (m = running column max, kept in
        // registers).  The exact column max of d (warp redux + 4-warp exchange)
        // is taken when some d exceeds 2^8 or a column sees its first valid row
        // (always on a unit's first tile); otherwise one barrier-OR suffices.
        float dmax = -INFINITY;
        bool newrow = false;
        if (allset) {
#pragma unroll
          for (int c = 0; c < CW; c += 2) {
            const float2 m2 = *reinterpret_cast<const float2*>(&sm.mcol[wg][c]);
            ffma2(s[c], s[c + 1], s[c], s[c + 1], sl2, sl2, -m2.x, -m2.y);
            dmax = fmaxf(dmax, fmaxf(s[c], s[c + 1]));
          }
        } else {
#pragma unroll
          for (int c = 0; c < CW; ++c) {
            const float mc = sm.mcol[wg][c];
            const bool sen = mc == kNoRowMax;
            s[c] = fmaf(s[c], sl2, sen ? 0.f : -mc);
            if (sen) newrow |= s[c] > -INFINITY;
            else dmax = fmaxf(dmax, s[c]);
          }
        }
        // ---- P^T = 2^d (bf16) into shared memory (+ per-thread row sums).
        // P buffer gt % kSBuf was last read by PV(gt - kSBuf), which the MMA
        // issued before QK(gt); s_full(gt) completing implies it completed.
        const int pb = gt % C::kSBuf;
        const uint32_t prow = smem_u32(sm.p[pb]) + (col0 >> 6) * (kTcTile * 128) + row * 128;
        auto store_p = [&]() {
#pragma unroll
          for (int c8 = 0; c8 < CW; c8 += 8) {
            float pv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) pv[e] = fast_ex2(s[c8 + e]);
            const uint32_t w0 = pack_bf16(pv[0], pv[1]), w1 = pack_bf16(pv[2], pv[3]);
            const uint32_t w2 = pack_bf16(pv[4], pv[5]), w3 = pack_bf16(pv[6], pv[7]);
            // the row sums add the bf16-rounded weights that PV multiplies, so
            // the normalisation matches the numerator term by term
            fadd2(lpart[c8 + 0], lpart[c8 + 1], bf16_lo(w0), bf16_hi(w0));
            fadd2(lpart[c8 + 2], lpart[c8 + 3], bf16_lo(w1), bf16_hi(w1));
            fadd2(lpart[c8 + 4], lpart[c8 + 5], bf16_lo(w2), bf16_hi(w2));
            fadd2(lpart[c8 + 6], lpart[c8 + 7], bf16_lo(w3), bf16_hi(w3));
            const int chunk = ((col0 & 63) >> 3) + (c8 >> 3);
            const uint32_t addr = prow + ((chunk ^ (row & 7)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w0), "r"(w1), "r"(w2), "r"(w3)
                         : "memory");
          }
        };
        // Once every column has a max (seeded by the sink, or fixed by the
        // first rows), no group-wide decision is taken per tile: arguments
        // stay below 2^64 of the max (bf16 / fp32 hold them exactly enough);
        // a larger one is clamped and the unit is recomputed exactly at its end.
        bool full_max = false;
        if (allset) {
          if (dmax > kClampD) {
            tainted = true;
#pragma unroll
            for (int c = 0; c < CW; ++c) s[c] = fminf(s[c], kClampD);
          }
        } else {
          full_max = bar_red_or(bar_id, 128, dmax > 8.0f || newrow);
        }
        if (threadIdx.x == 0 && i < 8) CSA_TR(it, 8 + i, 1);
        if (full_max) {
#pragma unroll
          for (int c4 = 0; c4 < CW; c4 += 4) {
            const float a0 = redux_max(s[c4]), a1 = redux_max(s[c4 + 1]);
            const float a2 = redux_max(s[c4 + 2]), a3 = redux_max(s[c4 + 3]);
            if (lane == 0) *reinterpret_cast<float4*>(&sm.xch[wg][wq][c4]) = make_float4(a0, a1, a2, a3);
          }
          named_bar_sync(bar_id, 128);
          if (threadIdx.x == 0) CSA_TR(it, i, 6);
          if (row < CW) {
            const int c = row;
            const float x = fmaxf(fmaxf(sm.xch[wg][0][c], sm.xch[wg][1][c]), fmaxf(sm.xch[wg][2][c], sm.xch[wg][3][c]));
            const float mo = sm.mcol[wg][c];
            float mn = mo, a = 1.f, delta = 0.f;
            if (mo == kNoRowMax) {
              if (x > -INFINITY) { mn = x; delta = x; }   // first valid rows: d was s * scale
            } else if (x > 8.0f) {
              mn = mo + x; delta = x; a = exp2f(-x);
            }
            sm.mcol[wg][c] = mn;
            sm.alpha[wg][c] = a;
            sm.dlt[wg][c] = delta;
          }
          named_bar_sync(bar_id, 128);
          if (threadIdx.x == 0) CSA_TR(it, i, 7);
          // every thread reads the same arrays, so these decisions are uniform
          bool rescale = false, any_unset = false;
#pragma unroll
          for (int c4 = 0; c4 < CW; c4 += 4) {
            const float4 m4 = *reinterpret_cast<const float4*>(&sm.mcol[wg][c4]);
            const float4 d4 = *reinterpret_cast<const float4*>(&sm.dlt[wg][c4]);
            const float4 a4 = *reinterpret_cast<const float4*>(&sm.alpha[wg][c4]);
            s[c4] -= d4.x; s[c4 + 1] -= d4.y; s[c4 + 2] -= d4.z; s[c4 + 3] -= d4.w;
            rescale |= (a4.x != 1.f) | (a4.y != 1.f) | (a4.z != 1.f) | (a4.w != 1.f);
            any_unset |= (m4.x == kNoRowMax) | (m4.y == kNoRowMax) | (m4.z == kNoRowMax) | (m4.w == kNoRowMax);
          }
          rescale = rescale && i > 0;
          allset = !any_unset;
          if (rescale) {
            // rare: the running max rose by more than 2^8; PV(i-1) must be complete
            const int gp = gt - 1;
            if (!tc_wait(&sm.p_empty[gp % C::kSBuf], (gp / C::kSBuf) & 1, args.status, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t oaddr = tmem + lane_addr + C::kOCol + ob * N + col0;
#pragma unroll
            for (int h2 = 0; h2 < CW / 16; ++h2) {
              uint32_t v[16];
              tmem_ld16(oaddr + 16 * h2, v);
              tmem_ld_wait();
#pragma unroll
              for (int c = 0; c < 16; ++c)
                v[c] = __float_as_uint(__uint_as_float(v[c]) * sm.alpha[wg][16 * h2 + c]);
              tmem_st16(oaddr + 16 * h2, v);
            }
#pragma unroll
            for (int c = 0; c < CW; ++c) lpart[c] *= sm.alpha[wg][c];
            tmem_st_wait();
            tc_fence_before();
          }
        }
        store_p();
        if (threadIdx.x == 0 && i < 8) CSA_TR(it, 8 + i, 3);
        fence_proxy_async();
        mbar_arrive(&sm.p_full[pb]);
        if (threadIdx.x == 0) CSA_TR(it, i, 5);
        if (i == 0 && pend && !flush()) {
          ok = false;
          break;
        }
      }
      if (!ok) break;
      if (threadIdx.x == 0) CSA_TR(it, 14, 0);
      // the unit's fields are read again here rather than kept in registers
      // through the tile loop (the producer rewrites this slot only after the
      // softmax warps release it below)
      const TcUnit ue = sm.info[slot];
      // ---- unit epilogue: per-column row sums l (butterfly so lane l ends
      // with column l % CW summed over the warp's 32 rows, then the 4 warps
      // through shared memory), output scale 2^(m-M) / (l 2^(m-M) + 2^(sigma-M))
      // with M = max(m, sigma), and lse = (m + log2 l) ln 2 (sink excluded).
      // None of it reads O^T, so it overlaps the unit's last PV.
#pragma unroll
      for (int st = CW / 2; st >= 1; st >>= 1) {
        const bool up = (lane & st) != 0;
#pragma unroll
        for (int e = 0; e < st; ++e) {
          const float send = up ? lpart[e] : lpart[e + st];
          const float keep = up ? lpart[e + st] : lpart[e];
          lpart[e] = keep + __shfl_xor_sync(0xffffffffu, send, st);
        }
      }
#pragma unroll
      for (int o = CW; o < 32; o <<= 1) lpart[0] += __shfl_xor_sync(0xffffffffu, lpart[0], o);
      if (lane < CW) sm.xch[wg][wq][lane] = lpart[0];
      named_bar_sync(bar_id, 128);
      bool redo_local = tainted;
      {
        // lane c (mod CW) of every warp computes column c once; warp 0 keeps
        // the CW scales in sm.oscale for the read-out
        const int c = lane % CW;
        const float l = (sm.xch[wg][0][c] + sm.xch[wg][1][c]) + (sm.xch[wg][2][c] + sm.xch[wg][3][c]);
        float mcl = 0.f;
#pragma unroll
        for (int e = 0; e < CW; ++e)
          if (e == c) mcl = sm.mcol[wg][e];
        const int col = col0 + c;
        const int h = ue.hoff + (col & (args.H - 1));
        const bool tok_ok = (col >> args.hshift) < ue.ntok;
        float scale = 0.f, lse_v = -INFINITY;
        if (mcl > 0.5f * kNoRowMax) {
          // approximate ex2 / rcp / lg2 (relative error ~2^-22) are ample for a
          // bf16 output and an fp32 lse
          const float sg = sm.sink_l2[h];
          const float mx = fmaxf(mcl, sg);
          const float f = fast_ex2(mcl - mx);
          const float den = fmaf(l, f, fast_ex2(sg - mx));
          scale = den > 0.f ? f * fast_rcp(den) : 0.f;
          if (l > 0.f) lse_v = (mcl + fast_lg2(l)) * 0.6931471805599453f;
        }
        // every weight underflowed although the unit has rows: recompute
        if (tok_ok && l == 0.f && ue.n_c + ue.n_w > 0) redo_local = true;
        if (wq == 0 && lane < CW && args.lse != nullptr && tok_ok)
          args.lse[(static_cast<size_t>(ue.b) * args.Tq + args.row0 + ue.r0 + (col >> args.hshift)) * args.Hq + h] =
              lse_v;
        if (wq == 0 && lane < CW) sm.oscale[wg][lane] = scale;
      }
      // group-wide decision; a tainted group recomputes its own columns exactly
      const bool redo = bar_red_or(bar_id, 128, redo_local);
      if (threadIdx.x == 0) CSA_TR(it, 14, 1);
      if (redo) {
        if (!tc_wait(&sm.o_full[ob], ouse & 1, args.status, abort_flag)) break;
        tc_fence_after();
        tc_unit_exact(args, ue, sm.sink_l2, col0, col0 + CW, wq, 4);
        tc_fence_before();
        mbar_arrive(&sm.o_empty[ob]);
      } else {
        pend = true;
        pend_ob = ob;
        pend_par = static_cast<uint32_t>(ouse & 1);
        pend_out = args.out + ((static_cast<size_t>(ue.b) * args.Tq + args.row0 + ue.r0) * args.Hq + ue.hoff) * kTcDim + row;
        uint32_t cols = 0;
#pragma unroll
        for (int c = 0; c < CW; ++c)
          if (((col0 + c) >> args.hshift) < ue.ntok) cols |= 1u << c;
        pend_cols = cols;
      }
      if (threadIdx.x == 0) CSA_TR(it, 15, 7);
      named_bar_sync(bar_id, 128);      // mcol / alpha reused, oscale visible to the group
      mbar_arrive(&sm.q_empty[slot]);
    }
    if (pend) flush();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// 2D bf16 map over [rows, 128] with 128-byte swizzle and a 64 x box_rows box.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kTcDim), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kTcDim) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

template <int NB>
int launch_attn_tc_nb(const TcArgs& a, const TcMaps& maps, cudaStream_t st) {
  const size_t smem = sizeof(TcSmem<NB>) + 1024;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return set_cuda_error(e);
    attr_set = true;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = a.n_units < sms ? a.n_units : sms;
  attn_tc_kernel<NB><<<grid, TcCfg<NB>::kThreads, smem, st>>>(a, maps);
  return check_launch();
}

// bf16 tcgen05 attention.  Requirements: D == 128; every call runs units of
// N = G*H = 64 columns: G = 1 token of 64 heads (128 heads split in two), or
// for dense (HCA) calls with H < 64, G = 64 / H tokens sharing the entries.
int launch_attn_tc(const void* q, const void* kv_c, const int32_t* idx, const void* kv_raw, const float* sink,
                   float tau, int W, int B, int Tq, int row0, int T_chunk, int H, int kv_bstride, int k, int S, int m,
                   int raw_cap, const int32_t* q_pos0, void* out, float* lse, int sparse, cudaStream_t st) {
  int G = 1;
  if (sparse) {
    CSA_REQUIRE(H == 64 || H == 128, CSA_ERR_UNSUPPORTED);
  } else {
    CSA_REQUIRE(H == 16 || H == 32 || H == 64 || H == 128, CSA_ERR_UNSUPPORTED);
    G = H < 64 ? 64 / H : 1;     // units of N = 64 (token, head) columns
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // 128 heads run as two 64-head units of one token each: the N = 64 tile
  // (three S / P buffers, 80 registers without spilling its softmax loop) beats
  // the N = 128 tile even though each KV tile is fetched twice (from L2)
  const int Hq = H;
  const int hsplit = H == 128 ? 2 : 1;
  if (hsplit == 2) G = 1;
  H = Hq / hsplit;
  const int N = G * H;
  TcArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.kv_c = static_cast<const __nv_bfloat16*>(kv_c);
  a.idx = idx;
  a.kv_raw = static_cast<const __nv_bfloat16*>(kv_raw);
  a.sink = sink;
  a.q_pos0 = q_pos0;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.status = device_status_ptr();
  CSA_REQUIRE(a.status != nullptr, CSA_ERR_CUDA);
  a.scale_log2 = tau * 1.4426950408889634f;
  a.W = W; a.Tq = Tq; a.row0 = row0; a.T_chunk = T_chunk; a.H = H; a.kv_bstride = kv_bstride; a.k = k;
  a.S = S; a.m = m; a.raw_cap = raw_cap > 0 ? raw_cap : 1;
  a.G = G;
  a.hshift = 31 - __builtin_clz(static_cast<unsigned>(H));
  a.sparse = sparse;
  a.Hq = Hq;
  a.hsplit = hsplit;
  a.units_per_b = (T_chunk + G - 1) / G * hsplit;
  const long long nu = static_cast<long long>(B) * a.units_per_b;
  CSA_REQUIRE(nu < (1ll << 31), CSA_ERR_UNSUPPORTED);
  a.n_units = static_cast<int>(nu);
  if (a.n_units == 0) return CSA_OK;
  if (sparse) CSA_REQUIRE(k <= kTcMaxIdxTiles * kTcTile, CSA_ERR_UNSUPPORTED);
  const long long q_rows = static_cast<long long>(B) * Tq * Hq;
  const long long kv_rows = static_cast<long long>(B) * kv_bstride;
  const long long raw_rows = static_cast<long long>(B) * a.raw_cap;
  CSA_REQUIRE(q_rows < (1ll << 31) && kv_rows < (1ll << 31) - 1 && raw_rows < (1ll << 31) - 1, CSA_ERR_UNSUPPORTED);
  a.kv_rows = static_cast<int>(kv_rows);
  a.raw_rows = static_cast<int>(raw_rows);
  TcMaps maps;
  if (!make_map(&maps.q, q, static_cast<uint64_t>(q_rows), static_cast<uint32_t>(H)) ||
      !make_map(&maps.kv, kv_c, static_cast<uint64_t>(kv_rows), kTcTile) ||
      !make_map(&maps.raw, kv_raw ? kv_raw : kv_c, static_cast<uint64_t>(kv_raw ? raw_rows : kv_rows), kTcTile))
    return CSA_ERR_CUDA;
  if (!kv_raw) a.raw_rows = a.kv_rows;
  CSA_REQUIRE(N == 64, CSA_ERR_UNSUPPORTED);
  return launch_attn_tc_nb<1>(a, maps, st);
}

}  // namespace csa
