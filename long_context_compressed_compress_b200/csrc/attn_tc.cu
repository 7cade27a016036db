// bf16 attention on tcgen05 with TMEM accumulators: CSA sparse attention over
// the top-k entries (cf-1.com/news/5231315 §3.1), HCA dense attention over all
// visible entries (§3.2), both with the 128-token raw window and the sink in
// the softmax denominator (§3.3).  MQA: one K = V row serves every head (§3.4).
//
// Orientation.  A work unit is 128 query rows = (tokens x heads) that share
// one list of KV rows, and each thread of a softmax warpgroup owns one query
// row (its TMEM lane), so the softmax needs no cross-thread reduction:
//   S [128 q-rows x 128 KV rows] = Q . KV^T      (A = Q, smem; B = KV tile)
//   O [128 q-rows x 128 dims]   += P . V         (A = P, TMEM; B = the same
//                                                 KV tile read MN-major)
// P is written as bf16 pairs over the first 64 columns of its S buffer, so the
// PV MMA takes its A operand straight from TMEM.
//
// Units.  With H = 128 a unit is one token's 128 heads; dense (HCA) calls with
// H = 64 / 32 / 16 put 2 / 4 / 8 tokens of a block in a unit, which share the
// entries (their windows are masked per row).  Sparse calls with H = 64 put
// two tokens in a unit whose top-k sets differ: each KV tile then holds 64
// rows of each token's list ("split" units), and every query row only uses
// its own token's half of the tile (the other half's P is zero).
//
// Roles (one CTA per SM, persistent over units; 16 warps):
//   softmax warpgroups 0 and 1 (warps 0-7): tile g of the CTA's tile sequence
//     goes to warpgroup g % 2 and S/P buffer g % 2, so one warpgroup's softmax
//     overlaps the other's tile on the tensor pipe;
//   producer warps (8, 9): Q by 2D TMA; KV rows gathered with cp.async into
//     128-byte-swizzled tiles (TMA boxes for contiguous dense / window tiles);
//     warp w fills tile rows [64 w, 64 w + 64);
//   MMA warp (10): QK(g) is issued before PV(g - 1), so QK runs one tile ahead;
//   epilogue warpgroup (warps 11-14): row sums from both softmax warpgroups,
//     output scale and lse, O read-out from TMEM (O is double-buffered), bf16
//     stores; rows whose fast path was inexact are recomputed exactly.
// Softmax stabiliser: the running max of a row is fixed for the whole unit:
// the head's sink logit, or without a sink the max of the row's first tile.
// Arguments then stay below 2^64 for any sane input; a row whose weights leave
// that range (row sum above 2^64, or every weight underflowing) is recomputed
// on CUDA cores in fp32 with an online softmax.
// All waits are bounded in time (a runtime limit); a wait that gives up
// records CSA_ERR_TIMEOUT in the caller's status word and sets an abort flag
// every role polls, so the kernel always returns; waits that guard warp-wide
// (.sync.aligned) instructions are made warp-uniform.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace csa {

namespace fa {

constexpr int kTile = 128;                  // KV rows per tile (MMA N of QK, K of PV)
constexpr int kDim = 128;                   // head dim
constexpr int kStages = 4;                  // KV tile ring
constexpr int kTileBytes = 128 * kDim * 2;  // a Q tile or a KV tile: 32 KB
constexpr int kRegion = 128 * 128;          // one 64-column half of a tile (16 KB)
// warps: softmax warpgroups 0-3 and 4-7, epilogue warpgroup 8-11, producers
// 12-13, MMA 14, scheduler 15
constexpr int kSoftWarps = 8, kEpi0 = 8, kProd0 = 12, kProdWarps = 2, kMmaWarp = 14, kSchedWarp = 15;
constexpr int kThreads = 32 * 16;
constexpr uint32_t kTmemCols = 512;
constexpr int kSBuf = 3;                    // S/P buffers: QK runs two tiles ahead of PV
constexpr uint32_t kColS = 0;               // S/P buffer j at column 128 j
constexpr uint32_t kColO = 384;             // O accumulator
constexpr int kInfo = 4;                    // ring of unit descriptors / row-sum slots
constexpr int kMaxTopk = 1024;
constexpr uint64_t kDrainNs = 1000000ull;   // exit-time wait for in-flight copies / MMAs

struct Unit {
  int b, r0, ntok, nt, p0;
  int n_c[2], jlo[2], n_w[2];   // shared units use index 0; split units one per token
};

struct __align__(1024) Smem {
  uint8_t q[2][kTileBytes];
  uint8_t kv[kStages][kTileBytes];
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[kSBuf], p_full[kSBuf];
  uint64_t o_full, o_empty;
  uint64_t info_ready[kInfo], info_free[kInfo], l_ready[kInfo], m_ready[kInfo];
  uint64_t drain;
  float lsum[kInfo][2][128];
  float mrow[kInfo][128];
  float sink_l2[128];
  Unit info[kInfo];
  uint32_t tmem;
  int abort_flag;
};

struct Args {
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
  int sparse, split;
  int upb;               // units per sequence
  int n_units;
  int has_sink;
  unsigned long long wait_ns;
  unsigned hint_ns;
};

struct Maps {
  CUtensorMap q;     // [B*Tq*H, 128] bf16, box 64 x H (one token)
  CUtensorMap kv;    // [B*kv_bstride, 128] bf16, box 64 x 64 (one producer warp's rows)
  CUtensorMap raw;   // [B*raw_cap, 128] bf16, box 64 x 64
};

// ------------------------------------------------------------------ waits
__device__ __forceinline__ bool try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint)
      : "memory");
  return ok != 0;
}
// Time-bounded wait of one thread: false when another role has aborted, or
// (recording the site) after the call's limit.
__device__ __noinline__ bool wait1(uint64_t* bar, uint32_t parity, const Args& a, volatile int* abort_flag,
                                   int site) {
  if (try_wait_hint(bar, parity, a.hint_ns)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (try_wait_hint(bar, parity, a.hint_ns)) return true;
    if (*abort_flag) return false;
    if (global_ns() - t0 > a.wait_ns) break;
  }
  atomicCAS(a.status, 0, CSA_ERR_TIMEOUT | (site << 8));
  *abort_flag = 1;
  return false;
}
// Warp-uniform wait: every lane gets the same answer (a lane that timed out
// makes the whole warp leave), so the warp-wide instructions after it run
// with all lanes or none.
__device__ __forceinline__ bool waitw(uint64_t* bar, uint32_t parity, const Args& a, volatile int* abort_flag,
                                      int site) {
  const bool ok = wait1(bar, parity, a, abort_flag, site);
  return __all_sync(0xffffffffu, ok);
}
// Non-blocking probe of a phase.
__device__ __forceinline__ bool test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Exit-time wait with a fixed short limit that ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!try_wait_hint(bar, parity, 1000u))
    if (global_ns() - t0 > kDrainNs) break;
}

// ------------------------------------------------------------ PTX helpers
__device__ __forceinline__ float ex2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float rcp(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float lg2(float x) {
  float r;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
// (d0, d1) = (a0, a1) * (b0, b1) + (c0, c1) on the packed f32x2 pipe
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
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

#define FA_TMEM_LD_X32(taddr, r)                                                                          \
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "                                                 \
               "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"                                  \
               "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"                 \
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),      \
                 "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),  \
                 "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),            \
                 "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),            \
                 "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])             \
               : "r"(taddr))

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t r[32]) { FA_TMEM_LD_X32(taddr, r); }
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t r[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem], kind::f16 (bf16 via idesc), fp32 accumulate.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Descriptor of a K-major SW128 operand (rows of 128 B, 8-row atoms 1024 B):
// K-step j (16 bf16) of a [128 x 128] bf16 tile lives in region j/4 at byte j%4*32.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t base, int j) {
  return make_sdesc(base + (j >> 2) * kRegion + (j & 3) * 32, 16, 1024, kLayoutSw128);
}
// Descriptor of the same tile read MN-major (K = tile rows, MN = dims; the two
// 64-dim halves kRegion apart): K-step j = rows 16j..16j+15.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t base, int j) {
  return make_sdesc(base + j * 2048, kRegion, 1024, kLayoutSw128);
}
// byte offset of 16-byte chunk c (0..15) of row r in a two-region SW128 tile
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
  return (c >> 3) * kRegion + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

// Number of valid (non-negative) indices in a top-k row (they form a prefix):
// lane l tests the last index of 32-entry chunk l, then the warp counts the
// first partial chunk.
__device__ __forceinline__ int count_valid(const int32_t* irow, int k, int lane) {
  const int Lp = 32 * lane + 31;
  const int vlast = Lp < k ? irow[Lp] : -1;
  const int full = __popc(__ballot_sync(0xffffffffu, vlast >= 0));
  const int Lc = 32 * full + lane;
  const int vc = (full < 32 && Lc < k) ? irow[Lc] : -1;
  return 32 * full + __popc(__ballot_sync(0xffffffffu, vc >= 0));
}

// Unit descriptor (computed identically by every producer lane).
__device__ __forceinline__ Unit make_unit(const Args& a, int u, int lane) {
  Unit un;
  un.b = u / a.upb;
  un.r0 = (u - un.b * a.upb) * a.G;
  un.ntok = min(a.G, a.T_chunk - un.r0);
  un.p0 = a.q_pos0[un.b] + a.row0 + un.r0;
  const int plast = un.p0 + un.ntok - 1;
  if (a.split) {
    int nmax = 0;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      int nc = 0, jl = 0, nw = 0;
      if (g < un.ntok) {
        const int32_t* irow = a.idx + (static_cast<size_t>(un.b) * a.T_chunk + un.r0 + g) * a.k;
        nc = count_valid(irow, a.k, lane);
        if (a.W > 0) {
          const int p = un.p0 + g;
          jl = max(0, p - a.W + 1);
          nw = p - jl + 1;
        }
      }
      un.n_c[g] = nc; un.jlo[g] = jl; un.n_w[g] = nw;
      nmax = max(nmax, nc + nw);
    }
    un.nt = max(1, (nmax + 63) / 64);
  } else {
    int nc;
    if (a.sparse) {
      const int32_t* irow = a.idx + (static_cast<size_t>(un.b) * a.T_chunk + un.r0) * a.k;
      nc = count_valid(irow, a.k, lane);
    } else {
      nc = min(a.S, (plast + 1) / a.m);
    }
    int jl = 0, nw = 0;
    if (a.W > 0) {
      jl = max(0, un.p0 - a.W + 1);
      nw = plast - jl + 1;
    }
    un.n_c[0] = nc; un.jlo[0] = jl; un.n_w[0] = nw;
    un.n_c[1] = 0; un.jlo[1] = 0; un.n_w[1] = 0;
    un.nt = max(1, (nc + nw + kTile - 1) / kTile);
  }
  return un;
}

// Valid list rows of query row (token g) of a unit, as two ranges [0, a1) and
// [b0, b1) in list coordinates.
struct RowRange {
  int a1, b0, b1;
};
__device__ __forceinline__ RowRange row_range(const Args& a, const Unit& un, int g) {
  RowRange rr{0, 0, 0};
  if (g >= un.ntok) return rr;
  if (a.split) {
    rr.a1 = g == 0 ? un.n_c[0] + un.n_w[0] : un.n_c[1] + un.n_w[1];
    return rr;
  }
  const int p = un.p0 + g;
  const int nc = un.n_c[0];
  rr.a1 = a.sparse ? nc : min(nc, min(a.S, (p + 1) / a.m));
  if (a.W > 0) {
    rr.b0 = nc + max(0, p - a.W + 1 - un.jlo[0]);
    rr.b1 = nc + (p - un.jlo[0] + 1);
  } else {
    rr.b0 = rr.b1 = nc;
  }
  return rr;
}

// Exact recomputation of one query row on CUDA cores (a warp; lane = 4 dims):
// an online softmax in fp32 over the row's entries and window rows, then the
// sink, as the definition states.  For rows whose fast path left its range.
__device__ __noinline__ void row_exact(const Args& a, const Unit& un, int g, int h, const float* sink_l2) {
  const int lane = threadIdx.x & 31;
  const int p = un.p0 + g;
  const size_t qrow = (static_cast<size_t>(un.b) * a.Tq + a.row0 + un.r0 + g) * a.H + h;
  float qv[4];
  {
    const uint2 u = *reinterpret_cast<const uint2*>(a.q + qrow * kDim + 4 * lane);
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
    const int32_t* ir = a.idx + (static_cast<size_t>(un.b) * a.T_chunk + un.r0 + g) * a.k;
    for (int j = 0; j < a.k; ++j) {
      const int s = ir[j];
      if (s < 0) break;
      visit(a.kv_c + (static_cast<size_t>(un.b) * a.kv_bstride + s) * kDim);
    }
  } else {
    const int nv = min(a.S, (p + 1) / a.m);
    for (int e = 0; e < nv; ++e) visit(a.kv_c + (static_cast<size_t>(un.b) * a.kv_bstride + e) * kDim);
  }
  if (a.W > 0)
    for (int j = max(0, p - a.W + 1); j <= p; ++j)
      visit(a.kv_raw + (static_cast<size_t>(un.b) * a.raw_cap + (j % a.raw_cap)) * kDim);
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
  *reinterpret_cast<uint2*>(a.out + qrow * kDim + 4 * lane) = ov;
  if (a.lse != nullptr && lane == 0) a.lse[qrow] = lse_v;
}

// Softmax of one 32-column chunk of S (values v) into 16 bf16x2 words of P:
// p = 2^(s * scale_log2 - M), columns outside [0, ua) u [ub0, ub1) give 0
// (tile-local coordinates; `full` skips the masks).  The row sum adds the
// bf16-rounded weights into four independent partial sums (lsum[0..3]).
__device__ __forceinline__ void softmax_chunk(const uint32_t v[32], uint32_t w[16], float sl2, float negM,
                                              bool full, int c0, int ua, int ub0, int ub1, float lsum[4]) {
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    float p0 = ex2(fmaf(__uint_as_float(v[e]), sl2, negM));
    float p1 = ex2(fmaf(__uint_as_float(v[e + 1]), sl2, negM));
    if (!full) {
      const int c = c0 + e;
      const bool ok0 = c < ua || (c >= ub0 && c < ub1);
      const bool ok1 = c + 1 < ua || (c + 1 >= ub0 && c + 1 < ub1);
      p0 = ok0 ? p0 : 0.f;
      p1 = ok1 ? p1 : 0.f;
    }
    const uint32_t pk = pack_bf16(p0, p1);
    w[e >> 1] = pk;
    // the bf16-rounded weights that PV multiplies, so numerator and
    // denominator see the same rounding
    lsum[(e >> 1) & 3] += bf16_lo(pk) + bf16_hi(pk);
  }
}

__global__ void __launch_bounds__(kThreads, 1) attn_fa_kernel(const __grid_constant__ Args args,
                                                               const __grid_constant__ Maps maps) {
  extern __shared__ __align__(1024) uint8_t fa_smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(fa_smem_raw) + 1023) &
                                      ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;
  const Args& a = args;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 32 * kProdWarps);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.q_full[s], 1);
      mbar_init(&sm.q_empty[s], 1);
    }
    for (int s = 0; s < kSBuf; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], 128);
    }
    mbar_init(&sm.o_full, 1);
    mbar_init(&sm.o_empty, 128);
    for (int s = 0; s < kInfo; ++s) {
      mbar_init(&sm.info_ready[s], 1);
      mbar_init(&sm.info_free[s], 128);
      mbar_init(&sm.l_ready[s], 256);
      mbar_init(&sm.m_ready[s], 128);
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  for (int h = threadIdx.x; h < 128; h += blockDim.x)
    sm.sink_l2[h] = (a.sink != nullptr && h < a.H) ? a.sink[h] * 1.4426950408889634f : -INFINITY;
  if (warp == kMmaWarp) {
    tmem_alloc(&sm.tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem;
  const int Hu = 1 << a.hshift;   // heads per token
  if (warp == kSchedWarp) {
    // ===================================================================== scheduler
    // Unit descriptors (their top-k counts need dependent index loads) and Q
    // tiles, computed ahead of the producers so neither sits on their path.
    int it = 0, q_it = -1;
    for (int u = blockIdx.x; u < a.n_units; u += gridDim.x, ++it) {
      if (*abort_flag) break;
      const int slot = it & (kInfo - 1), qs = it & 1;
      if (it >= kInfo && !waitw(&sm.info_free[slot], ((it / kInfo) - 1) & 1, a, abort_flag, 1)) break;
      const Unit un = make_unit(a, u, lane);
      if (lane == 0) {
        sm.info[slot] = un;
        mbar_arrive(&sm.info_ready[slot]);
      }
      if (it >= 2 && !waitw(&sm.q_empty[qs], ((it >> 1) - 1) & 1, a, abort_flag, 2)) break;
      if (lane == 0) {
        q_it = it;
        const int qrow0 = (un.b * a.Tq + a.row0 + un.r0) * a.H;
        mbar_arrive_expect_tx(&sm.q_full[qs], un.ntok * Hu * kDim * 2);
        for (int g = 0; g < un.ntok; ++g) {
          const uint32_t qd = smem_u32(sm.q[qs]) + g * Hu * 128;
          tma_load_2d(qd, reinterpret_cast<uint64_t>(&maps.q), 0, qrow0 + g * a.H, &sm.q_full[qs]);
          tma_load_2d(qd + kRegion, reinterpret_cast<uint64_t>(&maps.q), 64, qrow0 + g * a.H, &sm.q_full[qs]);
        }
      }
    }
    if (*abort_flag && lane == 0 && q_it >= 0) drain_wait(&sm.q_full[q_it & 1], (q_it >> 1) & 1);
  } else if (warp >= kProd0 && warp < kProd0 + kProdWarps) {
    // ===================================================================== producers
    const int pw = warp - kProd0;
    const uint64_t map_kv = reinterpret_cast<uint64_t>(&maps.kv);
    const uint64_t map_raw = reinterpret_cast<uint64_t>(&maps.raw);
    const int half = lane >> 4, c = lane & 15;
    int it = 0, kvc = 0;
    int armed_use[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) armed_use[s] = -1;
    bool ok = true;
    for (int u = blockIdx.x; u < a.n_units && ok; u += gridDim.x, ++it) {
      const int slot = it & (kInfo - 1);
      if (!waitw(&sm.info_ready[slot], (it / kInfo) & 1, a, abort_flag, 3)) break;
      const Unit un = sm.info[slot];
      // this warp's list: its own token's (split units) or the unit's
      const int tg = a.split ? pw : 0;
      const int nc = tg == 0 ? un.n_c[0] : un.n_c[1];
      const int jlo = tg == 0 ? un.jlo[0] : un.jlo[1];
      const int nw = tg == 0 ? un.n_w[0] : un.n_w[1];
      const int nrows = (a.split && tg >= un.ntok) ? 0 : nc + nw;
      const int32_t* irow =
          a.sparse ? a.idx + (static_cast<size_t>(un.b) * a.T_chunk + un.r0 + (tg < un.ntok ? tg : 0)) * a.k
                   : nullptr;
      const __nv_bfloat16* kvb = a.kv_c + static_cast<size_t>(un.b) * a.kv_bstride * kDim + c * 8;
      const __nv_bfloat16* rwb = a.kv_raw + static_cast<size_t>(un.b) * a.raw_cap * kDim + c * 8;
      // list offset of this warp's 64 rows in tile i: 64 i (split) or 128 i + 64 pw
      const int lstep = a.split ? 64 : 128;
      const int loff = a.split ? 0 : 64 * pw;
      // top-k indices of this warp's rows of the next tile (two per lane), prefetched
      int ir0 = 0, ir1 = 0;
      auto load_idx = [&](int i) {
        const int L = lstep * i + loff + lane;
        ir0 = (a.sparse && L < nc) ? irow[L] : 0;
        ir1 = (a.sparse && L + 32 < nc) ? irow[L + 32] : 0;
      };
      load_idx(0);
      for (int i = 0; i < un.nt; ++i, ++kvc) {
        const int stage = kvc % kStages;
        const int use = kvc / kStages;
        if (use >= 1 && !waitw(&sm.kv_empty[stage], (use - 1) & 1, a, abort_flag, 4)) { ok = false; break; }
        const int t0 = ir0, t1 = ir1;
        if (i + 1 < un.nt) load_idx(i + 1);
        const uint32_t ks = smem_u32(sm.kv[stage]);
        const int L0 = lstep * i + loff;           // list row of this warp's first tile row
        const int R0 = 64 * pw;                    // its first tile row
        // destination of row pair j (rows R0 + 2 j + half): tile row & 7 is
        // (2 j & 7) | half since R0 is a multiple of 8
        const uint32_t dbase = ks + (c >> 3) * kRegion + (R0 + half) * 128;
        const uint32_t cx = static_cast<uint32_t>((c & 7) ^ half);
        // contiguous 64-row chunks (dense entries, or window rows whose ring
        // slots do not wrap) come by TMA: two 64 x 64 boxes, one per dim half
        const bool dense_chunk = !a.sparse && L0 + 64 <= nc;
        int wslot = 0;
        bool win_chunk = false;
        if (!dense_chunk && L0 >= nc && L0 + 64 <= nrows) {
          wslot = (jlo + (L0 - nc)) % a.raw_cap;
          win_chunk = wslot + 64 <= a.raw_cap;
        }
        if (dense_chunk || win_chunk) {
          if (lane == 0) {
            const uint64_t map = dense_chunk ? map_kv : map_raw;
            const int y = dense_chunk ? un.b * a.kv_bstride + L0 : un.b * a.raw_cap + wslot;
            mbar_arrive_expect_tx(&sm.kv_full[stage], 64 * kDim * 2);
            tma_load_2d(ks + R0 * 128, map, 0, y, &sm.kv_full[stage]);
            tma_load_2d(ks + kRegion + R0 * 128, map, 64, y, &sm.kv_full[stage]);
#pragma unroll
            for (int s2 = 0; s2 < kStages; ++s2)
              if (s2 == stage) armed_use[s2] = use;
          } else {
            mbar_arrive(&sm.kv_full[stage]);
          }
        } else if (a.sparse && L0 + 64 <= nc) {
          // every row is a selected entry: row base hoisted, one shuffle per
          // row pair, swizzle term constant after unrolling
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int s_g = __shfl_sync(0xffffffffu, j < 16 ? t0 : t1, (2 * j + half) & 31);
            const uint32_t dst = dbase + j * 256 + ((cx ^ static_cast<uint32_t>((2 * j) & 7)) << 4);
            cp_async16(dst, kvb + static_cast<size_t>(s_g) * kDim, 16u);
          }
          cp_async_mbar_arrive(&sm.kv_full[stage]);
        } else if (L0 >= nc && L0 + 64 <= nrows) {
          // every row is a window row: consecutive ring slots (at most one wrap,
          // since the 64 rows span less than raw_cap >= W positions... or wrap
          // again for rings shorter than 64; handled by the loop below)
          int slot = (jlo + (L0 - nc) + half) % a.raw_cap;
#pragma unroll 8
          for (int j = 0; j < 32; ++j) {
            const uint32_t dst = dbase + j * 256 + ((cx ^ static_cast<uint32_t>((2 * j) & 7)) << 4);
            cp_async16(dst, rwb + static_cast<size_t>(slot) * kDim, 16u);
            slot += 2;
            while (slot >= a.raw_cap) slot -= a.raw_cap;
          }
          cp_async_mbar_arrive(&sm.kv_full[stage]);
        } else {
          // mixed rows: entries, window rows, zero padding
          const int Lw0 = max(L0, nc);
          int sw0 = 0;
          if (nw > 0 && Lw0 < nc + nw) sw0 = (jlo + (Lw0 - nc)) % a.raw_cap;
#pragma unroll 4
          for (int j = 0; j < 32; ++j) {
            const int rl = 2 * j + half;
            const int L = L0 + rl;
            const int s_g = __shfl_sync(0xffffffffu, j < 16 ? t0 : t1, rl & 31);
            const __nv_bfloat16* src = kvb;
            uint32_t bytes = 0;
            if (L < nc) {
              src = kvb + static_cast<size_t>(a.sparse ? s_g : L) * kDim;
              bytes = 16;
            } else if (L < nrows) {
              int slot = sw0 + (L - Lw0);
              while (slot >= a.raw_cap) slot -= a.raw_cap;
              src = rwb + static_cast<size_t>(slot) * kDim;
              bytes = 16;
            }
            const uint32_t dst = dbase + j * 256 + ((cx ^ static_cast<uint32_t>((2 * j) & 7)) << 4);
            cp_async16(dst, src, bytes);
          }
          cp_async_mbar_arrive(&sm.kv_full[stage]);
        }
      }
    }
    cp_async_wait<0>();
    if (*abort_flag && lane == 0) {
      // TMA boxes still in flight land within microseconds; wait for them
#pragma unroll
      for (int s = 0; s < kStages; ++s)
        if (armed_use[s] >= 0) drain_wait(&sm.kv_full[s], armed_use[s] & 1);
    }
  } else if (warp == kMmaWarp) {
    // ===================================================================== MMA issuer
    // Global tile g of this CTA: S/P buffer g % 3, KV stage g % kStages.  QK(g)
    // may be issued once PV(g - 3) has been issued (the tensor pipe executes in
    // issue order, so the S buffer's P is consumed first): QK runs up to two
    // tiles ahead of the PV that waits for the softmax.
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(128, 128, 0, 1);
      // QK cursor: unit qu (local index qit), tile qi, global tile qg
      int qu = blockIdx.x, qit = 0, qi = 0, qg = 0, q_nt = -1;
      // PV cursor: unit pit, tile pi, global tile pg
      int pu = blockIdx.x, pit = 0, pi = 0, pg = 0, p_nt = 0;
      // Whichever of the next PV and the next QK is ready goes first (PV
      // preferred: it frees a KV stage and an S buffer); nothing blocks on one
      // while the other could run.  The wait limit counts from the last issue.
      uint64_t t_last = global_ns();
      while (pu < a.n_units) {
        bool did = false;
        if (pg < qg) {
          if (pi == 0) p_nt = sm.info[pit & (kInfo - 1)].nt;   // its QK(0) was issued: info is ready
          const int sb = pg % kSBuf;
          if (test_wait(&sm.p_full[sb], (pg / kSBuf) & 1) &&
              (pi != 0 || pit == 0 || test_wait(&sm.o_empty, (pit - 1) & 1))) {
            tc_fence_after();
            const uint32_t kb = smem_u32(sm.kv[pg % kStages]);
            const uint32_t pcol = tmem + kColS + 128 * sb;
#pragma unroll
            for (int j = 0; j < kTile / 16; ++j)
              mma_bf16_ts(tmem + kColO, pcol + 8 * j, desc_mnmajor(kb, j), idesc_pv,
                          (pi == 0 && j == 0) ? 0u : 1u);
            tc_commit(&sm.kv_empty[pg % kStages]);
            ++pg;
            if (++pi == p_nt) {
              tc_commit(&sm.o_full);
              pi = 0;
              ++pit;
              pu += gridDim.x;
            }
            did = true;
          }
        }
        if (!did && qu < a.n_units && qg < pg + kSBuf) {
          if (q_nt < 0 && test_wait(&sm.q_full[qit & 1], (qit >> 1) & 1))
            q_nt = sm.info[qit & (kInfo - 1)].nt;
          const int st = qg % kStages;
          if (q_nt >= 0 && test_wait(&sm.kv_full[st], (qg / kStages) & 1)) {
            fence_proxy_async();
            tc_fence_after();
            const uint32_t qbase = smem_u32(sm.q[qit & 1]);
            const uint32_t kb = smem_u32(sm.kv[st]);
            const int sb = qg % kSBuf;
#pragma unroll
            for (int j = 0; j < kDim / 16; ++j)
              mma_bf16(tmem + kColS + 128 * sb, desc_kmajor(qbase, j), desc_kmajor(kb, j), idesc_qk,
                       j > 0 ? 1u : 0u);
            tc_commit(&sm.s_full[sb]);
            ++qg;
            if (++qi == q_nt) {
              tc_commit(&sm.q_empty[qit & 1]);   // the unit's Q tile is no longer read
              qi = 0;
              q_nt = -1;
              ++qit;
              qu += gridDim.x;
            }
            did = true;
          }
        }
        if (did) {
          t_last = global_ns();
        } else {
          if (*abort_flag) break;
          __nanosleep(32);
          if (global_ns() - t_last > a.wait_ns) {
            atomicCAS(a.status, 0, CSA_ERR_TIMEOUT | (14 << 8));
            *abort_flag = 1;
            break;
          }
        }
      }
      if (*abort_flag) {
        // let every MMA this thread issued finish before TMEM is released
        tc_commit(&sm.drain);
        drain_wait(&sm.drain, 0);
      }
    }
    __syncwarp();
  } else if (warp < kSoftWarps) {
    // ===================================================================== softmax
    const int wg = warp >> 2;                    // warpgroup: tiles g with g % 2 == wg
    const int r = (warp & 3) * 32 + lane;        // query row = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float sl2 = a.scale_log2;
    const int g_tok = r >> a.hshift;
    const int h = r & (Hu - 1);
    const int half_c = a.split ? 64 * g_tok : 0;   // this row's S columns (split units)
    const int ncols = a.split ? 64 : 128;
    int it = 0, gt0 = 0;
    for (int u = blockIdx.x; u < a.n_units; u += gridDim.x, ++it) {
      const int slot = it & (kInfo - 1);
      if (!waitw(&sm.info_ready[slot], (it / kInfo) & 1, a, abort_flag, 9)) break;
      const Unit un = sm.info[slot];
      const RowRange rr = row_range(a, un, g_tok);
      float M = sm.sink_l2[h];
      const int i_first = (gt0 & 1) == wg ? 0 : 1;
      bool ok = true;
      if (!a.has_sink && i_first == 1 && un.nt > 1) {
        if (!waitw(&sm.m_ready[slot], (it / kInfo) & 1, a, abort_flag, 10)) break;
        M = sm.mrow[slot][r];
      }
      float lacc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int i = i_first; i < un.nt; i += 2) {
        const int g = gt0 + i;
        const int sb = g % kSBuf;
        const uint32_t scol = tmem + lane_addr + kColS + 128 * sb;
        if (!waitw(&sm.s_full[sb], (g / kSBuf) & 1, a, abort_flag, 11)) { ok = false; break; }
        tc_fence_after();
        const int base = ncols * i;
        const int ua = min(max(rr.a1 - base, 0), ncols);
        const int ub0 = min(max(rr.b0 - base, 0), ncols);
        const int ub1 = min(max(rr.b1 - base, 0), ncols);
        const bool full = ua == ncols || (ub0 <= ua && ub1 == ncols);
        // all-masked tile for every row of the warp (warp-uniform: the TMEM
        // stores below are warp-wide instructions)
        const bool none = __all_sync(0xffffffffu, ua == 0 && ub1 <= ub0);
        if (i == 0 && !a.has_sink) {
          // the row's stabiliser: the max over its valid columns of this tile
          float mx = -INFINITY;
          for (int cc = 0; cc < ncols; cc += 32) {
            uint32_t v[32];
            tmem_ld32(scol + half_c + cc, v);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int cl = cc + e;
              const bool okc = cl < ua || (cl >= ub0 && cl < ub1);
              if (okc) mx = fmaxf(mx, __uint_as_float(v[e]) * sl2);
            }
          }
          M = mx > -INFINITY ? mx : -1e30f;
          sm.mrow[slot][r] = M;
          mbar_arrive(&sm.m_ready[slot]);
        }
        const float negM = -M;
        if (none) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) w[e] = 0u;
#pragma unroll
          for (int pc = 0; pc < 64; pc += 16) tmem_st16(scol + pc, w);
        } else {
          // 64 columns per TMEM round trip (two loads, one wait); P is written
          // over S columns that this thread has already read
          for (int cc = 0; cc < ncols; cc += 64) {
            uint32_t v[64];
            tmem_ld32(scol + half_c + cc, v);
            tmem_ld32(scol + half_c + cc + 32, v + 32);
            tmem_ld_wait();
#pragma unroll
            for (int sub = 0; sub < 2; ++sub) {
              uint32_t w[16];
              softmax_chunk(v + 32 * sub, w, sl2, negM, full, cc + 32 * sub, ua, ub0, ub1, lacc);
              tmem_st16(scol + ((half_c + cc) >> 1) + 16 * sub, w);
            }
          }
          if (a.split) {
            // the other token's half of P is zero
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = 0u;
            const uint32_t oc = scol + (g_tok == 0 ? 32 : 0);
            tmem_st16(oc, w);
            tmem_st16(oc + 16, w);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&sm.p_full[sb]);
      }
      if (!ok) break;
      gt0 += un.nt;
      sm.lsum[slot][wg][r] = (lacc[0] + lacc[1]) + (lacc[2] + lacc[3]);
      mbar_arrive(&sm.l_ready[slot]);
    }
  } else {
    // ===================================================================== epilogue
    // Row sums of both softmax warpgroups, the output scale
    // 2^(M-X) / (l 2^(M-X) + 2^(sigma-X)) with X = max(M, sigma), and
    // lse = (M + log2 l) ln 2 (sink excluded); O read out of TMEM, scaled and
    // stored as bf16.
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int g_tok = r >> a.hshift;
    const int h = r & (Hu - 1);
    int it = 0;
    for (int u = blockIdx.x; u < a.n_units; u += gridDim.x, ++it) {
      const int slot = it & (kInfo - 1);
      if (!waitw(&sm.l_ready[slot], (it / kInfo) & 1, a, abort_flag, 12)) break;
      const Unit un = sm.info[slot];
      const float l = sm.lsum[slot][0][r] + sm.lsum[slot][1][r];
      const float M = a.has_sink ? sm.sink_l2[h] : sm.mrow[slot][r];
      mbar_arrive(&sm.info_free[slot]);           // unit descriptor, row sums and maxima read
      const RowRange rr = row_range(a, un, g_tok);
      const bool tok_ok = g_tok < un.ntok;
      const bool has_rows = rr.a1 > 0 || rr.b1 > rr.b0;
      const float sg = sm.sink_l2[h];
      float scale = 0.f, lse_v = -INFINITY;
      // fast-path range: every weight within 2^64 of the stabiliser
      const bool redo = tok_ok && has_rows && !(l > 0.f && l <= 18446744073709551616.0f);
      if (tok_ok && !redo && l > 0.f) {
        const float mx = fmaxf(M, sg);
        const float f = ex2(M - mx);
        const float den = fmaf(l, f, ex2(sg - mx));
        scale = f * rcp(den);
        lse_v = (M + lg2(l)) * 0.6931471805599453f;
      }
      const size_t qrow = (static_cast<size_t>(un.b) * a.Tq + a.row0 + un.r0 + g_tok) * a.H + h;
      if (tok_ok && !redo && a.lse != nullptr) a.lse[qrow] = lse_v;
      if (!waitw(&sm.o_full, it & 1, a, abort_flag, 13)) break;
      tc_fence_after();
      const bool store = tok_ok && !redo;
      __nv_bfloat16* orow = a.out + qrow * kDim;
      // O is single-buffered: read it out in two 64-column halves and release
      // it before the second half's stores
      {
        uint32_t v[64], w[32];
        tmem_ld32(tmem + lane_addr + kColO, v);
        tmem_ld32(tmem + lane_addr + kColO + 32, v + 32);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e)
          w[e] = pack_bf16(__uint_as_float(v[2 * e]) * scale, __uint_as_float(v[2 * e + 1]) * scale);
        if (store) {
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            *reinterpret_cast<uint4*>(orow + 8 * q4) = make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
        }
        tmem_ld32(tmem + lane_addr + kColO + 64, v);
        tmem_ld32(tmem + lane_addr + kColO + 96, v + 32);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&sm.o_empty);
#pragma unroll
        for (int e = 0; e < 32; ++e)
          w[e] = pack_bf16(__uint_as_float(v[2 * e]) * scale, __uint_as_float(v[2 * e + 1]) * scale);
        if (store) {
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            *reinterpret_cast<uint4*>(orow + 64 + 8 * q4) =
                make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
        }
      }
      // rows left to the exact path: the warp takes them one at a time
      uint32_t todo = __ballot_sync(0xffffffffu, redo);
      while (todo) {
        const int ln = __ffs(todo) - 1;
        todo &= todo - 1;
        const int rw = (warp & 3) * 32 + ln;
        row_exact(a, un, rw >> a.hshift, rw & (Hu - 1), sm.sink_l2);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace fa

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
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(fa::kDim), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(fa::kDim) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

// bf16 tcgen05 attention.  D == 128.  Sparse calls: H in {64, 128}, k <= 1024;
// dense calls: H in {16, 32, 64, 128}.
int launch_attn_tc(const void* q, const void* kv_c, const int32_t* idx, const void* kv_raw, const float* sink,
                   float tau, int W, int B, int Tq, int row0, int T_chunk, int H, int kv_bstride, int k, int S, int m,
                   int raw_cap, const int32_t* q_pos0, void* out, float* lse, int sparse, int* status,
                   cudaStream_t st) {
  using namespace fa;
  if (sparse) {
    CSA_REQUIRE(H == 64 || H == 128, CSA_ERR_UNSUPPORTED);
    CSA_REQUIRE(k <= kMaxTopk, CSA_ERR_UNSUPPORTED);
  } else {
    CSA_REQUIRE(H == 16 || H == 32 || H == 64 || H == 128, CSA_ERR_UNSUPPORTED);
  }
  Args a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.kv_c = static_cast<const __nv_bfloat16*>(kv_c);
  a.idx = idx;
  a.kv_raw = static_cast<const __nv_bfloat16*>(kv_raw ? kv_raw : kv_c);
  a.sink = sink;
  a.q_pos0 = q_pos0;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.status = status;
  CSA_REQUIRE(a.status != nullptr, CSA_ERR_CUDA);
  a.scale_log2 = tau * 1.4426950408889634f;
  a.W = W; a.Tq = Tq; a.row0 = row0; a.T_chunk = T_chunk; a.H = H; a.kv_bstride = kv_bstride; a.k = k;
  a.S = S; a.m = m; a.raw_cap = raw_cap > 0 ? raw_cap : 1;
  a.G = 128 / H;
  a.hshift = 31 - __builtin_clz(static_cast<unsigned>(H));
  a.sparse = sparse;
  a.split = sparse && H == 64;
  a.has_sink = sink != nullptr;
  a.upb = (T_chunk + a.G - 1) / a.G;
  const long long nu = static_cast<long long>(B) * a.upb;
  CSA_REQUIRE(nu < (1ll << 31), CSA_ERR_UNSUPPORTED);
  a.n_units = static_cast<int>(nu);
  a.wait_ns = wait_limit_ns();
  a.hint_ns = static_cast<unsigned>(a.wait_ns < 200000ull ? a.wait_ns : 200000ull);
  if (a.n_units == 0) return CSA_OK;
  const long long q_rows = static_cast<long long>(B) * Tq * H;
  const long long kv_rows = static_cast<long long>(B) * kv_bstride;
  const long long raw_rows = static_cast<long long>(B) * a.raw_cap;
  CSA_REQUIRE(q_rows < (1ll << 31) && kv_rows < (1ll << 31) - 1 && raw_rows < (1ll << 31) - 1, CSA_ERR_UNSUPPORTED);
  Maps maps;
  if (!make_map(&maps.q, q, static_cast<uint64_t>(q_rows), static_cast<uint32_t>(H)) ||
      !make_map(&maps.kv, kv_c, static_cast<uint64_t>(kv_rows), 64) ||
      !make_map(&maps.raw, kv_raw ? kv_raw : kv_c, static_cast<uint64_t>(kv_raw ? raw_rows : kv_rows), 64))
    return CSA_ERR_CUDA;
  const size_t smem = sizeof(Smem) + 1024;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_fa_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return set_cuda_error(e);
    attr_set = true;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = a.n_units < sms ? a.n_units : sms;
  attn_fa_kernel<<<grid, kThreads, smem, st>>>(a, maps);
  return check_launch();
}

}  // namespace csa
