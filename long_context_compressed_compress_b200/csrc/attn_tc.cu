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
//   producer warps (2): gather the unit's KV rows (top-k entries or every
//     visible entry, then the raw-window tokens) into 128-row tiles with
//     cp.async in the 128-byte-swizzled layout; load Q.
//   MMA warp (1): issues QK(i+1) before PV(i) so the tensor core works on the
//     next tile while the softmax runs.
//   softmax warpgroups (N/64, 4 warps each): thread = TMEM lane = KV row of S^T
//     and dim row of O^T; a warpgroup owns 64 columns.  Column maxima are warp
//     redux.sync.max + a 4-warp exchange; running maxima are raised only when a
//     tile exceeds them by 2^8 (then O^T and the row sums are rescaled), row
//     sums stay per thread until the unit's end.  P^T goes to shared memory as
//     bf16 (MN-major, swizzled) for the PV MMA.
// All waits are bounded; a wait that gives up sets the device status word and
// an abort flag that every role polls, so the kernel always returns.
#include "common.cuh"

namespace csa {

constexpr int kTcTile = 128;   // KV rows per tile
constexpr int kTcDim = 128;    // head dim

// NB = number of 64-column blocks of N; each softmax warpgroup owns 32 columns.
template <int NB>
struct TcCfg {
  static constexpr int N = 64 * NB;                       // MMA N (token, head) columns
  static constexpr int kGroups = N / 32;                  // softmax warpgroups
  static constexpr int kSoftWarps = 4 * kGroups;
  static constexpr int kProdWarps = NB == 1 ? 2 : 1;
  static constexpr int kThreads = 32 * (kSoftWarps + kProdWarps + 1);
  static constexpr int kStages = NB == 1 ? 4 : 2;
  static constexpr int kQBytes = N * kTcDim * 2;
  static constexpr int kKVBytes = kTcTile * kTcDim * 2;   // 32 KB
  static constexpr int kPBytes = kTcTile * N * 2;
  static constexpr uint32_t kTmemCols = 4 * N;            // S x2, O x2
};

struct TcUnit {
  int b, r0, ntok, n_c, n_w, jlo, p0, nt;
  int n_all;   // leading rows valid for every token of the unit
};

template <int NB>
struct __align__(1024) TcSmem {
  using C = TcCfg<NB>;
  uint8_t q[2][C::kQBytes];
  uint8_t kv[C::kStages][C::kKVBytes];
  uint8_t p[2][C::kPBytes];
  uint64_t kv_full[C::kStages], kv_empty[C::kStages];
  uint64_t q_full[2], q_empty[2], s_full[2], s_free[2], p_full[2], p_empty[2], o_full[2], o_empty[2];
  float xch[2 * NB][4][32];
  float mcol[2 * NB][32];
  float alpha[2 * NB][32];
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
  int n_units;
};

__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag) {
  for (long long i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255) == 255 && *abort_flag) return false;
  }
  atomicExch(status, CSA_ERR_TIMEOUT);
  *abort_flag = 1;
  return false;
}

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
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
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

template <int NB>
__global__ void __launch_bounds__(TcCfg<NB>::kThreads, 1) attn_tc_kernel(const TcArgs args) {
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
      mbar_init(&sm.q_full[s], 32 * C::kProdWarps);
      mbar_init(&sm.q_empty[s], 1 + 128 * C::kGroups);
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.s_free[s], 128 * C::kGroups);
      mbar_init(&sm.p_full[s], 128 * C::kGroups);
      mbar_init(&sm.p_empty[s], 1);
      mbar_init(&sm.o_full[s], 1);
      mbar_init(&sm.o_empty[s], 128 * C::kGroups);
    }
    sm.abort_flag = 0;
    fence_mbar_init();
  }
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
    const int pt = threadIdx.x - 32 * kProd0;   // 0..63
    int it = 0, kvc = 0;
    for (int u = blockIdx.x; u < args.n_units; u += gridDim.x, ++it) {
      if (*abort_flag) break;
      const int slot = it & 1;
      if (it >= 2 && !tc_wait(&sm.q_empty[slot], ((it >> 1) - 1) & 1, args.status, abort_flag)) break;
      const int b = u / args.units_per_b;
      const int r0 = (u - b * args.units_per_b) * args.G;
      const int ntok = min(args.G, args.T_chunk - r0);
      const int p0 = args.q_pos0[b] + args.row0 + r0;
      const int plast = p0 + ntok - 1;
      int n_c;
      const int32_t* irow = args.idx + (static_cast<size_t>(b) * args.T_chunk + r0) * args.k;
      if (args.sparse) {
        // indices are ascending with -1 padding at the end: binary-search the count
        int lo = 0, hi = args.k;
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (irow[mid] >= 0) lo = mid + 1; else hi = mid;
        }
        n_c = lo;
      } else {
        n_c = min(args.S, (plast + 1) / args.m);
      }
      int jlo = 0, n_w = 0;
      if (args.W > 0) {
        jlo = max(0, p0 - args.W + 1);
        n_w = plast - jlo + 1;
      }
      const int n_rows = n_c + n_w;
      const int nt = max(1, (n_rows + kTcTile - 1) / kTcTile);
      const int n_all = args.G > 1 ? min(n_c, (p0 + 1) / args.m) : n_rows;
      if (pt == 0) sm.info[slot] = TcUnit{b, r0, ntok, n_c, n_w, jlo, p0, nt, n_all};
      // ---- Q: N rows (token-major, head-minor), 16 chunks of 16 B each
      {
        const uint32_t qs = smem_u32(sm.q[slot]);
        const size_t qrow0 = (static_cast<size_t>(b) * args.Tq + args.row0 + r0) * args.H;
        for (int i = pt; i < N * 16; i += 32 * C::kProdWarps) {
          const int row = i >> 4, ch = i & 15;
          const bool ok = row < ntok * args.H;
          const __nv_bfloat16* src = args.q + (ok ? (qrow0 + row) * kTcDim + ch * 8 : 0);
          cp_async16(qs + sw128_off(row, ch, N), src, ok ? 16u : 0u);
        }
        cp_async_mbar_arrive(&sm.q_full[slot]);
      }
      // ---- KV tiles
      for (int i = 0; i < nt; ++i, ++kvc) {
        const int stage = kvc % C::kStages;
        const int use = kvc / C::kStages;
        if (use >= 1 && !tc_wait(&sm.kv_empty[stage], (use - 1) & 1, args.status, abort_flag)) break;
        const uint32_t ks = smem_u32(sm.kv[stage]);
#pragma unroll
        for (int rr2 = 0; rr2 < kTcTile / (32 * C::kProdWarps); ++rr2) {
          const int rr = pt + rr2 * 32 * C::kProdWarps;
          const int L = i * kTcTile + rr;
          const __nv_bfloat16* src = nullptr;
          if (L < n_c) {
            const int s = args.sparse ? irow[L] : L;
            src = args.kv_c + (static_cast<size_t>(b) * args.kv_bstride + s) * kTcDim;
          } else if (L < n_rows) {
            const int j = jlo + (L - n_c);
            src = args.kv_raw + (static_cast<size_t>(b) * args.raw_cap + (j % args.raw_cap)) * kTcDim;
          }
#pragma unroll
          for (int ch = 0; ch < 16; ++ch)
            cp_async16(ks + sw128_off(rr, ch, kTcTile), src ? src + ch * 8 : args.kv_c, src ? 16u : 0u);
        }
        cp_async_mbar_arrive(&sm.kv_full[stage]);
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
          const int sb = g & 1, suse = g >> 1;
          if (suse >= 1 && !tc_wait(&sm.s_free[sb], (suse - 1) & 1, args.status, abort_flag)) return false;
          fence_proxy_async();
          tc_fence_after();
          const uint32_t kb = smem_u32(sm.kv[stage]);
#pragma unroll
          for (int j = 0; j < kTcDim / 16; ++j)
            mma_bf16(tmem + sb * N, desc_kmajor(kb, kTcTile * 128, j), desc_kmajor(qbase, N * 128, j), idesc_qk,
                     j > 0 ? 1u : 0u);
          tc_commit(&sm.s_full[sb]);
          return true;
        };
        if (!issue_qk(0)) { ok = false; break; }
        for (int i = 0; i < nt; ++i) {
          if (i + 1 < nt && !issue_qk(i + 1)) { ok = false; break; }
          const int g = gt + i;
          const int pb = g & 1, puse = g >> 1;
          if (!tc_wait(&sm.p_full[pb], puse & 1, args.status, abort_flag)) { ok = false; break; }
          if (i == 0 && ouse >= 1 && !tc_wait(&sm.o_empty[ob], (ouse - 1) & 1, args.status, abort_flag)) {
            ok = false;
            break;
          }
          fence_proxy_async();
          tc_fence_after();
          const int stage = (kvc + i) % C::kStages;
          const uint32_t kb = smem_u32(sm.kv[stage]);
          const uint32_t pbase = smem_u32(sm.p[pb]);
#pragma unroll
          for (int j = 0; j < kTcTile / 16; ++j)
            mma_bf16(tmem + 2 * N + ob * N, desc_mnmajor(kb, kTcTile * 128, j), desc_mnmajor(pbase, kTcTile * 128, j),
                     idesc_pv, (i > 0 || j > 0) ? 1u : 0u);
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
  } else {
    // ===================================================================== softmax
    const int wg = warp >> 2, wq = warp & 3;    // warpgroup wg owns columns [32 wg, 32 wg + 32)
    const int row = wq * 32 + lane;             // TMEM lane: KV tile row / O^T dim row
    const int bar_id = 1 + wg;
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    const int col0 = 32 * wg;
    const float sl2 = args.scale_log2;
    int it = 0, gt = 0;
    for (int u = blockIdx.x; u < args.n_units; u += gridDim.x, ++it) {
      const int slot = it & 1;
      if (!tc_wait(&sm.q_full[slot], (it >> 1) & 1, args.status, abort_flag)) break;
      const TcUnit inf = sm.info[slot];
      const int n_rows = inf.n_c + inf.n_w;
      const int ob = it & 1, ouse = it >> 1;
      float lpart[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) lpart[c] = 0.f;
      if (row < 32) sm.mcol[wg][row] = -INFINITY;
      named_bar_sync(bar_id, 128);
      bool ok = true;
      for (int i = 0; i < inf.nt; ++i, ++gt) {
        const int sb = gt & 1;
        if (!tc_wait(&sm.s_full[sb], (gt >> 1) & 1, args.status, abort_flag)) { ok = false; break; }
        tc_fence_after();
        float s[32];
        {
          uint32_t v[32];
          tmem_ld32(tmem + lane_addr + sb * N + col0, v);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c) s[c] = __uint_as_float(v[c]);
        }
        tc_fence_before();
        mbar_arrive(&sm.s_free[sb]);
        // ---- masks (only tiles that reach past the rows every token sees):
        // padding rows, and for multi-token units per-token visibility
        if ((i + 1) * kTcTile > inf.n_all) {
          const int L = i * kTcTile + row;
          if (L >= n_rows) {
#pragma unroll
            for (int c = 0; c < 32; ++c) s[c] = -INFINITY;
          } else if (args.G > 1) {
            uint32_t vmask = 0;
            for (int g = 0; g < args.G; ++g) {
              const int p = inf.p0 + g;
              bool vis;
              if (L < inf.n_c) {
                vis = args.m * (L + 1) - 1 <= p;
              } else {
                const int j = inf.jlo + (L - inf.n_c);
                vis = j <= p && j > p - args.W;
              }
              if (vis && g < inf.ntok) vmask |= 1u << g;
            }
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (!((vmask >> ((col0 + c) >> args.hshift)) & 1u)) s[c] = -INFINITY;
          }
        }
        // ---- column maxima: warp redux, then 4-warp exchange
#pragma unroll
        for (int c4 = 0; c4 < 32; c4 += 4) {
          const float a0 = redux_max(s[c4]), a1 = redux_max(s[c4 + 1]);
          const float a2 = redux_max(s[c4 + 2]), a3 = redux_max(s[c4 + 3]);
          if (lane == 0) *reinterpret_cast<float4*>(&sm.xch[wg][wq][c4]) = make_float4(a0, a1, a2, a3);
        }
        named_bar_sync(bar_id, 128);
        bool need = false;
        if (row < 32) {
          const int c = row;
          const float tmax = fmaxf(fmaxf(sm.xch[wg][0][c], sm.xch[wg][1][c]), fmaxf(sm.xch[wg][2][c], sm.xch[wg][3][c]));
          const float tm = tmax * sl2;
          const float mo = sm.mcol[wg][c];
          float mn = mo, a = 1.f;
          if (tm > mo + 8.0f) {
            mn = tm;
            a = (mo == -INFINITY) ? 0.f : exp2f(mo - mn);
            need = (i > 0) && (mo != -INFINITY);
          }
          sm.mcol[wg][c] = mn;
          sm.alpha[wg][c] = a;
        }
        const bool rescale = bar_red_or(bar_id, 128, need);
        if (rescale) {
          // rare: the running max rose by more than 2^8; PV(i-1) must be complete
          const int gp = gt - 1;
          if (!tc_wait(&sm.p_empty[gp & 1], (gp >> 1) & 1, args.status, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t oaddr = tmem + lane_addr + 2 * N + ob * N + col0;
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            uint32_t v[16];
            tmem_ld16(oaddr + 16 * h2, v);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float a = sm.alpha[wg][16 * h2 + c];
              v[c] = __float_as_uint(__uint_as_float(v[c]) * a);
              lpart[16 * h2 + c] *= a;
            }
            tmem_st16(oaddr + 16 * h2, v);
          }
          tmem_st_wait();
          tc_fence_before();
        }
        // ---- P^T = 2^(s * scale_log2 - m), row sums, bf16 into shared memory
        const int pb = gt & 1, puse = gt >> 1;
        if (puse >= 1 && !tc_wait(&sm.p_empty[pb], (puse - 1) & 1, args.status, abort_flag)) { ok = false; break; }
        const uint32_t prow = smem_u32(sm.p[pb]) + (wg >> 1) * (kTcTile * 128) + row * 128;
#pragma unroll
        for (int c8 = 0; c8 < 32; c8 += 8) {
          const float4 m0 = *reinterpret_cast<const float4*>(&sm.mcol[wg][c8]);
          const float4 m1 = *reinterpret_cast<const float4*>(&sm.mcol[wg][c8 + 4]);
          const float mm[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
          float pv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float me = mm[e] == -INFINITY ? 0.f : mm[e];
            pv[e] = fast_ex2(fmaf(s[c8 + e], sl2, -me));
            lpart[c8 + e] += pv[e];
          }
          const uint32_t w0 = pack_bf16(pv[0], pv[1]), w1 = pack_bf16(pv[2], pv[3]);
          const uint32_t w2 = pack_bf16(pv[4], pv[5]), w3 = pack_bf16(pv[6], pv[7]);
          const int chunk = (wg & 1) * 4 + (c8 >> 3);
          const uint32_t addr = prow + ((chunk ^ (row & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w0), "r"(w1), "r"(w2), "r"(w3)
                       : "memory");
        }
        fence_proxy_async();
        mbar_arrive(&sm.p_full[pb]);
      }
      if (!ok) break;
      // ---- unit epilogue: column sums of lpart over the 128 rows (butterfly:
      // lane l ends with column l's warp total), then the 4-warp total
#pragma unroll
      for (int st = 16; st >= 1; st >>= 1) {
        const bool up = (lane & st) != 0;
#pragma unroll
        for (int e = 0; e < st; ++e) {
          const float send = up ? lpart[e] : lpart[e + st];
          const float keep = up ? lpart[e + st] : lpart[e];
          lpart[e] = keep + __shfl_xor_sync(0xffffffffu, send, st);
        }
      }
      sm.xch[wg][wq][lane] = lpart[0];
      named_bar_sync(bar_id, 128);
      if (row < 32) {
        const int c = row;
        sm.alpha[wg][c] = (sm.xch[wg][0][c] + sm.xch[wg][1][c]) + (sm.xch[wg][2][c] + sm.xch[wg][3][c]);
      }
      named_bar_sync(bar_id, 128);
      if (!tc_wait(&sm.o_full[ob], ouse & 1, args.status, abort_flag)) break;
      tc_fence_after();
      {
        const uint32_t oaddr = tmem + lane_addr + 2 * N + ob * N + col0;
        const int d = row;
        uint32_t v[32];
        tmem_ld32(oaddr, v);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int col = col0 + c;
          const int g = col >> args.hshift, h = col & (args.H - 1);
          if (g >= inf.ntok) continue;
          const float mcl = sm.mcol[wg][c];
          const float l = sm.alpha[wg][c];
          float res = 0.f;
          if (mcl != -INFINITY) {
            const float sg = args.sink ? args.sink[h] * 1.4426950408889634f : -INFINITY;
            const float mx = fmaxf(mcl, sg);
            const float f = exp2f(mcl - mx);
            const float den = fmaf(l, f, exp2f(sg - mx));
            res = den > 0.f ? __fdiv_rn(__uint_as_float(v[c]) * f, den) : 0.f;
          }
          const size_t orow = (static_cast<size_t>(inf.b) * args.Tq + args.row0 + inf.r0 + g) * args.H + h;
          args.out[orow * kTcDim + d] = __float2bfloat16_rn(res);
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.o_empty[ob]);
      if (args.lse != nullptr && row < 32) {
        const int col = col0 + row;
        const int g = col >> args.hshift, h = col & (args.H - 1);
        if (g < inf.ntok) {
          const float mcl = sm.mcol[wg][row];
          const float l = sm.alpha[wg][row];
          const float v = (mcl == -INFINITY || !(l > 0.f)) ? -INFINITY : (mcl + log2f(l)) * 0.6931471805599453f;
          args.lse[(static_cast<size_t>(inf.b) * args.Tq + args.row0 + inf.r0 + g) * args.H + h] = v;
        }
      }
      named_bar_sync(bar_id, 128);      // mcol / alpha reused by the next unit
      mbar_arrive(&sm.q_empty[slot]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int NB>
int launch_attn_tc_nb(const TcArgs& a, cudaStream_t st) {
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
  attn_tc_kernel<NB><<<grid, TcCfg<NB>::kThreads, smem, st>>>(a);
  return check_launch();
}

// bf16 tcgen05 attention.  Requirements: D == 128, and N = G*H in {64, 128}
// with G = 1 for sparse (CSA) units; for dense (HCA) units G = 128 / H.
int launch_attn_tc(const void* q, const void* kv_c, const int32_t* idx, const void* kv_raw, const float* sink,
                   float tau, int W, int B, int Tq, int row0, int T_chunk, int H, int kv_bstride, int k, int S, int m,
                   int raw_cap, const int32_t* q_pos0, void* out, float* lse, int sparse, cudaStream_t st) {
  int G = 1;
  if (sparse) {
    CSA_REQUIRE(H == 64 || H == 128, CSA_ERR_UNSUPPORTED);
  } else {
    CSA_REQUIRE(H == 16 || H == 32 || H == 64 || H == 128, CSA_ERR_UNSUPPORTED);
    G = 128 / H;
  }
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
  a.units_per_b = (T_chunk + G - 1) / G;
  const long long nu = static_cast<long long>(B) * a.units_per_b;
  CSA_REQUIRE(nu < (1ll << 31), CSA_ERR_UNSUPPORTED);
  a.n_units = static_cast<int>(nu);
  if (a.n_units == 0) return CSA_OK;
  return N == 64 ? launch_attn_tc_nb<1>(a, st) : launch_attn_tc_nb<2>(a, st);
}

}  // namespace csa
