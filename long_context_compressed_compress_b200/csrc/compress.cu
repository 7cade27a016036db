// Streaming kernels of the CSA/HCA layer: the gated overlapping 4:1 compressor
// (cf-1.com/news/5231315 §3.1), the 128:1 compressor (§3.2), NVFP4 block
// quantisation of the indexer QK path (§3.4, §4.4), and the decode-state
// helpers (ring append, position advance, the fused per-step state update;
// §4.4 KV cache tiers).
//
// All of these are HBM-bound: one thread owns 8 channels of one entry and
// moves 16-byte vectors, consecutive threads cover consecutive channels so a
// warp reads whole contiguous rows.
#include "common.cuh"

namespace csa {

__device__ int g_dev_status = 0;

static thread_local int t_last_cuda_error = 0;

int* device_status_ptr() {
  static int* ptrs[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (ptrs[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dev_status) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int*>(p);
  }
  return ptrs[dev];
}

static uint64_t g_wait_limit_ns = 0;   // 0: the default of 2 s
uint64_t wait_limit_ns() { return g_wait_limit_ns ? g_wait_limit_ns : 2000000000ull; }

int set_cuda_error(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return CSA_ERR_CUDA;
}
int check_launch() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? CSA_OK : set_cuda_error(e);
}

// ---------------------------------------------------------------------------
// The gated pooling of one compressed entry for 8 channels (one thread): the
// per-channel max of the 2m gate logits, then the exp-weighted sums of a over
// the block's rows cur0 .. cur0 + m - 1 and of b over the predecessor's rows
// pred0 .. (when has_pred), in fp32; the result rounded to Tout.  a, b, z
// point at the thread's 8 channels of row 0 of its slab.  Shared by the
// compressor and the fused decode-state update, so both give the same bits.
// ---------------------------------------------------------------------------
template <typename Tin, typename Tout>
__device__ __forceinline__ void pool_entry8(const Tin* __restrict__ a, const Tin* __restrict__ b,
                                            const Tin* __restrict__ zb, int D, int m, int cur0, int pred0,
                                            int has_pred, bool active, float e8[8]) {
  float mx[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) mx[c] = -INFINITY;
  float v[8];
  if (active) {
    for (int r = 0; r < m; ++r) {
      Vec8<Tin>::load(zb + static_cast<size_t>(cur0 + r) * D, v);
#pragma unroll
      for (int c = 0; c < 8; ++c) mx[c] = fmaxf(mx[c], v[c]);
      if (has_pred) {
        Vec8<Tin>::load(zb + static_cast<size_t>(pred0 + r) * D, v);
#pragma unroll
        for (int c = 0; c < 8; ++c) mx[c] = fmaxf(mx[c], v[c]);
      }
    }
  }
  float sum[8], acc[8], x[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) { sum[c] = 0.f; acc[c] = 0.f; }
  if (active) {
    for (int r = 0; r < m; ++r) {
      Vec8<Tin>::load(zb + static_cast<size_t>(cur0 + r) * D, v);
      Vec8<Tin>::load(a + static_cast<size_t>(cur0 + r) * D, x);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float e = expf(v[c] - mx[c]);
        sum[c] += e;
        acc[c] = fmaf(e, x[c], acc[c]);
      }
      if (has_pred) {
        Vec8<Tin>::load(zb + static_cast<size_t>(pred0 + r) * D, v);
        Vec8<Tin>::load(b + static_cast<size_t>(pred0 + r) * D, x);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float e = expf(v[c] - mx[c]);
          sum[c] += e;
          acc[c] = fmaf(e, x[c], acc[c]);
        }
      }
    }
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) e8[c] = active ? round_to(__fdiv_rn(acc[c], sum[c]), (Tout*)nullptr) : 0.f;
}

// ---------------------------------------------------------------------------
// csa_compress: thread = (b, entry, 8-channel group).  Two passes over the 2m
// rows of the block pair: the per-channel max of the gate logits, then the
// exp-weighted sums of a (current block) and b (predecessor block).
// ---------------------------------------------------------------------------
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) csa_compress_kernel(
    const Tin* __restrict__ a, const Tin* __restrict__ b, const Tin* __restrict__ z, int B, int T, int D, int m,
    int fhp, int S, const int32_t* __restrict__ ring_pos, int out_bstride, Tout* __restrict__ out,
    uint8_t* __restrict__ out_fp4, uint8_t* __restrict__ out_sf, float g) {
  const int G = D >> 3;
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const bool decode = ring_pos != nullptr;
  const long long total = decode ? static_cast<long long>(B) * G : static_cast<long long>(B) * S * G;
  const bool valid = gid < total;
  const long long g2 = valid ? gid : 0;
  const int cg = static_cast<int>(g2 % G);
  long long eidx;   // entry index written (within the batch row)
  int bi;
  // row offsets (within the batch's [rows, D] slab) of the current / predecessor blocks
  int cur0, pred0, has_pred;
  bool active = valid;
  if (!decode) {
    const long long e = (g2 / G) % S;
    bi = static_cast<int>(g2 / (static_cast<long long>(G) * S));
    const int blk = static_cast<int>(e) + fhp;
    cur0 = m * blk;
    pred0 = m * (blk - 1);
    has_pred = blk > 0;
    eidx = e;
  } else {
    bi = static_cast<int>(g2 / G);
    const int p = ring_pos[bi];
    const int i = (p + 1) / m - 1;
    // an entry is emitted when block i completes; entries past the cache's
    // capacity (out_bstride rows) are dropped rather than written out of bounds
    active = valid && ((p + 1) % m == 0) && i >= 0 && i < out_bstride;
    cur0 = (i & 1) * m;
    pred0 = ((i + 1) & 1) * m;
    has_pred = i > 0;
    eidx = i;
  }
  const int rows = decode ? 2 * m : T;
  const size_t slab = static_cast<size_t>(bi) * rows * D + static_cast<size_t>(cg) * 8;
  float e8[8];
  pool_entry8<Tin, Tout>(a + slab, b + slab, z + slab, D, m, cur0, pred0, has_pred, active, e8);
  const size_t orow = static_cast<size_t>(bi) * out_bstride + static_cast<size_t>(eidx);
  if (out != nullptr && active) Vec8<Tout>::store(out + orow * D + cg * 8, e8);
  if (out_fp4 != nullptr) {
    // 16-element NVFP4 block = this thread's 8 channels + its neighbour's.
    float am = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) am = fmaxf(am, fabsf(e8[c]));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
    uint32_t sfb;
    const uint32_t codes = nvfp4_encode8(e8, am, g, &sfb);
    if (active) {
      reinterpret_cast<uint32_t*>(out_fp4 + orow * (D / 2))[cg] = codes;
      if ((cg & 1) == 0) out_sf[orow * (D / 16) + (cg >> 1)] = static_cast<uint8_t>(sfb);
    }
  }
}

// ---------------------------------------------------------------------------
// hca_compress: CTA = (b, entry).  Thread (rg, cg) reduces rows rg, rg+RG, ...
// of the block for 8 channels (max, then exp-sums with its own max); the RG
// partial (max, sum, acc) triples are merged in shared memory.
// ---------------------------------------------------------------------------
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) hca_compress_kernel(const Tin* __restrict__ a, const Tin* __restrict__ z,
                                                           int T, int D, int m, int S, Tout* __restrict__ out) {
  extern __shared__ float sm[];
  const int G = D >> 3;
  const int RG = blockDim.x / G;
  const int cg = threadIdx.x % G;
  const int rg = threadIdx.x / G;
  const int e = blockIdx.x % S;
  const int bi = blockIdx.x / S;
  const size_t base = (static_cast<size_t>(bi) * T + static_cast<size_t>(e) * m) * D + cg * 8;
  float mx[8], sum[8], acc[8], v[8], x[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) { mx[c] = -INFINITY; sum[c] = 0.f; acc[c] = 0.f; }
  for (int r = rg; r < m; r += RG) {
    Vec8<Tin>::load(z + base + static_cast<size_t>(r) * D, v);
#pragma unroll
    for (int c = 0; c < 8; ++c) mx[c] = fmaxf(mx[c], v[c]);
  }
  for (int r = rg; r < m; r += RG) {
    Vec8<Tin>::load(z + base + static_cast<size_t>(r) * D, v);
    Vec8<Tin>::load(a + base + static_cast<size_t>(r) * D, x);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float ex = expf(v[c] - mx[c]);
      sum[c] += ex;
      acc[c] = fmaf(ex, x[c], acc[c]);
    }
  }
  // partials: sm[(rg*3 + {0,1,2}) * D + channel]
  const int ch = cg * 8;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    sm[(rg * 3 + 0) * D + ch + c] = mx[c];
    sm[(rg * 3 + 1) * D + ch + c] = sum[c];
    sm[(rg * 3 + 2) * D + ch + c] = acc[c];
  }
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float M = -INFINITY;
    for (int r = 0; r < RG; ++r) M = fmaxf(M, sm[(r * 3) * D + c]);
    float Ssum = 0.f, A = 0.f;
    for (int r = 0; r < RG; ++r) {
      const float mr = sm[(r * 3) * D + c];
      if (mr == -INFINITY) continue;     // row group saw no rows (m < RG)
      const float f = expf(mr - M);
      Ssum = fmaf(sm[(r * 3 + 1) * D + c], f, Ssum);
      A = fmaf(sm[(r * 3 + 2) * D + c], f, A);
    }
    const float val = __fdiv_rn(A, Ssum);
    Tout* o = out + (static_cast<size_t>(bi) * S + e) * D + c;
    *o = static_cast<Tout>(val);
  }
}

// ---------------------------------------------------------------------------
// nvfp4_quantize: thread = 8 elements; pairs of threads share a 16-block.
// ---------------------------------------------------------------------------
template <typename Tin>
__global__ void __launch_bounds__(256) nvfp4_quantize_kernel(const Tin* __restrict__ x, long long n8, float g,
                                                             uint8_t* __restrict__ packed,
                                                             uint8_t* __restrict__ sf) {
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const bool valid = gid < n8;
  float v[8];
  if (valid) {
    Vec8<Tin>::load(x + gid * 8, v);
  } else {
#pragma unroll
    for (int c = 0; c < 8; ++c) v[c] = 0.f;
  }
  float am = 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) am = fmaxf(am, fabsf(v[c]));
  am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
  uint32_t sfb;
  const uint32_t codes = nvfp4_encode8(v, am, g, &sfb);
  if (valid) {
    reinterpret_cast<uint32_t*>(packed)[gid] = codes;
    if ((gid & 1) == 0) sf[gid >> 1] = static_cast<uint8_t>(sfb);
  }
}

// ---------------------------------------------------------------------------
// decode helpers
// ---------------------------------------------------------------------------
template <typename T>
__global__ void ring_append_kernel(const T* __restrict__ rows, int B, int D, T* __restrict__ ring, int cap,
                                   const int32_t* __restrict__ pos) {
  const int bi = blockIdx.x;
  const int slot = pos[bi] % cap;
  for (int c = threadIdx.x; c < D; c += blockDim.x)
    ring[(static_cast<size_t>(bi) * cap + slot) * D + c] = rows[static_cast<size_t>(bi) * D + c];
}

// One CTA per (sequence, snapshot); thread = (slot, 8-channel group).  Slot s
// of the destination ring holds the token j <= p with j = s (mod dst_cap)
// closest to p; it is copied when j lies in the snapshot's row range and is
// >= 0, else zeroed, so every slot of the destination is written.
template <typename T>
__global__ void state_gather_kernel(const T* __restrict__ src, int D, int src_cap, const int32_t* __restrict__ pos,
                                    int npos, int m, int nrows, T* __restrict__ dst, int dst_cap) {
  const int snap = blockIdx.x;                 // b * npos + c
  const int b = snap / npos;
  const int p = pos[snap];
  int lo;
  if (m > 0) lo = m * ((p + 1) / m - 1);       // last complete block and the block in progress
  else lo = p - nrows + 1;                     // the window
  const int G = D >> 3;
  for (int e = threadIdx.x; e < dst_cap * G; e += blockDim.x) {
    const int sl = e / G, g = e - sl * G;
    int d = (p - sl) % dst_cap;
    if (d < 0) d += dst_cap;
    const int j = p - d;
    float v[8];
    if (p >= 0 && j >= 0 && j >= lo) {
      int ss = j % src_cap;
      Vec8<T>::load(src + (static_cast<size_t>(b) * src_cap + ss) * D + 8 * g, v);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
    }
    Vec8<T>::store(dst + (static_cast<size_t>(snap) * dst_cap + sl) * D + 8 * g, v);
  }
}

__global__ void pos_advance_kernel(int32_t* pos, int B, int delta) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < B) pos[i] += delta;
}


// ---------------------------------------------------------------------------
// Fused decode-state update, one CTA per sequence: the work of six compressor
// carry appends, the raw-window append, the two decode-mode compressions and
// the q_I quantisation of one decode step, in one launch with the same results
// (the same pooling and NVFP4 code as the separate kernels).
//   threads [0, 3 G + 3 GI + G) : 16-byte copies of this step's rows into the
//                                 carry rings (slot p % 2m) and the window ring
//                                 (slot p % W)
//   warps   [0, wk)             : the KV entry, one thread per 8 channels
//   warp    wk                  : the indexer key entry + NVFP4 (GI <= 32)
//   warps   [wq, wq + nq)       : q_I -> NVFP4, one thread per 8 values
// ---------------------------------------------------------------------------
struct DecodeUpdateArgs {
  const void* row[7];        // a, b, z, a_I, b_I, z_I, kv_raw: [B, D or DI]
  void* ring[7];             // carry rings [B, 2m, D or DI] (x6), window ring [B, W, D]
  const void* q_I;           // [B, HI, DI]
  void* kv_c;                // [B, cap, D]
  uint8_t* k_fp4;            // [B, cap, DI/2]
  uint8_t* k_sf;             // [B, cap, DI/16]
  uint8_t* q_fp4;            // [B, HI, DI/2]
  uint8_t* q_sf;             // [B, HI, DI/16]
  const int32_t* pos;
  int D, DI, HI, m, W, cap, wk, wq;
  float g;
};

template <typename T>
__global__ void __launch_bounds__(256) decode_update_kernel(const DecodeUpdateArgs args) {
  const DecodeUpdateArgs& a = args;
  const int bi = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int p = a.pos[bi];
  const int G = a.D >> 3, GI = a.DI >> 3;
  // ---- appends (16 bytes = 8 elements per thread and copy)
  const int cslot = p % (2 * a.m), rslot = p % a.W;
  for (int v = tid; v < 3 * G + 3 * GI + G; v += blockDim.x) {
    int s, off, width, slot, cap;
    if (v < 3 * G) {
      s = v / G; off = v - s * G; width = a.D; slot = cslot; cap = 2 * a.m;
    } else if (v < 3 * G + 3 * GI) {
      const int u = v - 3 * G;
      s = 3 + u / GI; off = u - (u / GI) * GI; width = a.DI; slot = cslot; cap = 2 * a.m;
    } else {
      s = 6; off = v - 3 * G - 3 * GI; width = a.D; slot = rslot; cap = a.W;
    }
    const uint4 x = reinterpret_cast<const uint4*>(static_cast<const T*>(a.row[s]) + static_cast<size_t>(bi) * width)[off];
    reinterpret_cast<uint4*>(static_cast<T*>(a.ring[s]) + (static_cast<size_t>(bi) * cap + slot) * width)[off] = x;
  }
  __syncthreads();
  // ---- the entry (p + 1) / m - 1 when this token completes its block
  const int i = (p + 1) / a.m - 1;
  const bool emit = ((p + 1) % a.m == 0) && i >= 0 && i < a.cap;
  const int cur0 = (i & 1) * a.m, pred0 = ((i + 1) & 1) * a.m;
  const int has_pred = i > 0;
  if (warp < a.wk) {
    const int cg = tid;
    if (cg < G) {
      const size_t slab = static_cast<size_t>(bi) * 2 * a.m * a.D + static_cast<size_t>(cg) * 8;
      float e8[8];
      pool_entry8<T, T>(static_cast<const T*>(a.ring[0]) + slab, static_cast<const T*>(a.ring[1]) + slab,
                        static_cast<const T*>(a.ring[2]) + slab, a.D, a.m, cur0, pred0, has_pred, emit, e8);
      if (emit) Vec8<T>::store(static_cast<T*>(a.kv_c) + (static_cast<size_t>(bi) * a.cap + i) * a.D + cg * 8, e8);
    }
  } else if (warp == a.wk) {
    const int cg = lane;
    const bool act = emit && cg < GI;
    const size_t slab = static_cast<size_t>(bi) * 2 * a.m * a.DI + static_cast<size_t>(cg < GI ? cg : 0) * 8;
    float e8[8];
    pool_entry8<T, T>(static_cast<const T*>(a.ring[3]) + slab, static_cast<const T*>(a.ring[4]) + slab,
                      static_cast<const T*>(a.ring[5]) + slab, a.DI, a.m, cur0, pred0, has_pred, act, e8);
    // 16-element NVFP4 block = this lane's 8 channels + its neighbour's
    float am = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) am = fmaxf(am, fabsf(e8[c]));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
    uint32_t sfb;
    const uint32_t codes = nvfp4_encode8(e8, am, a.g, &sfb);
    if (act) {
      const size_t orow = static_cast<size_t>(bi) * a.cap + i;
      reinterpret_cast<uint32_t*>(a.k_fp4 + orow * (a.DI / 2))[cg] = codes;
      if ((cg & 1) == 0) a.k_sf[orow * (a.DI / 16) + (cg >> 1)] = static_cast<uint8_t>(sfb);
    }
  } else if (warp >= a.wq) {
    // ---- q_I of this sequence: HI * DI / 8 threads of 8 values
    const int n8 = a.HI * a.DI / 8;
    const int u = tid - 32 * a.wq;
    const bool ok = u < n8;
    const long long gid = static_cast<long long>(bi) * n8 + (ok ? u : 0);
    float v[8];
    if (ok) {
      Vec8<T>::load(static_cast<const T*>(a.q_I) + gid * 8, v);
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) v[c] = 0.f;
    }
    float am = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) am = fmaxf(am, fabsf(v[c]));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
    uint32_t sfb;
    const uint32_t codes = nvfp4_encode8(v, am, a.g, &sfb);
    if (ok) {
      reinterpret_cast<uint32_t*>(a.q_fp4)[gid] = codes;
      if ((gid & 1) == 0) a.q_sf[gid >> 1] = static_cast<uint8_t>(sfb);
    }
  }
}
}  // namespace csa

using namespace csa;

// ============================================================== C ABI entries
extern "C" {

const char* csa_status_string(int status) {
  switch (status) {
    case CSA_OK: return "CSA_OK";
    case CSA_ERR_INVALID_ARG: return "CSA_ERR_INVALID_ARG";
    case CSA_ERR_UNSUPPORTED: return "CSA_ERR_UNSUPPORTED";
    case CSA_ERR_ALIGNMENT: return "CSA_ERR_ALIGNMENT";
    case CSA_ERR_CUDA: return "CSA_ERR_CUDA";
    case CSA_ERR_TIMEOUT: return "CSA_ERR_TIMEOUT";
    default: return "CSA_ERR_UNKNOWN";
  }
}

int csa_last_cuda_error(void) { return t_last_cuda_error; }

int csa_version(void) { return 100; }

int csa_set_wait_timeout_ns(uint64_t ns) {
  g_wait_limit_ns = ns;
  return CSA_OK;
}

int csa_device_status(int* status_out) {
  if (status_out == nullptr) return CSA_ERR_INVALID_ARG;
  int v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_dev_status, sizeof(int));
  if (e != cudaSuccess) return set_cuda_error(e);
  e = cudaMemcpyToSymbol(g_dev_status, &zero, sizeof(int));
  if (e != cudaSuccess) return set_cuda_error(e);
  *status_out = v;
  return CSA_OK;
}

int csa_compress(const void* a, const void* b, const void* z, int in_dtype, int B, int T, int D, int m,
                 int first_has_pred, const int32_t* ring_pos, int out_bstride, void* out, int out_dtype,
                 uint8_t* out_fp4, uint8_t* out_sf, float gscale, csa_stream_t stream) {
  CSA_REQUIRE(a && b && z, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(out || out_fp4, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(B >= 0 && T >= 0 && D > 0 && m >= 1 && m <= 16, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(in_dtype == CSA_F32 || in_dtype == CSA_BF16, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(out_dtype == CSA_F32 || out_dtype == CSA_BF16, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(D % 8 == 0, CSA_ERR_UNSUPPORTED);
  CSA_REQUIRE(aligned16(a) && aligned16(b) && aligned16(z), CSA_ERR_ALIGNMENT);
  CSA_REQUIRE(!out || aligned16(out), CSA_ERR_ALIGNMENT);
  if (out_fp4) {
    CSA_REQUIRE(out_sf != nullptr && gscale > 0.f, CSA_ERR_INVALID_ARG);
    CSA_REQUIRE(D % 16 == 0, CSA_ERR_UNSUPPORTED);
    CSA_REQUIRE((reinterpret_cast<uintptr_t>(out_fp4) & 3u) == 0, CSA_ERR_ALIGNMENT);
  }
  const bool decode = ring_pos != nullptr;
  int S = 0;
  if (!decode) {
    CSA_REQUIRE(first_has_pred == 0 || first_has_pred == 1, CSA_ERR_INVALID_ARG);
    S = T / m - first_has_pred;
    if (S <= 0 || B == 0) return CSA_OK;
    if (out_bstride == 0) out_bstride = S;
    CSA_REQUIRE(out_bstride >= S, CSA_ERR_INVALID_ARG);
  } else {
    CSA_REQUIRE(out_bstride > 0, CSA_ERR_INVALID_ARG);
    if (B == 0) return CSA_OK;
  }
  const long long threads = decode ? static_cast<long long>(B) * (D / 8) : static_cast<long long>(B) * S * (D / 8);
  const int bs = 256;
  const long long grid = (threads + bs - 1) / bs;
  CSA_REQUIRE(grid < (1ll << 31), CSA_ERR_UNSUPPORTED);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#define CSA_LAUNCH_COMPRESS(TI, TO)                                                                       \
  csa_compress_kernel<TI, TO><<<static_cast<unsigned>(grid), bs, 0, st>>>(                               \
      static_cast<const TI*>(a), static_cast<const TI*>(b), static_cast<const TI*>(z), B, T, D, m,       \
      first_has_pred, S, ring_pos, out_bstride, static_cast<TO*>(out), out_fp4, out_sf, gscale)
  if (in_dtype == CSA_F32 && out_dtype == CSA_F32) CSA_LAUNCH_COMPRESS(float, float);
  else if (in_dtype == CSA_F32) CSA_LAUNCH_COMPRESS(float, __nv_bfloat16);
  else if (out_dtype == CSA_F32) CSA_LAUNCH_COMPRESS(__nv_bfloat16, float);
  else CSA_LAUNCH_COMPRESS(__nv_bfloat16, __nv_bfloat16);
#undef CSA_LAUNCH_COMPRESS
  return check_launch();
}

int hca_compress(const void* a, const void* z, int in_dtype, int B, int T, int D, int m, void* out,
                 int out_dtype, csa_stream_t stream) {
  CSA_REQUIRE(a && z && out, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(B >= 0 && T >= 0 && D > 0 && m >= 1, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(in_dtype == CSA_F32 || in_dtype == CSA_BF16, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(out_dtype == CSA_F32 || out_dtype == CSA_BF16, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(D % 8 == 0 && D <= 2048, CSA_ERR_UNSUPPORTED);
  CSA_REQUIRE(aligned16(a) && aligned16(z), CSA_ERR_ALIGNMENT);
  const int S = T / m;
  if (S == 0 || B == 0) return CSA_OK;
  const long long grid = static_cast<long long>(B) * S;
  CSA_REQUIRE(grid < (1ll << 31), CSA_ERR_UNSUPPORTED);
  const int G = D / 8;
  int RG = 256 / G;
  if (RG < 1) RG = 1;
  const int bs = G * RG;
  const size_t smem = static_cast<size_t>(RG) * 3 * D * sizeof(float);
  CSA_REQUIRE(smem <= 48 * 1024, CSA_ERR_UNSUPPORTED);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
#define CSA_LAUNCH_HCA(TI, TO)                                                                        \
  hca_compress_kernel<TI, TO><<<static_cast<unsigned>(grid), bs, smem, st>>>(                        \
      static_cast<const TI*>(a), static_cast<const TI*>(z), T, D, m, S, static_cast<TO*>(out))
  if (in_dtype == CSA_F32 && out_dtype == CSA_F32) CSA_LAUNCH_HCA(float, float);
  else if (in_dtype == CSA_F32) CSA_LAUNCH_HCA(float, __nv_bfloat16);
  else if (out_dtype == CSA_F32) CSA_LAUNCH_HCA(__nv_bfloat16, float);
  else CSA_LAUNCH_HCA(__nv_bfloat16, __nv_bfloat16);
#undef CSA_LAUNCH_HCA
  return check_launch();
}

int nvfp4_quantize(const void* x, int in_dtype, int64_t rows, int D, float gscale, uint8_t* packed,
                   uint8_t* sf, csa_stream_t stream) {
  CSA_REQUIRE(x && packed && sf, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(rows >= 0 && D > 0 && gscale > 0.f, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(in_dtype == CSA_F32 || in_dtype == CSA_BF16, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(D % 16 == 0, CSA_ERR_UNSUPPORTED);
  CSA_REQUIRE(aligned16(x) && (reinterpret_cast<uintptr_t>(packed) & 3u) == 0, CSA_ERR_ALIGNMENT);
  const long long n8 = rows * (D / 8);
  if (n8 == 0) return CSA_OK;
  const int bs = 256;
  const long long grid = (n8 + bs - 1) / bs;
  CSA_REQUIRE(grid < (1ll << 31), CSA_ERR_UNSUPPORTED);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (in_dtype == CSA_F32)
    nvfp4_quantize_kernel<float><<<static_cast<unsigned>(grid), bs, 0, st>>>(static_cast<const float*>(x), n8,
                                                                             gscale, packed, sf);
  else
    nvfp4_quantize_kernel<__nv_bfloat16><<<static_cast<unsigned>(grid), bs, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), n8, gscale, packed, sf);
  return check_launch();
}

int csa_decode_update(const void* a, const void* b, const void* z, const void* a_I, const void* b_I,
                      const void* z_I, const void* kv_raw, const void* q_I, int dtype, int B, int D, int DI, int HI,
                      int m, int W, int cap, void* carry_a, void* carry_b, void* carry_z, void* carry_aI,
                      void* carry_bI, void* carry_zI, void* ring, void* kv_c, uint8_t* k_fp4, uint8_t* k_sf,
                      uint8_t* q_fp4, uint8_t* q_sf, float gscale, const int32_t* pos, csa_stream_t stream) {
  CSA_REQUIRE(a && b && z && a_I && b_I && z_I && kv_raw && q_I && pos, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(carry_a && carry_b && carry_z && carry_aI && carry_bI && carry_zI && ring, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(kv_c && k_fp4 && k_sf && q_fp4 && q_sf, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(B >= 0 && m >= 1 && m <= 16 && W >= 1 && cap >= 1 && HI >= 1 && gscale > 0.f, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(dtype == CSA_F32 || dtype == CSA_BF16, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(D > 0 && DI > 0 && D % 16 == 0 && DI % 16 == 0, CSA_ERR_UNSUPPORTED);
  const int esz = dtype == CSA_F32 ? 4 : 2;
  const int G = D / 8, GI = DI / 8;
  // 8 elements per 16-byte copy: bf16 rows only (fp32 rows take the separate calls)
  CSA_REQUIRE(esz == 2, CSA_ERR_UNSUPPORTED);
  const int wk = (G + 31) / 32;
  const int wq = wk + 1;
  const int n8 = HI * DI / 8;
  CSA_REQUIRE(GI <= 32 && wq + (n8 + 31) / 32 <= 8, CSA_ERR_UNSUPPORTED);
  const void* rows[7] = {a, b, z, a_I, b_I, z_I, kv_raw};
  void* rings[7] = {carry_a, carry_b, carry_z, carry_aI, carry_bI, carry_zI, ring};
  for (int i = 0; i < 7; ++i) CSA_REQUIRE(aligned16(rows[i]) && aligned16(rings[i]), CSA_ERR_ALIGNMENT);
  CSA_REQUIRE(aligned16(q_I) && aligned16(kv_c) && (reinterpret_cast<uintptr_t>(k_fp4) & 3u) == 0 &&
                  (reinterpret_cast<uintptr_t>(q_fp4) & 3u) == 0,
              CSA_ERR_ALIGNMENT);
  if (B == 0) return CSA_OK;
  DecodeUpdateArgs args{};
  for (int i = 0; i < 7; ++i) {
    args.row[i] = rows[i];
    args.ring[i] = rings[i];
  }
  args.q_I = q_I;
  args.kv_c = kv_c;
  args.k_fp4 = k_fp4;
  args.k_sf = k_sf;
  args.q_fp4 = q_fp4;
  args.q_sf = q_sf;
  args.pos = pos;
  args.D = D;
  args.DI = DI;
  args.HI = HI;
  args.m = m;
  args.W = W;
  args.cap = cap;
  args.wk = wk;
  args.wq = wq;
  args.g = gscale;
  decode_update_kernel<__nv_bfloat16><<<B, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(args);
  return check_launch();
}

int csa_ring_append(const void* rows, int dtype, int B, int D, void* ring, int cap, const int32_t* pos,
                    csa_stream_t stream) {
  CSA_REQUIRE(rows && ring && pos, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(B >= 0 && D > 0 && cap > 0, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(dtype == CSA_F32 || dtype == CSA_BF16, CSA_ERR_INVALID_ARG);
  if (B == 0) return CSA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == CSA_F32)
    ring_append_kernel<float><<<B, 128, 0, st>>>(static_cast<const float*>(rows), B, D, static_cast<float*>(ring),
                                                 cap, pos);
  else
    ring_append_kernel<__nv_bfloat16><<<B, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(rows), B, D,
                                                         static_cast<__nv_bfloat16*>(ring), cap, pos);
  return check_launch();
}

int csa_state_gather(const void* src, int dtype, int B, int D, int src_cap, const int32_t* pos, int npos, int m,
                     int nrows, void* dst, int dst_cap, csa_stream_t stream) {
  CSA_REQUIRE(src && dst && pos, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(B >= 0 && npos >= 0 && D > 0 && src_cap > 0 && dst_cap > 0 && m >= 0, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(m > 0 ? dst_cap >= 2 * m : (nrows >= 1 && dst_cap >= nrows), CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(dtype == CSA_F32 || dtype == CSA_BF16, CSA_ERR_INVALID_ARG);
  CSA_REQUIRE(D % 8 == 0, CSA_ERR_UNSUPPORTED);
  CSA_REQUIRE(aligned16(src) && aligned16(dst), CSA_ERR_ALIGNMENT);
  const long long snaps = static_cast<long long>(B) * npos;
  if (snaps == 0) return CSA_OK;
  CSA_REQUIRE(snaps < (1ll << 31), CSA_ERR_UNSUPPORTED);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == CSA_F32)
    state_gather_kernel<float><<<static_cast<unsigned>(snaps), 256, 0, st>>>(
        static_cast<const float*>(src), D, src_cap, pos, npos, m, nrows, static_cast<float*>(dst), dst_cap);
  else
    state_gather_kernel<__nv_bfloat16><<<static_cast<unsigned>(snaps), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(src), D, src_cap, pos, npos, m, nrows, static_cast<__nv_bfloat16*>(dst),
        dst_cap);
  return check_launch();
}

int csa_pos_advance(int32_t* pos, int B, int delta, csa_stream_t stream) {
  CSA_REQUIRE(pos != nullptr && B >= 0, CSA_ERR_INVALID_ARG);
  if (B == 0) return CSA_OK;
  pos_advance_kernel<<<(B + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(pos, B, delta);
  return check_launch();
}

}  // extern "C"
