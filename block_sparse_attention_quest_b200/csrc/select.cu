// Group scoring with the pooled Quest bound, and top-n block selection.
//
// "Rectified Sparse Attention" (pith.science review), section "What carries
// the argument": each GQA group pools its queries and picks the same top
// blocks via Quest-style min/max descriptors; n = max(n_min, ceil(M p)) (Eq. 5,
// p read as the active ratio); the most recent block is always kept
// ("Assumptions & free parameters", n_local = 1).
//
// Score of block j for group g:
//   s_j = sum_{h in g} sum_c max(q_hc lo_jc, q_hc hi_jc).
// Because lo <= hi, max(q lo, q hi) = min(q, 0) lo + max(q, 0) hi, so the sum
// over the group's heads folds into two coefficient vectors computed once per
// group: s_j = sum_c (N_c lo_jc + P_c hi_jc) with N_c = sum_h min(q_hc, 0) and
// P_c = sum_h max(q_hc, 0). The kernel then streams the descriptors once, at
// two multiply-adds per channel.
#include "launch.h"

namespace resa {

// Sum U per-lane values over aligned segments of W lanes, transposed so that
// each round halves the number of live values: after the call lane `l` holds
// the full segment sum of value index seg_value_index<U, W>(l) in v[0].
template <int U, int W>
__device__ __forceinline__ float transpose_reduce(float (&v)[U], int lane) {
  int count = U;
#pragma unroll
  for (int m = W / 2; m >= 1; m >>= 1) {
    if (count > 1) {
      const int half = count / 2;
      const bool upper = (lane & m) != 0;
#pragma unroll
      for (int i = 0; i < U / 2; ++i) {
        if (i < half) {
          const float send = upper ? v[i] : v[i + half];
          const float keep = upper ? v[i + half] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
      }
      count = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
    }
  }
  return v[0];
}
template <int U, int W>
__device__ __forceinline__ int seg_value_index(int lane) {
  int idx = 0, count = U;
#pragma unroll
  for (int m = W / 2; m >= 1; m >>= 1) {
    if (count > 1) {
      count /= 2;
      if (lane & m) idx += count;
    }
  }
  return idx;
}

// lanes that hold a unique reduced value: the low log2(W / U) lane bits are 0
template <int U, int W>
__device__ __forceinline__ bool seg_value_owner(int lane) {
  constexpr int dup = W / U;   // lanes sharing one value
  return (lane % dup) == 0;
}

struct ScoreArgs {
  const void* q;
  const void* desc;
  float* scores;
  const void* k_new;
  const void* v_new;
  void* k;
  void* v;
  void* desc_w;
  int64_t L_max;
  int64_t len;
  int H, G, Mmax, M;
  int blocks_per_cta;
};

// Grid (chunks, H, B); 256 threads. A warp-wide load covers BPL blocks (W
// lanes each, CPL 16-byte chunks per lane per block); U loads are issued back
// to back before any arithmetic so that U * 512 bytes per warp are in flight.
template <typename T, int D>
__global__ void __launch_bounds__(256) score_kernel(ScoreArgs a) {
  constexpr int CH = Chunk<T>::N;
  constexpr int CPB = 2 * D / CH;                  // 16-byte chunks per descriptor block
  constexpr int W = CPB < 32 ? CPB : 32;           // lanes per block
  constexpr int CPL = CPB / W;                     // chunks per lane per block
  constexpr int BPL = 32 / W;                      // blocks per warp-wide load
  constexpr int U = 8;                             // loads in flight per lane
  constexpr int NW = 8;

  __shared__ float coef[2 * D];                    // [N (for lo) | P (for hi)]
  const int g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t bh = static_cast<int64_t>(b) * a.H + g;
  const int last_scored = a.M - 1;                 // block M-1 is forced, not scored
  const int j_begin = blockIdx.x * a.blocks_per_cta;
  const int j_end = min(j_begin + a.blocks_per_cta, last_scored);
  const T* dbase = static_cast<const T*>(a.desc) + bh * a.Mmax * 2 * D;
  float* sout = a.scores + bh * a.M;
  const int seg = lane / W;

  uint4 raw[U][CPL];
  auto load_batch = [&](int j0) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j0 + u * BPL + seg;
#pragma unroll
      for (int w = 0; w < CPL; ++w)
        raw[u][w] = j < j_end ? ld_stream16(dbase + static_cast<int64_t>(j) * 2 * D +
                                            ((lane % W) + w * W) * CH)
                              : make_uint4(0, 0, 0, 0);
    }
  };
  // the first descriptor loads go out before the coefficient set-up
  int j0 = j_begin + warp * U * BPL;
  if (j0 < j_end) load_batch(j0);

  const T* q = static_cast<const T*>(a.q) + (static_cast<int64_t>(b) * a.H * a.G + g * a.G) * D;
  if (tid < D) {
    float n = 0.f, p = 0.f;
    for (int h = 0; h < a.G; ++h) {
      const float x = Dt<T>::to_f(q[h * D + tid]);
      n += fminf(x, 0.f);
      p += fmaxf(x, 0.f);
    }
    coef[tid] = n;
    coef[D + tid] = p;
  }
  __syncthreads();

  // this lane's coefficients: position in the block is (lane % W) + w * W
  float cf[CPL][CH];
#pragma unroll
  for (int w = 0; w < CPL; ++w)
#pragma unroll
    for (int e = 0; e < CH; ++e) cf[w][e] = coef[((lane % W) + w * W) * CH + e];

  for (; j0 < j_end; j0 += NW * U * BPL) {
    float v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < CPL; ++w) {
        float f[CH];
        Chunk<T>::unpack(raw[u][w], f);
#pragma unroll
        for (int e = 0; e < CH; ++e) acc = fmaf(cf[w][e], f[e], acc);
      }
      v[u] = acc;
    }
    if (j0 + NW * U * BPL < j_end) load_batch(j0 + NW * U * BPL);
    transpose_reduce<U, W>(v, lane);
    if (seg_value_owner<U, W>(lane)) {
      const int u = seg_value_index<U, W>(lane);
      const int j = j0 + u * BPL + seg;
      if (j < j_end) sout[j] = v[0];
    }
  }

  // fused append of the decode token (the scoring above never reads block M-1)
  if (a.k_new != nullptr && blockIdx.x == gridDim.x - 1 && tid < D) {
    const int64_t t = a.len - 1;
    const T kn = static_cast<const T*>(a.k_new)[bh * D + tid];
    static_cast<T*>(a.k)[(bh * a.L_max + t) * D + tid] = kn;
    static_cast<T*>(a.v)[(bh * a.L_max + t) * D + tid] =
        static_cast<const T*>(a.v_new)[bh * D + tid];
    T* d = static_cast<T*>(a.desc_w) + (bh * a.Mmax + t / kBlock) * 2 * D;
    if (t % kBlock == 0) {
      d[tid] = kn;
      d[D + tid] = kn;
    } else {
      const float x = Dt<T>::to_f(kn);
      d[tid] = Dt<T>::from_f(fminf(Dt<T>::to_f(d[tid]), x));
      d[D + tid] = Dt<T>::from_f(fmaxf(Dt<T>::to_f(d[D + tid]), x));
    }
  }
}

template <typename T, int D>
static cudaError_t score_t(const Shape& s, const ScoreArgs& a0, int num_sms, cudaStream_t st) {
  ScoreArgs a = a0;
  static int occ[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (occ[dev] == 0) {
    int o = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, score_kernel<T, D>, 256, 0);
    if (e != cudaSuccess) return e;
    occ[dev] = o > 0 ? o : 1;
  }
  const int scored = a.M - 1;
  const int units = s.B * s.H;
  // one wave: every CTA resident at once, each a multiple of one warp pass
  const int slots = occ[dev] * num_sms;
  const int target = max(1, slots / units);
  int bpc = (scored + target - 1) / target;
  constexpr int BPL = 32 / ((2 * D / Chunk<T>::N) < 32 ? (2 * D / Chunk<T>::N) : 32);
  const int quantum = 8 * BPL;                     // blocks of one warp-wide U-load
  bpc = max(quantum, ((bpc + quantum - 1) / quantum) * quantum);
  a.blocks_per_cta = bpc;
  const int chunks = max(1, (scored + bpc - 1) / bpc);
  dim3 grid(chunks, s.H, s.B);
  score_kernel<T, D><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_score(const Shape& s, const void* q, const void* desc, float* scores,
                         const void* k_new, const void* v_new, void* k, void* v, void* desc_w,
                         int64_t len, int num_sms, cudaStream_t st) {
  ScoreArgs a{};
  a.q = q; a.desc = desc; a.scores = scores; a.k_new = k_new; a.v_new = v_new;
  a.k = k; a.v = v; a.desc_w = desc_w; a.L_max = s.L_max; a.len = len;
  a.H = s.H; a.G = s.G; a.Mmax = s.Mmax;
  a.M = static_cast<int>((len + kBlock - 1) / kBlock);
  if (s.bf16)
    return s.D == 128 ? score_t<__nv_bfloat16, 128>(s, a, num_sms, st)
                      : score_t<__nv_bfloat16, 64>(s, a, num_sms, st);
  return s.D == 128 ? score_t<float, 128>(s, a, num_sms, st)
                    : score_t<float, 64>(s, a, num_sms, st);
}

// ---------------------------------------------------------------------------
// top-n selection: radix select over order-preserving 32-bit keys
// ---------------------------------------------------------------------------
constexpr int kSelThreads = 1024;
constexpr int kSelSmemKeys = 40960;   // keys kept in shared memory up to this M

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (f == 0.0f) u = 0u;                          // -0 and +0 are the same score
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// exclusive prefix sum over the block (kSelThreads threads); returns the
// thread's exclusive offset, writes the block total to *total
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t x, uint32_t* warp_tot,
                                                         uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    uint32_t t = lane < nw ? warp_tot[lane] : 0u;
    uint32_t ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += y;
    }
    if (lane < nw) warp_tot[lane] = ti - t;        // exclusive warp offsets
    if (lane == 31) *total = ti;
  }
  __syncthreads();
  const uint32_t r = warp_tot[warp] + inc - x;
  __syncthreads();
  return r;
}

// Grid (H, B). Keeps block M-1 and the n-1 best of blocks 0 .. M-2; among
// equal scores the lower index wins. Output ascending.
//
// Radix select over the keys' offsets from their minimum: the digits start at
// the highest bit in which the keys differ, so the first histogram is spread
// over its 256 bins even when every score has the same sign and exponent, and
// plain shared-memory atomics see little contention.
__global__ void __launch_bounds__(kSelThreads) select_kernel(const float* __restrict__ scores,
                                                             int32_t* __restrict__ sel, int H,
                                                             int M, int n, int keys_in_smem) {
  extern __shared__ uint32_t skeys[];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t red_min[32], red_max[32];
  __shared__ uint32_t s_prefix, s_remaining, s_total, s_kmin, s_kmax, s_done;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t bh = static_cast<int64_t>(blockIdx.y) * H + blockIdx.x;
  const float* s = scores + bh * M;
  int32_t* out = sel + bh * n;
  const int Mo = M - 1;                            // candidates: blocks 0 .. M-2
  const int need = n - 1;                          // how many of them to keep

  if (need >= Mo) {                                // every block is selected
    for (int j = tid; j < M; j += blockDim.x) out[j] = j;
    return;
  }
  if (need <= 0) {
    if (tid == 0) out[0] = M - 1;
    return;
  }
  auto key_at = [&](int j) -> uint32_t { return keys_in_smem ? skeys[j] : score_key(s[j]); };
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int j0 = tid; j0 < Mo; j0 += 8 * kSelThreads) {
    float x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u * kSelThreads;
      x[u] = j < Mo ? __ldcg(s + j) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u * kSelThreads;
      if (j < Mo) {
        const uint32_t k = score_key(x[u]);
        if (keys_in_smem) skeys[j] = k;
        kmin = min(kmin, k);
        kmax = max(kmax, k);
      }
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (lane == 0) { red_min[warp] = kmin; red_max[warp] = kmax; }
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    uint32_t a = lane < nw ? red_min[lane] : 0xffffffffu;
    uint32_t b = lane < nw ? red_max[lane] : 0u;
    a = __reduce_min_sync(0xffffffffu, a);
    b = __reduce_max_sync(0xffffffffu, b);
    if (lane == 0) {
      s_kmin = a; s_kmax = b;
      s_prefix = 0u; s_remaining = static_cast<uint32_t>(need); s_done = 0u;
    }
  }
  __syncthreads();
  const uint32_t base = s_kmin;
  const uint32_t range = s_kmax - base;
  // radix passes over rel = key - base, from the top differing bit down
  int top = 32 - __clz(range);                     // bits of rel that can differ
  while (top > 0) {
    const int shift = top > 8 ? top - 8 : 0;
    const int width = top - shift;
    if (tid < 256) hist[tid] = 0u;
    __syncthreads();
    const uint32_t prefix = s_prefix;              // fixed bits above `top`
    const uint32_t hi_mask = top >= 32 ? 0u : ~((1u << top) - 1u);
    for (int j = tid; j < Mo; j += blockDim.x) {
      const uint32_t rel = key_at(j) - base;
      if ((rel & hi_mask) == prefix) atomicAdd(&hist[(rel >> shift) & ((1u << width) - 1u)], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns bins 255-8l .. 248-8l, scanned from the top
      uint32_t c[8], local = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) { c[i] = hist[255 - 8 * lane - i]; local += c[i]; }
      uint32_t inc = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
      }
      const uint32_t before = inc - local;
      const uint32_t rem = s_remaining;
      if (before < rem && rem <= inc) {
        uint32_t acc = before;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (acc < rem && rem <= acc + c[i]) {
            const uint32_t digit = static_cast<uint32_t>(255 - 8 * lane - i);
            s_prefix = prefix | (digit << shift);
            s_remaining = rem - acc;
            // the whole bin is needed: every key at or above its floor is kept
            if (rem - acc == c[i]) s_done = 1u;
          }
          acc += c[i];
        }
      }
    }
    __syncthreads();
    top = s_done ? 0 : shift;
  }
  const uint32_t T = s_prefix;                     // rel threshold
  const bool whole_bin = s_done != 0u;
  const uint32_t need_eq = s_remaining;            // rel == T keys to take, lowest index first

  const int per = (Mo + blockDim.x - 1) / blockDim.x;
  const int j0 = min(Mo, tid * per), j1 = min(Mo, j0 + per);
  uint32_t n_sel = 0, seen = 0, n_eq = 0;
  if (whole_bin) {
    for (int j = j0; j < j1; ++j) n_sel += (key_at(j) - base) >= T;
  } else {
    for (int j = j0; j < j1; ++j) n_eq += (key_at(j) - base) == T;
    seen = block_exclusive_scan(n_eq, warp_tot, &s_total);
    const uint32_t eq_before = seen;
    for (int j = j0; j < j1; ++j) {
      const uint32_t rel = key_at(j) - base;
      if (rel > T) ++n_sel;
      else if (rel == T) { if (seen < need_eq) ++n_sel; ++seen; }
    }
    seen = eq_before;
  }
  uint32_t pos = block_exclusive_scan(n_sel, warp_tot, &s_total);
  for (int j = j0; j < j1; ++j) {
    const uint32_t rel = key_at(j) - base;
    bool take;
    if (whole_bin) {
      take = rel >= T;
    } else {
      take = rel > T;
      if (rel == T) { take = seen < need_eq; ++seen; }
    }
    if (take) out[pos++] = j;
  }
  if (tid == 0) out[need] = M - 1;
}

cudaError_t launch_select(const Shape& s, const float* scores, int32_t* sel, int M, int n,
                          cudaStream_t st) {
  const int in_smem = M <= kSelSmemKeys ? 1 : 0;
  const size_t smem = in_smem ? static_cast<size_t>(M) * sizeof(uint32_t) : 0;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSelSmemKeys * static_cast<int>(sizeof(uint32_t)));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  dim3 grid(s.H, s.B);
  select_kernel<<<grid, kSelThreads, smem, st>>>(scores, sel, s.H, M, n, in_smem);
  return cudaGetLastError();
}

}  // namespace resa
