// Quest block descriptors: full build, incremental append, and the refresh
// after a rectification.
//
// "Rectified Sparse Attention" (pith.science review), section "What carries
// the argument": blocks are ranked through Quest-style per-channel min/max
// block descriptors; rectification replaces KV entries and updates the block
// statistics. Block size b = 16 ("Assumptions & free parameters").
//
// All three kernels are bound by HBM traffic of the keys they read; the
// min/max of bf16 values is exact in float and converts back exactly.
#include <atomic>

#include "launch.h"

namespace resa {

// One warp per (b, h, block). Lane `lane` owns 16-byte chunk lane % CPR of a
// row and rows lane / CPR, lane / CPR + TPP, ...; lanes that own the same
// chunk are then combined with xor-shuffles.
template <typename T, int D>
__global__ void __launch_bounds__(256) build_desc_kernel(const T* __restrict__ k,
                                                         T* __restrict__ desc, int64_t L_max,
                                                         int Mmax, int M, int64_t len,
                                                         int64_t total, const int32_t* lens,
                                                         int H) {
  constexpr int CH = Chunk<T>::N;
  constexpr int CPR = D / CH;                 // 16-byte chunks per token row
  constexpr int TPP = 32 / CPR;               // rows covered by one warp-wide load
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= total) return;
  const int64_t bh = wid / M;
  const int j = static_cast<int>(wid % M);
  const int64_t len_b = row_len(lens, len, static_cast<int>(bh / H));
  if (static_cast<int64_t>(j) * kBlock >= len_b) return;     // past this row's length
  const int valid = static_cast<int>(len_b - static_cast<int64_t>(j) * kBlock < kBlock ? len_b - static_cast<int64_t>(j) * kBlock : kBlock);
  const int chunk = lane % CPR;
  const int r0 = lane / CPR;
  const T* base = k + (bh * L_max + static_cast<int64_t>(j) * kBlock) * D + chunk * CH;

  float mn[CH], mx[CH];
#pragma unroll
  for (int e = 0; e < CH; ++e) { mn[e] = INFINITY; mx[e] = -INFINITY; }
  uint4 raw[kBlock / TPP];
#pragma unroll
  for (int i = 0; i < kBlock / TPP; ++i) {
    const int t = r0 + i * TPP;
    raw[i] = t < valid ? ld_stream16(base + static_cast<int64_t>(t) * D) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int i = 0; i < kBlock / TPP; ++i) {
    const int t = r0 + i * TPP;
    if (t < valid) {
      float f[CH];
      Chunk<T>::unpack(raw[i], f);
#pragma unroll
      for (int e = 0; e < CH; ++e) { mn[e] = fminf(mn[e], f[e]); mx[e] = fmaxf(mx[e], f[e]); }
    }
  }
#pragma unroll
  for (int m = CPR; m < 32; m <<= 1) {
#pragma unroll
    for (int e = 0; e < CH; ++e) {
      mn[e] = fminf(mn[e], __shfl_xor_sync(0xffffffffu, mn[e], m));
      mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], m));
    }
  }
  if (lane < CPR) {
    T* d = desc + (bh * Mmax + j) * 2 * D + chunk * CH;
    *reinterpret_cast<uint4*>(d) = Chunk<T>::pack(mn);
    *reinterpret_cast<uint4*>(d + D) = Chunk<T>::pack(mx);
  }
}

// Decode-time append: token len-1 is written to the cache and merged into the
// descriptor of its block (or opens it). Grid (H, B), D threads.
template <typename T>
__global__ void append_kernel(const T* __restrict__ k_new, const T* __restrict__ v_new,
                              T* __restrict__ k, T* __restrict__ v, T* __restrict__ desc, int H,
                              int D, int64_t L_max, int Mmax, int64_t len, const int32_t* lens) {
  const int c = threadIdx.x;
  const int64_t bh = static_cast<int64_t>(blockIdx.y) * H + blockIdx.x;
  const int64_t t = row_len(lens, len, blockIdx.y) - 1;
  const T kn = k_new[bh * D + c];
  k[(bh * L_max + t) * D + c] = kn;
  v[(bh * L_max + t) * D + c] = v_new[bh * D + c];
  if (desc) {
    T* d = desc + (bh * Mmax + t / kBlock) * 2 * D;
    if (t % kBlock == 0) {
      d[c] = kn;
      d[D + c] = kn;
    } else {
      const float x = Dt<T>::to_f(kn);
      d[c] = Dt<T>::from_f(fminf(Dt<T>::to_f(d[c]), x));
      d[D + c] = Dt<T>::from_f(fmaxf(Dt<T>::to_f(d[D + c]), x));
    }
  }
}

// Rectify write + refresh: grid (blocks touched, H, B), D threads. The CTA of
// block j writes the new K/V rows of that block (slots >= len - f), then
// recomputes the block's min/max over all its valid tokens.
template <typename T>
__global__ void rectify_write_kernel(const T* __restrict__ k_f, const T* __restrict__ v_f,
                                     T* __restrict__ k, T* __restrict__ v, T* __restrict__ desc,
                                     int H, int D, int64_t L_max, int Mmax, int64_t len, int f,
                                     const int32_t* lens, const int32_t* windows, Ctrl* ctrl) {
  // the attention over the rectified rows may launch now: its CTAs wait for
  // this grid before reading any row written here
  grid_launch_dependents();
  const int c = threadIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t bh = static_cast<int64_t>(b) * H + h;
  if (blockIdx.x == 0 && h == 0 && c == 0 &&
      (row_len_bad(lens, len, b) || row_window_bad(windows, f, b)))
    raise_error(ctrl, kErrBadIndex);
  len = row_len(lens, len, b);
  const int w = row_window(windows, f, b);  // this row's window (rows w .. f-1 of k_f unused)
  if (w == 0 || len < w) return;            // not rectified: left alone
  const int64_t t_first = len - w;
  const int64_t j = t_first / kBlock + blockIdx.x;
  if (j * kBlock >= len) return;           // this row touches fewer blocks
  const int64_t t0 = j * kBlock;
  const int64_t t1 = t0 + kBlock < len ? t0 + kBlock : len;
  // every load of the block is issued before the first store
  T kv[kBlock], vv[kBlock];
#pragma unroll
  for (int i = 0; i < kBlock; ++i) {
    const int64_t t = t0 + i;
    if (t >= t1) continue;
    if (t >= t_first) {
      const int64_t src = ((static_cast<int64_t>(b) * f + (t - t_first)) * H + h) * D + c;
      kv[i] = k_f[src];
      vv[i] = v_f[src];
    } else {
      kv[i] = k[(bh * L_max + t) * D + c];
    }
  }
  float mn = INFINITY, mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < kBlock; ++i) {
    const int64_t t = t0 + i;
    if (t >= t1) continue;
    if (t >= t_first) {
      k[(bh * L_max + t) * D + c] = kv[i];
      v[(bh * L_max + t) * D + c] = vv[i];
    }
    const float x = Dt<T>::to_f(kv[i]);
    mn = fminf(mn, x);
    mx = fmaxf(mx, x);
  }
  T* d = desc + (bh * Mmax + j) * 2 * D;
  d[c] = Dt<T>::from_f(mn);
  d[D + c] = Dt<T>::from_f(mx);
}

template <typename T, int D>
static cudaError_t build_desc_t(const Shape& s, const void* k, void* desc, int64_t len,
                                cudaStream_t st, const int32_t* lens) {
  const int M = static_cast<int>((len + kBlock - 1) / kBlock);
  const int64_t total = static_cast<int64_t>(s.B) * s.H * M;
  const int threads = 256;
  const int64_t grid = (total * 32 + threads - 1) / threads;
  build_desc_kernel<T, D><<<static_cast<unsigned>(grid), threads, 0, st>>>(
      static_cast<const T*>(k), static_cast<T*>(desc), s.L_max, s.Mmax, M, len, total, lens, s.H);
  return cudaGetLastError();
}

cudaError_t launch_build_desc(const Shape& s, const void* k, void* desc, int64_t len,
                              cudaStream_t st, const int32_t* lens) {
  if (s.bf16) {
    return s.D == 128 ? build_desc_t<__nv_bfloat16, 128>(s, k, desc, len, st, lens)
                      : build_desc_t<__nv_bfloat16, 64>(s, k, desc, len, st, lens);
  }
  return s.D == 128 ? build_desc_t<float, 128>(s, k, desc, len, st, lens)
                    : build_desc_t<float, 64>(s, k, desc, len, st, lens);
}

cudaError_t launch_append(const Shape& s, const void* k_new, const void* v_new, void* k, void* v,
                          void* desc, int64_t len, cudaStream_t st, const int32_t* lens) {
  dim3 grid(s.H, s.B);
  if (s.bf16) {
    using T = __nv_bfloat16;
    append_kernel<T><<<grid, s.D, 0, st>>>(static_cast<const T*>(k_new),
                                           static_cast<const T*>(v_new), static_cast<T*>(k),
                                           static_cast<T*>(v), static_cast<T*>(desc), s.H, s.D,
                                           s.L_max, s.Mmax, len, lens);
  } else {
    append_kernel<float><<<grid, s.D, 0, st>>>(
        static_cast<const float*>(k_new), static_cast<const float*>(v_new),
        static_cast<float*>(k), static_cast<float*>(v), static_cast<float*>(desc), s.H, s.D,
        s.L_max, s.Mmax, len, lens);
  }
  return cudaGetLastError();
}

cudaError_t launch_rectify_write(const Shape& s, const void* k_f, const void* v_f, void* k, void* v,
                                 void* desc, int64_t len, int f, cudaStream_t st,
                                 const int32_t* lens, const int32_t* windows, Ctrl* ctrl) {
  // blocks touched by f slots: at most f/16 + 2 (the bound covers every row)
  const int64_t j0 = (len - f) / kBlock;
  const int64_t M = (len + kBlock - 1) / kBlock;
  const int64_t touched = (lens || windows) ? f / kBlock + 2 : M - j0;
  dim3 grid(static_cast<unsigned>(touched), s.H, s.B);
  // The attention over the rectified rows, launched next, takes nearly all
  // of an SM's shared memory and may start while this grid runs: with the
  // same (maximal) shared-memory carveout its CTAs can start on the SMs this
  // grid occupies instead of waiting for them to drain.
  static std::atomic<bool> carveout_set[64][2];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!carveout_set[dev][s.bf16]) {
    cudaError_t e = s.bf16 ? cudaFuncSetAttribute(rectify_write_kernel<__nv_bfloat16>,
                                                  cudaFuncAttributePreferredSharedMemoryCarveout,
                                                  cudaSharedmemCarveoutMaxShared)
                           : cudaFuncSetAttribute(rectify_write_kernel<float>,
                                                  cudaFuncAttributePreferredSharedMemoryCarveout,
                                                  cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    carveout_set[dev][s.bf16] = true;
  }
  if (s.bf16) {
    using T = __nv_bfloat16;
    rectify_write_kernel<T><<<grid, s.D, 0, st>>>(
        static_cast<const T*>(k_f), static_cast<const T*>(v_f), static_cast<T*>(k),
        static_cast<T*>(v), static_cast<T*>(desc), s.H, s.D, s.L_max, s.Mmax, len, f, lens,
        windows, ctrl);
  } else {
    rectify_write_kernel<float><<<grid, s.D, 0, st>>>(
        static_cast<const float*>(k_f), static_cast<const float*>(v_f), static_cast<float*>(k),
        static_cast<float*>(v), static_cast<float*>(desc), s.H, s.D, s.L_max, s.Mmax, len, f, lens,
        windows, ctrl);
  }
  return cudaGetLastError();
}

// Failure-detection check: one thread runs the bounded counter wait of the
// one-launch decode kernel's group barrier on a caller's flag.
__global__ void wait_check_kernel(const int* flag, int target, unsigned long long limit_ns,
                                  Ctrl* ctrl) {
  if (threadIdx.x == 0) (void)wait_count_bounded(flag, target, limit_ns, ctrl);
}

cudaError_t launch_wait_check(const int* flag, int target, unsigned long long limit_ns,
                              Ctrl* ctrl, cudaStream_t st) {
  wait_check_kernel<<<1, 32, 0, st>>>(flag, target, limit_ns, ctrl);
  return cudaGetLastError();
}

}  // namespace resa
