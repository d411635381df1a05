// Split-KV block-sparse attention and the log-sum-exp merge of the splits.
//
// "Rectified Sparse Attention" (pith.science review), section "What carries
// the argument": all heads of a GQA group read the same selected key blocks;
// Eq. 2 (minor comment 3) masks token k through its block floor(k / b). The
// split/merge schedule follows Flash-Decoding (reference list of the same
// page): each CTA reduces a contiguous slice of the group's block list to an
// unnormalised (max, sum, accumulator) triple and a second kernel merges them.
//
// One CTA serves every query head of one KV group for one query row and one
// slice of blocks, so a gathered K/V block is fetched from HBM once and used
// by all G heads.
//
// bf16 path: each warp owns a private ring of STAGES tiles; a tile is the K
// and V rows of one 16-token block, brought in by 2-D TMA tensor copies
// (stream_bf16 in attend_core.cuh).
//
// fp32 path: the same schedule on CUDA cores with plain loads (no tensor
// cores: fp32 inputs must keep fp32 products).
#include "attend_core.cuh"

namespace resa {

// Query rows of batch row b in use (all R unless per-row windows are given).
__device__ __forceinline__ int query_rows(const AttnK& a, int b) {
  return row_window(a.windows, a.R, b);
}
// Tokens visible to query row r of batch row b: the row's last query row
// sees the whole row.
__device__ __forceinline__ int64_t query_len(const AttnK& a, int b, int r) {
  if (a.lens == nullptr && a.windows == nullptr) return a.len0 + r;
  return row_len(a.lens, a.len0 + a.R - 1, b) - query_rows(a, b) + 1 + r;
}
// query rows past the batch row's count, and batch rows shorter than their
// count (or with count 0), are skipped (variable lengths and windows only)
__device__ __forceinline__ bool row_skipped(const AttnK& a, int b, int r) {
  if (a.lens == nullptr && a.windows == nullptr) return false;
  const int w = query_rows(a, b);
  return r >= w || row_len(a.lens, a.len0 + a.R - 1, b) < w;
}

constexpr int kIdCache = 1024;   // block ids of one CTA kept in shared memory

__device__ __forceinline__ void split_range(const AttnK& a, int s, int64_t len_r, int& i0,
                                            int& i1) {
  const int n = a.sel ? (a.lens ? num_selected_dev(len_r, a.r, a.n_min) : a.n_sel)
                     : static_cast<int>((len_r + kBlock - 1) / kBlock);
  i0 = static_cast<int>(static_cast<int64_t>(s) * n / a.S);
  i1 = static_cast<int>(static_cast<int64_t>(s + 1) * n / a.S);
}

// Block ids of this CTA's slice of the list, cached in shared memory when the
// slice fits (always, for the sizes one GPU serves); dense rows need none.
struct IdCache {
  const int32_t* sel;   // this (b, g)'s list, or nullptr for dense
  const int* ids;       // shared copy of sel[i0 .. i1) or nullptr
  int i0;
  __device__ __forceinline__ int at(int i) const {
    if (sel == nullptr) return i;
    return ids ? ids[i - i0] : sel[i];
  }
};

__device__ __forceinline__ IdCache load_ids(const int32_t* selp, int i0, int i1, int* smem_ids) {
  IdCache c{selp, nullptr, i0};
  if (selp != nullptr && i1 - i0 <= kIdCache) {
    for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) smem_ids[i - i0] = selp[i];
    c.ids = smem_ids;
  }
  __syncthreads();
  return c;
}

// ---------------------------------------------------------------------- bf16
template <int D, int NW, int STAGES>
__global__ void __launch_bounds__(NW * 32) attend_bf16_kernel(const __grid_constant__ CUtensorMap tmK,
                                                              const __grid_constant__ CUtensorMap tmV,
                                                              AttnK a) {
  constexpr int KT = D / 16;                 // k-steps of the QK product, m-tiles of PV
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[NW][STAGES];
  __shared__ int ids_smem[kIdCache];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));

  const int s_idx = blockIdx.x, g = blockIdx.y, br = blockIdx.z;
  const int b = br / a.R, r = br % a.R;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (row_skipped(a, b, r)) return;
  const int64_t len_r = query_len(a, b, r);
  int i0, i1;
  split_range(a, s_idx, len_r, i0, i1);
  const int span = i1 - i0;
  const int my_count = span > warp ? (span - warp + NW - 1) / NW : 0;
  const int32_t* selp = a.sel ? a.sel + (static_cast<int64_t>(b) * a.H + g) * a.n_sel : nullptr;
  const int64_t row_base = (static_cast<int64_t>(b) * a.H + g) * a.L_max;
  if (lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
#pragma unroll
    for (int st = 0; st < STAGES; ++st) mbar_init(&bars[warp][st], 1);
    fence_mbar_init();
  }
  __syncwarp();

  uint32_t qb[KT][2];
  load_q_frags<D>(static_cast<const __nv_bfloat16*>(a.q) +
                      (static_cast<int64_t>(br) * a.Hq + g * a.G) * D, a.G, qb);

  // Everything above may run before the kernel that produced the block list
  // has finished (programmatic dependent launch); block ids are read after.
  grid_dependency_wait();
  const IdCache ids = load_ids(selp, i0, i1, ids_smem);

  const int m_r = static_cast<int>((len_r + kBlock - 1) / kBlock);
  // block id of this warp's k-th block; ids outside [0, m_r) come back as -1
  auto block_of = [&](int k) -> int {
    const int j = ids.at(i0 + warp + k * NW);
    return (j >= 0 && j < m_r) ? j : -1;
  };
  float o[KT][4];
  float m0, m1, l0, l1;
  const bool ok = stream_bf16<D, NW, STAGES>(&tmK, &tmV, tiles, bars, block_of, my_count, row_base,
                                             len_r, qb, a.scale_log2, a.ctrl, o, m0, m1, l0, l1);
  // The next kernel in the stream may launch once every CTA has streamed its
  // blocks (whatever it reads from this kernel it reads after its own
  // dependency wait); launched earlier its prologue would compete with the
  // stream, launched here it overlaps the merge tail.
  grid_launch_dependents();
  finish_bf16<D, NW, STAGES>(a, tiles, ok, o, m0, m1, l0, l1, br, g, s_idx);
}

// ---------------------------------------------------------------------- fp32
template <int D, int NW>
__global__ void __launch_bounds__(NW * 32) attend_f32_kernel(AttnK a) {
  constexpr int P = D + 1;                    // padded row (conflict-free column reads)
  constexpr int CPL = D / 32;                 // output channels per lane
  extern __shared__ float smf[];
  float* sq = smf;                            // [8][D]
  float* tiles = smf + 8 * D;                 // [NW][2][16][P]
  const int s_idx = blockIdx.x, g = blockIdx.y, br = blockIdx.z;
  const int b = br / a.R, r = br % a.R;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (row_skipped(a, b, r)) return;
  const int64_t len_r = query_len(a, b, r);
  const float* qrow = static_cast<const float*>(a.q) + (static_cast<int64_t>(br) * a.Hq + g * a.G) * D;
  for (int i = threadIdx.x; i < a.G * D; i += NW * 32) sq[i] = qrow[i];
  __syncthreads();
  int i0, i1;
  split_range(a, s_idx, len_r, i0, i1);
  const int32_t* selp = a.sel ? a.sel + (static_cast<int64_t>(b) * a.H + g) * a.n_sel : nullptr;
  const int64_t row_base = (static_cast<int64_t>(b) * a.H + g) * a.L_max;
  __shared__ int ids_smem[kIdCache];
  grid_dependency_wait();
  const IdCache ids = load_ids(selp, i0, i1, ids_smem);
  const float* kc = static_cast<const float*>(a.k);
  const float* vc = static_cast<const float*>(a.v);
  float* Ks = tiles + warp * 2 * 16 * P;
  float* Vs = Ks + 16 * P;

  float m[8], l[8], acc[8][CPL];
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) acc[h][i] = 0.f;
  }
  const int t = lane & 15, half = lane >> 4;
  const int m_r = static_cast<int>((len_r + kBlock - 1) / kBlock);
  for (int i = i0 + warp; i < i1; i += NW) {
    const int j = ids.at(i);
    if (j < 0 || j >= m_r) {                   // skip the block, report it
      if (lane == 0) raise_error(a.ctrl, kErrBadIndex);
      continue;
    }
    const float* kb = kc + (row_base + static_cast<int64_t>(j) * kBlock) * D;
    const float* vb = vc + (row_base + static_cast<int64_t>(j) * kBlock) * D;
    __syncwarp();
    const int valid_rows = static_cast<int>(len_r - static_cast<int64_t>(j) * kBlock);
    for (int e = lane; e < 16 * D / 4; e += 32) {
      const int row = e / (D / 4), c4 = (e % (D / 4)) * 4;
      // slots past the end of the cache are never read (their weight is 0)
      const bool ok_row = row < valid_rows;
      const float4 kv = ok_row ? *reinterpret_cast<const float4*>(kb + row * D + c4)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 vv = ok_row ? *reinterpret_cast<const float4*>(vb + row * D + c4)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
      Ks[row * P + c4] = kv.x; Ks[row * P + c4 + 1] = kv.y;
      Ks[row * P + c4 + 2] = kv.z; Ks[row * P + c4 + 3] = kv.w;
      Vs[row * P + c4] = vv.x; Vs[row * P + c4 + 1] = vv.y;
      Vs[row * P + c4 + 2] = vv.z; Vs[row * P + c4 + 3] = vv.w;
    }
    __syncwarp();
    const bool valid = static_cast<int64_t>(j) * kBlock + t < len_r;
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      if (h < a.G) {
        float part = 0.f;
#pragma unroll 8
        for (int c = half * (D / 2); c < (half + 1) * (D / 2); ++c)
          part = fmaf(sq[h * D + c], Ks[t * P + c], part);
        part += __shfl_xor_sync(0xffffffffu, part, 16);
        const float z = valid ? part * a.scale_log2 : -INFINITY;
        float mx = z;
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float mn = fmaxf(m[h], mx);
        const float al = exp2f(m[h] - mn);
        const float p = exp2f(z - mn);
        float ps = p;
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        l[h] = fmaf(l[h], al, ps);
        m[h] = mn;
#pragma unroll
        for (int i = 0; i < CPL; ++i) acc[h][i] *= al;
#pragma unroll
        for (int tt = 0; tt < 16; ++tt) {
          const float pt = __shfl_sync(0xffffffffu, p, tt);
#pragma unroll
          for (int i = 0; i < CPL; ++i) acc[h][i] = fmaf(pt, Vs[tt * P + lane + 32 * i], acc[h][i]);
        }
      }
    }
  }
  grid_launch_dependents();                   // see the bf16 kernel
  __syncthreads();
  float* sm = tiles;                       // reuse: needs merge_floats(D, NW) floats
  constexpr int OR = merge_row(D);
  float* sm_o = sm;
  float* sm_m = sm + NW * 8 * OR;
  float* sm_l = sm_m + NW * 8;
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    if (h < a.G) {
      if (lane == 0) { sm_m[warp * 8 + h] = m[h]; sm_l[warp * 8 + h] = l[h]; }
#pragma unroll
      for (int i = 0; i < CPL; ++i) sm_o[(warp * 8 + h) * OR + lane + 32 * i] = acc[h][i];
    }
  }
  __syncthreads();
  cta_finish<float, D, NW>(a, sm, br, g, s_idx);
}

// ---------------------------------------------------------------------- launch
constexpr int kNW = 8;        // warps per CTA (one CTA per SM for bf16)
constexpr int kStages = 2;    // tiles in flight per warp (3: no faster, more shared memory)

template <int D>
static cudaError_t attend_bf16_t(const Shape& s, const AttnK& k, const AttnArgs& a,
                                 cudaStream_t st) {
  using Cfg = Bf16Cfg<D, kNW, kStages>;
  static std::atomic<bool> attr_set[64];   // per device; launches may come from several host threads
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(attend_bf16_kernel<D, kNW, kStages>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.S, s.H, s.B * a.R);
  cfg.blockDim = dim3(kNW * 32);
  cfg.dynamicSmemBytes = Cfg::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, attend_bf16_kernel<D, kNW, kStages>, *a.tm_k, *a.tm_v, k);
}

template <int D>
static cudaError_t attend_f32_t(const Shape& s, const AttnK& k, const AttnArgs& a,
                                cudaStream_t st) {
  const size_t tiles = static_cast<size_t>(kNW) * 2 * 16 * (D + 1);
  const size_t merge = static_cast<size_t>(merge_floats(D, kNW));
  const size_t smem = (8 * D + (tiles > merge ? tiles : merge)) * sizeof(float);
  static std::atomic<bool> attr_set[64];   // per device; launches may come from several host threads
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(attend_f32_kernel<D, kNW>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.S, s.H, s.B * a.R);
  cfg.blockDim = dim3(kNW * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, attend_f32_kernel<D, kNW>, k);
}

int attend_ctas_per_sm(const Shape& s) { return s.bf16 ? 1 : 2; }

cudaError_t launch_attend(const Shape& s, const AttnArgs& a, cudaStream_t st) {
  AttnK k{};
  k.q = a.q; k.sel = a.sel; k.part_o = a.part_o; k.part_ml = a.part_ml; k.ctrl = a.ctrl;
  k.counters = a.counters; k.out = a.out; k.lse = a.lse;
  k.k = a.k; k.v = a.v; k.len0 = a.len0; k.L_max = s.L_max; k.R = a.R; k.Hq = s.Hq; k.H = s.H;
  k.G = s.G; k.n_sel = a.n_sel; k.S = a.S;
  k.lens = a.lens; k.windows = a.windows; k.r = a.r; k.n_min = a.n_min;
  k.scale_log2 = a.scale * 1.4426950408889634f;
  if (s.bf16) return s.D == 128 ? attend_bf16_t<128>(s, k, a, st) : attend_bf16_t<64>(s, k, a, st);
  return s.D == 128 ? attend_f32_t<128>(s, k, a, st) : attend_f32_t<64>(s, k, a, st);
}

}  // namespace resa
