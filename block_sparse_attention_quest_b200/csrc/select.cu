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
#include "select_core.cuh"

namespace resa {

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
  int64_t len;                // cache length (with lens: the bound on every row's)
  const int32_t* lens;        // optional per-row lengths [B]
  Ctrl* ctrl;
  int H, G, Mmax, M;          // M: blocks of len, the row stride of scores
  int blocks_per_cta;
};

// 16-byte descriptor loads in flight per lane. Four (rather than eight or
// sixteen) keep the kernel's registers low, so more CTAs stay resident and
// the one-wave grid is larger; measured back to back per decode call: 128K
// 28.8 -> 28.1 us, 256K 50.1 -> 45.9 us (two and one loads: slower again).
constexpr int kScoreLoads = 4;

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
  constexpr int U = kScoreLoads;                   // loads in flight per lane
  constexpr int NW = 8;

  __shared__ float coef[2 * D];                    // [N (for lo) | P (for hi)]
  const int g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t bh = static_cast<int64_t>(b) * a.H + g;
  const T* dbase = static_cast<const T*>(a.desc) + bh * a.Mmax * 2 * D;
  // Launched as a programmatic dependent of whatever precedes it in the
  // stream (q, the cache and the descriptors may come from there): nothing is
  // read before the wait. The start of this CTA's descriptor chunk (for the
  // length bound) is only prefetched into L2, which overlaps its HBM fetch with
  // the previous kernel's tail; the loads after the wait see that kernel's
  // writes. At most kPrefetchBytes per CTA: a larger prefetch delays the
  // previous kernel's own tail (its merge round trips queue behind it).
  {
    constexpr int64_t kPrefetchBytes = 80 * 1024;
    const int jb = blockIdx.x * a.blocks_per_cta;
    const int je = min(jb + a.blocks_per_cta, a.M - 1);
    const char* c0 = reinterpret_cast<const char*>(dbase + static_cast<int64_t>(jb) * 2 * D);
    const int64_t bytes = min(static_cast<int64_t>(max(je - jb, 0)) * 2 * D * sizeof(T),
                              kPrefetchBytes);
    for (int64_t off = static_cast<int64_t>(tid) * 128; off < bytes; off += 256 * 128)
      prefetch_l2(c0 + off);
  }
  grid_dependency_wait();
  grid_launch_dependents();
  const int64_t len_b = row_len(a.lens, a.len, b);
  if (a.lens != nullptr && blockIdx.x == 0 && g == 0 && tid == 0 && row_len_bad(a.lens, a.len, b))
    raise_error(a.ctrl, kErrBadIndex);
  const int last_scored = static_cast<int>((len_b + kBlock - 1) / kBlock) - 1;  // block M-1 is forced, not scored
  const int j_begin = blockIdx.x * a.blocks_per_cta;
  const int j_end = min(j_begin + a.blocks_per_cta, last_scored);
  float* sout = a.scores + bh * a.M;
  const int seg = lane / W;

  // the group's query values go out first: the coefficients need them before
  // any descriptor can be used, and behind the descriptor stream they would
  // wait for most of it
  const T* q = static_cast<const T*>(a.q) + (static_cast<int64_t>(b) * a.H * a.G + g * a.G) * D;
  float qv[8];
  if (tid < D) {
#pragma unroll
    for (int h = 0; h < 8; ++h) qv[h] = h < a.G ? Dt<T>::to_f(q[h * D + tid]) : 0.f;
  }
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
  int j0 = j_begin + warp * U * BPL;
  if (j0 < j_end) load_batch(j0);

  if (tid < D) {
    float n = 0.f, p = 0.f;
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      n += fminf(qv[h], 0.f);
      p += fmaxf(qv[h], 0.f);
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
    const int64_t t = len_b - 1;
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
  static std::atomic<int> occ[64];         // per device; launches may come from several host threads
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
  const int quantum = kScoreLoads * BPL;           // blocks of one warp-wide U-load
  bpc = max(quantum, ((bpc + quantum - 1) / quantum) * quantum);
  a.blocks_per_cta = bpc;
  const int chunks = max(1, (scored + bpc - 1) / bpc);
  dim3 grid(chunks, s.H, s.B);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, score_kernel<T, D>, a);
}

cudaError_t launch_score(const Shape& s, const void* q, const void* desc, float* scores,
                         const void* k_new, const void* v_new, void* k, void* v, void* desc_w,
                         int64_t len, int num_sms, cudaStream_t st, const int32_t* lens,
                         Ctrl* ctrl) {
  ScoreArgs a{};
  a.lens = lens; a.ctrl = ctrl;
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
constexpr int kSelMaxM = 262144;      // largest block count a selection accepts
// Per-row budget for variable lengths: the row's own block count M and
// Eq. 5 budget n (both at most the shared ones); the list keeps the shared
// stride and its unused tail is set to -1.
struct SelRows {
  const int32_t* lens;   // nullptr: every row has the shared length
  int64_t len;           // bound on the row lengths
  double r;
  int n_min;
};

__device__ __forceinline__ void row_budget(const SelRows& rl, int b, int& M, int& n, int32_t* out) {
  const int stride = n;
  const int64_t lb = row_len(rl.lens, rl.len, b);
  M = static_cast<int>((lb + kBlock - 1) / kBlock);
  n = num_selected_dev(lb, rl.r, rl.n_min);
  for (int i = n + static_cast<int>(threadIdx.x); i < stride; i += blockDim.x) out[i] = -1;
}

// Grid (H, B). Keeps block M-1 and the n-1 best of blocks 0 .. M-2; among
// equal scores the lower index wins. Output ascending.
//
// Keys are order-preserving 32-bit images of the scores, taken relative to
// the group minimum. A first histogram over the top 11 bits of that offset
// (starting at the highest bit in which the keys differ, so the bins spread
// even when all scores share sign and exponent) locates the threshold bin;
// its few candidates are then ranked exactly (key descending, index
// ascending) to find the last one kept. When the bin is crowded (near-constant scores) 8-bit radix
// passes continue on the remaining bits instead. The ascending output is
// written by warps that each own a contiguous index range and order their
// lanes with ballots, so every shared-memory read is conflict-free.
template <bool IN_SMEM>
__global__ void __launch_bounds__(kSelThreads) select_kernel(const float* __restrict__ scores,
                                                             int32_t* __restrict__ sel, int H,
                                                             int M, int n, SelRows rl) {
  extern __shared__ uint32_t dyn[];               // keys (if kept in shared memory)
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t cand_rel[kCand];
  __shared__ int cand_j[kCand];
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t red_min[32], red_max[32];
  __shared__ uint32_t s_prefix, s_remaining, s_total, s_kmin, s_kmax, s_ncand, s_cut_rel;
  __shared__ int s_mode;                          // 0 exact threshold, 1 bin floor, 2 ranked bin
  __shared__ int s_cut_j;
  grid_launch_dependents();
  // Scores come from the previous kernel. The wait comes before every exit,
  // the early ones included: the attention kernel launched after this one
  // waits only for this grid, so this wait is also what orders it after the
  // score kernel's append of the new token (block M-1 is always attended).
  grid_dependency_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t bh = static_cast<int64_t>(blockIdx.y) * H + blockIdx.x;
  const float* s = scores + bh * M;
  int32_t* out = sel + bh * n;
  if (rl.lens != nullptr) row_budget(rl, blockIdx.y, M, n, out);
  const int Mo = M - 1;                            // candidates: blocks 0 .. M-2
  const int need = n - 1;                          // how many of them to keep
  uint32_t* skeys = dyn;

  if (need >= Mo) {                                // every block is selected
    for (int j = tid; j < M; j += blockDim.x) out[j] = j;
    return;
  }
  if (need <= 0) {
    if (tid == 0) out[0] = M - 1;
    return;
  }
  auto key_at = [&](int j) -> uint32_t {
    if constexpr (IN_SMEM) return skeys[j];
    else return score_key(__ldcg(s + j));
  };
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
        if constexpr (IN_SMEM) skeys[j] = k;
        kmin = min(kmin, k);
        kmax = max(kmax, k);
      }
    }
  }
  for (int b = tid; b < kBins; b += blockDim.x) hist[b] = 0u;
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
      s_prefix = 0u; s_remaining = static_cast<uint32_t>(need); s_ncand = 0u; s_mode = 0;
    }
  }
  __syncthreads();
  const uint32_t base = s_kmin;
  const uint32_t range = s_kmax - base;
  int top = 32 - __clz(range);                     // bits of rel that can differ
  const int shift = top > 11 ? top - 11 : 0;
  if (top > 0) {
    // ---- first pass: 2048 bins
    for (int j = tid; j < Mo; j += blockDim.x) atomicAdd(&hist[(key_at(j) - base) >> shift], 1u);
    __syncthreads();
    {
      // thread t owns bins 2047-2t and 2046-2t (descending); a block scan of
      // the per-thread counts from the top finds the threshold bin
      const uint32_t c0 = hist[kBins - 1 - 2 * tid], c1 = hist[kBins - 2 - 2 * tid];
      const uint32_t before = block_exclusive_scan(c0 + c1, warp_tot, &s_total);
      const uint32_t rem = static_cast<uint32_t>(need);
      uint32_t acc = before;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const uint32_t c = e == 0 ? c0 : c1;
        if (acc < rem && rem <= acc + c) {
          const uint32_t digit = static_cast<uint32_t>(kBins - 1 - 2 * tid - e);
          s_prefix = digit << shift;
          s_remaining = rem - acc;
          s_mode = (rem - acc == c) ? 1 : (c <= static_cast<uint32_t>(kCand) && shift > 0 ? 2 : 0);
        }
        acc += c;
      }
    }
    __syncthreads();
    top = shift;
    if (s_mode == 2) {
      // ---- gather the threshold bin and rank its members exactly
      const uint32_t bin = s_prefix >> shift;
      for (int j = tid; j < Mo; j += blockDim.x) {
        const uint32_t rel = key_at(j) - base;
        if ((rel >> shift) == bin) {
          const uint32_t slot = atomicAdd(&s_ncand, 1u);
          cand_rel[slot] = rel;
          cand_j[slot] = j;
        }
      }
      __syncthreads();
      rank_cut(cand_rel, cand_j, static_cast<int>(s_ncand), s_remaining, &s_cut_rel, &s_cut_j);
      __syncthreads();
      top = 0;
    } else if (s_mode == 1) {
      top = 0;
    }
  }
  // ---- remaining 8-bit radix passes (crowded threshold bin)
  while (top > 0) {
    const int sh = top > 8 ? top - 8 : 0;
    const int width = top - sh;
    if (tid < 256) hist[tid] = 0u;
    __syncthreads();
    const uint32_t prefix = s_prefix;
    const uint32_t hi_mask = top >= 32 ? 0u : ~((1u << top) - 1u);
    for (int j = tid; j < Mo; j += blockDim.x) {
      const uint32_t rel = key_at(j) - base;
      if ((rel & hi_mask) == prefix) atomicAdd(&hist[(rel >> sh) & ((1u << width) - 1u)], 1u);
    }
    __syncthreads();
    if (warp == 0) {
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
            s_prefix = prefix | (static_cast<uint32_t>(255 - 8 * lane - i) << sh);
            s_remaining = rem - acc;
            if (rem - acc == c[i]) s_mode = 1;
          }
          acc += c[i];
        }
      }
    }
    __syncthreads();
    top = s_mode == 1 ? 0 : sh;
  }
  // ---- ascending compaction, one contiguous index range per warp
  // mode 0: rel > T, plus the need_eq lowest-index keys with rel == T
  // mode 1: rel >= T (the floor of a bin that is taken whole)
  // mode 2: (rel, index) at or above the cut found by ranking the bin
  const int mode = s_mode;
  const uint32_t T = s_prefix;
  const uint32_t cut_rel = s_cut_rel;
  const int cut_j = s_cut_j;
  const uint32_t need_eq = s_remaining;
  const int nw = blockDim.x >> 5;
  const int chunk = (((Mo + 31) / 32 + nw - 1) / nw) * 32;
  const int wb = min(Mo, warp * chunk), we = min(Mo, wb + chunk);
  auto plain_take = [&](int j, uint32_t rel) -> bool {
    if (mode == 0) return rel > T;
    if (mode == 1) return rel >= T;
    return at_or_above(rel, j, cut_rel, cut_j);
  };
  uint32_t cnt = 0, cnt_eq = 0;
  for (int b0 = wb; b0 < we; b0 += 32) {
    const int j = b0 + lane;
    const bool in = j < we;
    const uint32_t rel = in ? key_at(j) - base : 0u;
    cnt += __popc(__ballot_sync(0xffffffffu, in && plain_take(j, rel)));
    cnt_eq += __popc(__ballot_sync(0xffffffffu, in && mode == 0 && rel == T));
  }
  uint32_t eq_seen = 0;
  if (mode == 0) eq_seen = warp_exclusive_offset(cnt_eq, warp_tot, &s_total);
  const uint32_t eq_take = mode == 0
      ? (eq_seen >= need_eq ? 0u : min(cnt_eq, need_eq - eq_seen)) : 0u;
  uint32_t pos = warp_exclusive_offset(cnt + eq_take, warp_tot, &s_total);
  const uint32_t lt = (1u << lane) - 1u;
  for (int b0 = wb; b0 < we; b0 += 32) {
    const int j = b0 + lane;
    const bool in = j < we;
    const uint32_t rel = in ? key_at(j) - base : 0u;
    bool take = in && plain_take(j, rel);
    if (mode == 0) {
      const uint32_t eqb = __ballot_sync(0xffffffffu, in && rel == T);
      if (in && rel == T) take = eq_seen + __popc(eqb & lt) < need_eq;
      eq_seen += __popc(eqb);
    }
    const uint32_t tb = __ballot_sync(0xffffffffu, take);
    if (take) out[pos + __popc(tb & lt)] = j;
    pos += __popc(tb);
  }
  if (tid == 0) out[need] = M - 1;
}

// Exclusive scan of a [KPT][32] table of per-(round, warp) counts in
// (round, warp) order, in place; one warp does it. Returns the total.
template <int KPT>
__device__ __forceinline__ uint32_t scan_round_warp_table(uint32_t* tab) {
  const int lane = threadIdx.x & 31;
  uint32_t v[KPT], local = 0;
#pragma unroll
  for (int i = 0; i < KPT; ++i) { v[i] = tab[lane * KPT + i]; local += v[i]; }
  uint32_t inc = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  uint32_t run = inc - local;
#pragma unroll
  for (int i = 0; i < KPT; ++i) { tab[lane * KPT + i] = run; run += v[i]; }
  return __shfl_sync(0xffffffffu, inc, 31);
}

// Selection with every key in registers (M - 1 <= KPT * 1024): thread t holds
// blocks t, t + 1024, ..., so the index order of the output is (round k,
// warp, lane). Same result as select_kernel: block M-1 plus the n-1 best of
// the rest, ties to the lower index, ascending.
template <int KPT>
__global__ void __launch_bounds__(kSelThreads) select_reg_kernel(const float* __restrict__ scores,
                                                                 int32_t* __restrict__ sel, int H,
                                                                 int M, int n, SelRows rl) {
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t cand_rel[kCand];
  __shared__ int cand_j[kCand];
  __shared__ uint32_t tab[KPT * 32];
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t red_min[32], red_max[32];
  __shared__ uint32_t s_prefix, s_remaining, s_total, s_kmin, s_kmax, s_ncand, s_cut_rel;
  __shared__ int s_mode, s_cut_j;
  grid_launch_dependents();
  grid_dependency_wait();                          // before every exit (see select_kernel)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t bh = static_cast<int64_t>(blockIdx.y) * H + blockIdx.x;
  const float* s = scores + bh * M;
  int32_t* out = sel + bh * n;
  if (rl.lens != nullptr) row_budget(rl, blockIdx.y, M, n, out);
  const int Mo = M - 1;
  const int need = n - 1;
  if (need >= Mo) {
    for (int j = tid; j < M; j += blockDim.x) out[j] = j;
    return;
  }
  if (need <= 0) {
    if (tid == 0) out[0] = M - 1;
    return;
  }
  uint32_t kr[KPT];
  float x[KPT];
#pragma unroll
  for (int k = 0; k < KPT; ++k) {
    const int j = tid + k * kSelThreads;
    x[k] = j < Mo ? __ldcg(s + j) : 0.f;
  }
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int k = 0; k < KPT; ++k) {
    kr[k] = score_key(x[k]);
    if (tid + k * kSelThreads < Mo) { kmin = min(kmin, kr[k]); kmax = max(kmax, kr[k]); }
  }
  for (int b = tid; b < kBins; b += blockDim.x) hist[b] = 0u;
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (lane == 0) { red_min[warp] = kmin; red_max[warp] = kmax; }
  __syncthreads();
  if (warp == 0) {
    uint32_t a = red_min[lane], b = red_max[lane];
    a = __reduce_min_sync(0xffffffffu, a);
    b = __reduce_max_sync(0xffffffffu, b);
    if (lane == 0) {
      s_kmin = a; s_kmax = b;
      s_prefix = 0u; s_remaining = static_cast<uint32_t>(need); s_ncand = 0u; s_mode = 0;
    }
  }
  __syncthreads();
  const uint32_t base = s_kmin;
  const uint32_t range = s_kmax - base;
#pragma unroll
  for (int k = 0; k < KPT; ++k) kr[k] -= base;    // kr now holds rel = key - min
  auto valid = [&](int k) { return tid + k * kSelThreads < Mo; };
  int top = 32 - __clz(range);
  const int shift = top > 11 ? top - 11 : 0;
  if (top > 0) {
#pragma unroll
    for (int k = 0; k < KPT; ++k)
      if (valid(k)) atomicAdd(&hist[kr[k] >> shift], 1u);
    __syncthreads();
    {
      const uint32_t c0 = hist[kBins - 1 - 2 * tid], c1 = hist[kBins - 2 - 2 * tid];
      const uint32_t before = block_exclusive_scan(c0 + c1, warp_tot, &s_total);
      const uint32_t rem = static_cast<uint32_t>(need);
      uint32_t acc = before;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const uint32_t c = e == 0 ? c0 : c1;
        if (acc < rem && rem <= acc + c) {
          const uint32_t digit = static_cast<uint32_t>(kBins - 1 - 2 * tid - e);
          s_prefix = digit << shift;
          s_remaining = rem - acc;
          s_mode = (rem - acc == c) ? 1 : (c <= static_cast<uint32_t>(kCand) && shift > 0 ? 2 : 0);
        }
        acc += c;
      }
    }
    __syncthreads();
    top = shift;
    if (s_mode == 2) {
      const uint32_t bin = s_prefix >> shift;
#pragma unroll
      for (int k = 0; k < KPT; ++k) {
        if (valid(k) && (kr[k] >> shift) == bin) {
          const uint32_t slot = atomicAdd(&s_ncand, 1u);
          cand_rel[slot] = kr[k];
          cand_j[slot] = tid + k * kSelThreads;
        }
      }
      __syncthreads();
      rank_cut(cand_rel, cand_j, static_cast<int>(s_ncand), s_remaining, &s_cut_rel, &s_cut_j);
      __syncthreads();
      top = 0;
    } else if (s_mode == 1) {
      top = 0;
    }
  }
  while (top > 0) {                                // crowded threshold bin
    const int sh = top > 8 ? top - 8 : 0;
    const int width = top - sh;
    if (tid < 256) hist[tid] = 0u;
    __syncthreads();
    const uint32_t prefix = s_prefix;
    const uint32_t hi_mask = top >= 32 ? 0u : ~((1u << top) - 1u);
#pragma unroll
    for (int k = 0; k < KPT; ++k)
      if (valid(k) && (kr[k] & hi_mask) == prefix)
        atomicAdd(&hist[(kr[k] >> sh) & ((1u << width) - 1u)], 1u);
    __syncthreads();
    if (warp == 0) {
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
            s_prefix = prefix | (static_cast<uint32_t>(255 - 8 * lane - i) << sh);
            s_remaining = rem - acc;
            if (rem - acc == c[i]) s_mode = 1;
          }
          acc += c[i];
        }
      }
    }
    __syncthreads();
    top = s_mode == 1 ? 0 : sh;
  }
  // kept: mode 0 rel > T plus the need_eq lowest indices with rel == T;
  // mode 1 rel >= T (the threshold bin whole); mode 2 at or above the cut
  const int mode = s_mode;
  const uint32_t T = s_prefix;
  const uint32_t need_eq = s_remaining;
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t take = 0u;                              // bit k: block tid + 1024 k is kept
  {
    const uint32_t cut_rel = mode == 2 ? s_cut_rel : T;
    const int cut_j = mode == 1 ? 0x7fffffff : (mode == 2 ? s_cut_j : -1);
#pragma unroll
    for (int k = 0; k < KPT; ++k)
      if (valid(k) && at_or_above(kr[k], tid + k * kSelThreads, cut_rel, cut_j)) take |= 1u << k;
  }
  if (mode == 0) {
    // keys equal to the threshold: the need_eq lowest indices
#pragma unroll
    for (int k = 0; k < KPT; ++k) {
      const uint32_t eqb = __ballot_sync(0xffffffffu, valid(k) && kr[k] == T);
      if (lane == 0) tab[k * 32 + warp] = __popc(eqb);
    }
    __syncthreads();
    if (warp == 0) scan_round_warp_table<KPT>(tab);
    __syncthreads();
#pragma unroll
    for (int k = 0; k < KPT; ++k) {
      const bool eq = valid(k) && kr[k] == T;
      const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
      if (eq && tab[k * 32 + warp] + __popc(eqb & lt) < need_eq) take |= 1u << k;
    }
    __syncthreads();
  }
#pragma unroll
  for (int k = 0; k < KPT; ++k) {
    const uint32_t tb = __ballot_sync(0xffffffffu, (take >> k) & 1u);
    if (lane == 0) tab[k * 32 + warp] = __popc(tb);
  }
  __syncthreads();
  if (warp == 0) scan_round_warp_table<KPT>(tab);
  __syncthreads();
#pragma unroll
  for (int k = 0; k < KPT; ++k) {
    const bool t = (take >> k) & 1u;
    const uint32_t tb = __ballot_sync(0xffffffffu, t);
    if (t) out[tab[k * 32 + warp] + __popc(tb & lt)] = tid + k * kSelThreads;
  }
  if (tid == 0) out[need] = M - 1;
}

cudaError_t launch_select(const Shape& s, const float* scores, int32_t* sel, int M, int n,
                          cudaStream_t st, const int32_t* lens, int64_t len, double r,
                          int n_min) {
  const SelRows rl{lens, len, r, n_min};
  if (M > kSelMaxM) return cudaErrorInvalidValue;
  const bool in_smem = M <= kSelSmemKeys;
  const size_t smem = in_smem ? static_cast<size_t>(M) * sizeof(uint32_t) : 0;
  static std::atomic<bool> attr_set[64];   // per device; launches may come from several host threads
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    const int most = kSelSmemKeys * static_cast<int>(sizeof(uint32_t));
    cudaError_t e = cudaFuncSetAttribute(select_kernel<true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  // programmatic dependent launch: the grid may start while the scores are
  // still being written; it waits for them on the device
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(s.H, s.B);
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int Mo = M - 1;
  if (Mo <= 8 * kSelThreads) {
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, select_reg_kernel<8>, scores, sel, s.H, M, n, rl);
  }
  if (Mo <= 16 * kSelThreads) {
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, select_reg_kernel<16>, scores, sel, s.H, M, n, rl);
  }
  if (in_smem) return cudaLaunchKernelEx(&cfg, select_kernel<true>, scores, sel, s.H, M, n, rl);
  return cudaLaunchKernelEx(&cfg, select_kernel<false>, scores, sel, s.H, M, n, rl);
}

}  // namespace resa
