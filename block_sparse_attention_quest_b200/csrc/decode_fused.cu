// One-launch GBSA decode step (bf16): append, group scores, top-n selection,
// split-KV attention and the log-sum-exp merge in a single cooperative grid.
//
// "Rectified Sparse Attention" (pith.science review), section "What carries
// the argument": each GQA group ranks its key blocks with the pooled Quest
// bound, keeps the top n = max(n_min, ceil(M p)) (Eq. 5, p read as the active
// ratio) plus the newest block, and all its query heads attend to those
// blocks (Eq. 2); the split/merge schedule follows Flash-Decoding.
//
// The three stages of the step depend on each other through the whole score
// vector of a group, so as separate kernels every boundary costs a launch and
// a round trip through L2. Here the cpg CTAs of a group (one per SM, all
// resident: cooperative launch) do:
//   1. score a contiguous slice of the group's descriptors (CTA 0 of the
//      group also appends the new token) and publish the scores;
//   2. wait on one group barrier (bounded spin on an arrival counter);
//   3. every CTA reads all M-1 scores of its group and runs the same exact
//      selection (2048-bin radix over key offsets, threshold-bin members
//      ranked by (key desc, index asc)), so all CTAs agree on the ascending
//      block list without further exchange; CTA c then takes the c-th equal
//      share of that list (CTA 0 also writes the list to `sel`);
//   4. attend over its share with per-warp TMA rings and warp MMA, as in
//      attend_bf16_kernel, and merge the group's partials in the last CTA to
//      arrive, which also returns the group's counters to zero.
#include "launch.h"

namespace resa {

constexpr int kFW = 8;                 // warps per CTA
constexpr int kFStages = 3;            // tiles in flight per warp
constexpr int kFThreads = kFW * 32;
constexpr int kFBins = 2048;
constexpr int kFCand = 1024;
constexpr int kFMaxIds = 2048;         // blocks of one CTA's share
constexpr int kFMaxRounds = 184;       // rounds of 256 keys: M-1 <= 47104 (keys fit the tiles)

struct FusedArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k;
  __nv_bfloat16* v;
  __nv_bfloat16* desc;
  __nv_bfloat16* out;
  float* lse;
  int32_t* sel;
  float* scores;          // [groups][M]
  float* part_o;          // [groups*G][cpg][D]
  float* part_ml;         // [groups*G][cpg][2]
  int* sync;              // [groups][2]: barrier and merge arrivals
  Ctrl* ctrl;
  int64_t len, L_max;
  int H, Hq, G, Mmax, M, n, cpg;
  float scale_log2;
};

template <int D>
struct FCfg {
  static constexpr int kHalf = 16 * 64 * 2;
  static constexpr int kHalves = D / 64;
  static constexpr int kTile = 2 * kHalves * kHalf;
  static constexpr int kSmem = kFW * kFStages * kTile + 1024;
};

__device__ __forceinline__ uint32_t fkey(float f) {
  uint32_t u = __float_as_uint(f);
  if (f == 0.0f) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}



// exclusive scan of one value per thread over the CTA (kFThreads threads)
__device__ __forceinline__ uint32_t cta_exclusive_scan(uint32_t x, uint32_t* wtot, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) wtot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const uint32_t t = lane < kFW ? wtot[lane] : 0u;
    uint32_t ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += y;
    }
    if (lane < kFW) wtot[lane] = ti - t;
    if (lane == 31) *total = ti;
  }
  __syncthreads();
  const uint32_t r = wtot[warp] + inc - x;
  __syncthreads();
  return r;
}

// in-place exclusive scan of tab[0 .. count) (count <= kFMaxRounds * kFW)
__device__ __forceinline__ void scan_table(uint32_t* tab, int count, uint32_t* wtot, uint32_t* total) {
  const int per = (count + kFThreads - 1) / kFThreads;
  uint32_t loc = 0;
  for (int e = 0; e < per; ++e) {
    const int ix = threadIdx.x * per + e;
    loc += ix < count ? tab[ix] : 0u;
  }
  uint32_t run = cta_exclusive_scan(loc, wtot, total);
  for (int e = 0; e < per; ++e) {
    const int ix = threadIdx.x * per + e;
    if (ix < count) {
      const uint32_t v = tab[ix];
      tab[ix] = run;
      run += v;
    }
  }
  __syncthreads();
}

template <int D>
__global__ void __launch_bounds__(kFThreads, 1) decode_fused_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                    const __grid_constant__ CUtensorMap tmV,
                                                                    FusedArgs a) {
  using Cfg = FCfg<D>;
  constexpr int KT = D / 16;
  constexpr int CH = 8;                         // bf16 per 16-byte chunk
  constexpr int CPB = 2 * D / CH;               // chunks per descriptor block
  constexpr int W = CPB < 32 ? CPB : 32;
  constexpr int CPL = CPB / W;
  constexpr int BPL = 32 / W;
  constexpr int U = 8;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[kFW][kFStages];
  __shared__ float coef[2 * D];
  __shared__ uint32_t hist[kFBins];
  __shared__ uint32_t cand_rel[kFCand];
  __shared__ int cand_j[kFCand];
  __shared__ uint32_t tab[kFMaxRounds * kFW];
  __shared__ int ids[kFMaxIds];
  __shared__ uint32_t wtot[32];
  __shared__ uint32_t s_prefix, s_remaining, s_total, s_ncand, s_kmin, s_kmax;
  __shared__ int s_mode, s_last;
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));

  const int grp = blockIdx.x / a.cpg, slot = blockIdx.x % a.cpg;
  const int b = grp / a.H, g = grp % a.H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t bh = static_cast<int64_t>(b) * a.H + g;
  const int M = a.M, Mo = M - 1, need = a.n - 1;
  int* bar_cnt = a.sync + grp * 2;
  int* merge_cnt = a.sync + grp * 2 + 1;

  if (lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
#pragma unroll
    for (int st = 0; st < kFStages; ++st) mbar_init(&bars[warp][st], 1);
    fence_mbar_init();
  }
  // query values: score coefficients and the MMA B fragments
  const __nv_bfloat16* q = a.q + (static_cast<int64_t>(b) * a.Hq + g * a.G) * D;
  if (tid < D) {
    float nsum = 0.f, psum = 0.f;
    for (int h = 0; h < a.G; ++h) {
      const float x = __bfloat162float(q[h * D + tid]);
      nsum += fminf(x, 0.f);
      psum += fmaxf(x, 0.f);
    }
    coef[tid] = nsum;
    coef[D + tid] = psum;
  }
  const int gq = lane >> 2, cq = lane & 3;
  uint32_t qb[KT][2];
#pragma unroll
  for (int kk = 0; kk < KT; ++kk) {
    if (gq < a.G) {
      qb[kk][0] = *reinterpret_cast<const uint32_t*>(q + gq * D + kk * 16 + 2 * cq);
      qb[kk][1] = *reinterpret_cast<const uint32_t*>(q + gq * D + kk * 16 + 8 + 2 * cq);
    } else {
      qb[kk][0] = 0u;
      qb[kk][1] = 0u;
    }
  }
  for (int i = tid; i < kFBins; i += kFThreads) hist[i] = 0u;
  if (tid == 0) { s_ncand = 0u; s_mode = 0; }
  __syncthreads();

  // ------------------------------------------------------------ 1. scores
  float* sc = a.scores + static_cast<int64_t>(grp) * M;
  {
    const int j_begin = static_cast<int>(static_cast<int64_t>(slot) * Mo / a.cpg);
    const int j_end = static_cast<int>(static_cast<int64_t>(slot + 1) * Mo / a.cpg);
    const __nv_bfloat16* dbase = a.desc + bh * a.Mmax * 2 * D;
    const int seg = lane / W;
    float cf[CPL][CH];
#pragma unroll
    for (int w = 0; w < CPL; ++w)
#pragma unroll
      for (int e = 0; e < CH; ++e) cf[w][e] = coef[((lane % W) + w * W) * CH + e];
    for (int j0 = j_begin + warp * U * BPL; j0 < j_end; j0 += kFW * U * BPL) {
      uint4 raw[U][CPL];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + u * BPL + seg;
#pragma unroll
        for (int w = 0; w < CPL; ++w)
          raw[u][w] = j < j_end ? ld_stream16(dbase + static_cast<int64_t>(j) * 2 * D +
                                              ((lane % W) + w * W) * CH)
                                : make_uint4(0, 0, 0, 0);
      }
      float v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < CPL; ++w) {
          float f[CH];
          Chunk<__nv_bfloat16>::unpack(raw[u][w], f);
#pragma unroll
          for (int e = 0; e < CH; ++e) acc = fmaf(cf[w][e], f[e], acc);
        }
        v[u] = acc;
      }
      // sum each block's W lanes (transposed: one shuffle round per halving)
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
      int idx = 0, cnt = U;
#pragma unroll
      for (int m = W / 2; m >= 1; m >>= 1) {
        if (cnt > 1) {
          cnt /= 2;
          if (lane & m) idx += cnt;
        }
      }
      if ((lane % (W / U)) == 0) {
        const int j = j0 + idx * BPL + seg;
        if (j < j_end) sc[j] = v[0];
      }
    }
    // append of the decode token into its block (never read by any slice)
    if (slot == 0 && a.k_new != nullptr && tid < D) {
      const int64_t t = a.len - 1;
      const __nv_bfloat16 kn = a.k_new[bh * D + tid];
      a.k[(bh * a.L_max + t) * D + tid] = kn;
      a.v[(bh * a.L_max + t) * D + tid] = a.v_new[bh * D + tid];
      __nv_bfloat16* d = a.desc + (bh * a.Mmax + t / kBlock) * 2 * D;
      if (t % kBlock == 0) {
        d[tid] = kn;
        d[D + tid] = kn;
      } else {
        const float x = __bfloat162float(kn);
        d[tid] = __float2bfloat16_rn(fminf(__bfloat162float(d[tid]), x));
        d[D + tid] = __float2bfloat16_rn(fmaxf(__bfloat162float(d[D + tid]), x));
      }
    }
  }

  // ------------------------------------------------------------ 2. group barrier
  bool ok = true;
  // the appended K/V are read by other CTAs' TMA copies (async proxy)
  asm volatile("fence.proxy.async.global;" ::: "memory");
  if (a.cpg > 1) {
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      atomicAdd(bar_cnt, 1);
      if (!wait_count_bounded(bar_cnt, a.cpg, kWaitLimitNs, a.ctrl)) s_mode = -1;
      __threadfence();
    }
    __syncthreads();
    ok = s_mode >= 0;
    if (!ok) return;
  } else {
    __syncthreads();
  }

  // ------------------------------------------------------------ 3. selection
  uint32_t* skeys = reinterpret_cast<uint32_t*>(tiles);      // [Mo] (tiles idle until phase 4)
  uint32_t* chosen = skeys + Mo;                              // bitmap over Mo
  const int nwords = (Mo + 31) >> 5;
  const int rounds = (Mo + kFThreads - 1) / kFThreads;
  int lo = static_cast<int>(static_cast<int64_t>(slot) * a.n / a.cpg);
  int hi = static_cast<int>(static_cast<int64_t>(slot + 1) * a.n / a.cpg);
  const uint32_t lt = (1u << lane) - 1u;
  if (need >= Mo || need <= 0) {
    // every block, or only the newest one
    for (int r = tid; r < a.n; r += kFThreads) {
      const int j = need <= 0 ? M - 1 : r;
      if (r >= lo && r < hi) ids[r - lo] = j;
      if (slot == 0 && a.sel) a.sel[bh * a.n + r] = j;
    }
  } else {
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int j0 = tid; j0 < Mo; j0 += 8 * kFThreads) {
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + u * kFThreads;
        x[u] = j < Mo ? __ldcg(sc + j) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + u * kFThreads;
        if (j < Mo) {
          const uint32_t kk = fkey(x[u]);
          skeys[j] = kk;
          kmin = min(kmin, kk);
          kmax = max(kmax, kk);
        }
      }
    }
    for (int w = tid; w < nwords; w += kFThreads) chosen[w] = 0u;
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) { cand_rel[warp] = kmin; cand_rel[32 + warp] = kmax; }
    __syncthreads();
    if (warp == 0) {
      uint32_t x0 = lane < kFW ? cand_rel[lane] : 0xffffffffu;
      uint32_t x1 = lane < kFW ? cand_rel[32 + lane] : 0u;
      x0 = __reduce_min_sync(0xffffffffu, x0);
      x1 = __reduce_max_sync(0xffffffffu, x1);
      if (lane == 0) {
        s_kmin = x0; s_kmax = x1;
        s_prefix = 0u; s_remaining = static_cast<uint32_t>(need);
      }
    }
    __syncthreads();
    const uint32_t base = s_kmin;
    const uint32_t range = s_kmax - base;
    int top = 32 - __clz(range);
    const int shift = top > 11 ? top - 11 : 0;
    if (top > 0) {
      for (int j = tid; j < Mo; j += kFThreads) atomicAdd(&hist[(skeys[j] - base) >> shift], 1u);
      __syncthreads();
      {
        // thread t owns bins 2047-8t .. 2040-8t, scanned from the top
        uint32_t c[8], local = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) { c[e] = hist[kFBins - 1 - 8 * tid - e]; local += c[e]; }
        const uint32_t before = cta_exclusive_scan(local, wtot, &s_total);
        const uint32_t rem = static_cast<uint32_t>(need);
        uint32_t acc = before;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (acc < rem && rem <= acc + c[e]) {
            const uint32_t digit = static_cast<uint32_t>(kFBins - 1 - 8 * tid - e);
            s_prefix = digit << shift;
            s_remaining = rem - acc;
            s_mode = (rem - acc == c[e]) ? 1 : (c[e] <= static_cast<uint32_t>(kFCand) && shift > 0 ? 2 : 0);
          }
          acc += c[e];
        }
      }
      __syncthreads();
      top = shift;
      if (s_mode == 2) {
        const uint32_t bin = s_prefix >> shift;
        for (int j = tid; j < Mo; j += kFThreads) {
          const uint32_t rel = skeys[j] - base;
          if ((rel >> shift) == bin) {
            const uint32_t sl = atomicAdd(&s_ncand, 1u);
            cand_rel[sl] = rel;
            cand_j[sl] = j;
          }
        }
        __syncthreads();
        const int c = static_cast<int>(s_ncand);
        const uint32_t take = s_remaining;
        for (int i = tid; i < c; i += kFThreads) {
          const uint32_t r = cand_rel[i];
          const int jj = cand_j[i];
          uint32_t rank = 0;
          for (int k2 = 0; k2 < c; ++k2) {
            const uint32_t rk = cand_rel[k2];
            rank += (rk > r) || (rk == r && cand_j[k2] < jj);
          }
          if (rank < take) atomicOr(&chosen[jj >> 5], 1u << (jj & 31));
        }
        __syncthreads();
        top = 0;
      } else if (s_mode == 1) {
        top = 0;
      }
    }
    while (top > 0) {                                         // crowded threshold bin
      const int sh = top > 8 ? top - 8 : 0;
      const int width = top - sh;
      if (tid < 256) hist[tid] = 0u;
      __syncthreads();
      const uint32_t prefix = s_prefix;
      const uint32_t hi_mask = top >= 32 ? 0u : ~((1u << top) - 1u);
      for (int j = tid; j < Mo; j += kFThreads) {
        const uint32_t rel = skeys[j] - base;
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
    const int mode = s_mode;
    const uint32_t T = s_prefix;
    const uint64_t next_floor = static_cast<uint64_t>(T) + (1ull << shift);
    const uint32_t need_eq = s_remaining;
    auto take_of = [&](int j) -> bool {
      if (j >= Mo) return false;
      const uint32_t rel = skeys[j] - base;
      if (mode == 0) return rel > T;
      if (mode == 1) return rel >= T;
      return static_cast<uint64_t>(rel) >= next_floor || ((chosen[j >> 5] >> (j & 31)) & 1u);
    };
    // index order of keys: round k (j = tid + 256 k), then warp, then lane
    if (mode == 0) {
      // keys equal to the threshold are taken lowest index first: their
      // ranks among equals come from a (round, warp) table
      for (int k = 0; k < rounds; ++k) {
        const int j = tid + k * kFThreads;
        const uint32_t eqb = __ballot_sync(0xffffffffu, j < Mo && skeys[j] - base == T);
        if (lane == 0) tab[k * kFW + warp] = __popc(eqb);
      }
      __syncthreads();
      scan_table(tab, rounds * kFW, wtot, &s_total);
      for (int k = 0; k < rounds; ++k) {
        const int j = tid + k * kFThreads;
        const bool eq = j < Mo && skeys[j] - base == T;
        const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
        if (eq && tab[k * kFW + warp] + __popc(eqb & lt) < need_eq) atomicOr(&chosen[j >> 5], 1u << (j & 31));
      }
      __syncthreads();
    }
    auto taken = [&](int j) -> bool {
      if (j >= Mo) return false;
      if (mode == 0 && skeys[j] - base == T) return (chosen[j >> 5] >> (j & 31)) & 1u;
      return take_of(j);
    };
    for (int k = 0; k < rounds; ++k) {
      const uint32_t tb = __ballot_sync(0xffffffffu, taken(tid + k * kFThreads));
      if (lane == 0) tab[k * kFW + warp] = __popc(tb);
    }
    __syncthreads();
    // exclusive offsets of the (round, warp) counts, in index order
    scan_table(tab, rounds * kFW, wtot, &s_total);
    for (int k = 0; k < rounds; ++k) {
      const int j = tid + k * kFThreads;
      const bool t = taken(j);
      const uint32_t tb = __ballot_sync(0xffffffffu, t);
      if (t) {
        const int rank = static_cast<int>(tab[k * kFW + warp] + __popc(tb & lt));
        if (rank >= lo && rank < hi) ids[rank - lo] = j;
        if (slot == 0 && a.sel) a.sel[bh * a.n + rank] = j;
      }
    }
    if (tid == 0) {
      if (need >= lo && need < hi) ids[need - lo] = M - 1;
      if (slot == 0 && a.sel) a.sel[bh * a.n + need] = M - 1;
    }
  }
  __syncthreads();

  // ------------------------------------------------------------ 4. attention
  const int span = hi - lo;
  const int my_count = span > warp ? (span - warp + kFW - 1) / kFW : 0;
  const int64_t row_base = bh * a.L_max;
  const int64_t len = a.len;
  auto block_of = [&](int kx) -> int { return ids[warp + kx * kFW]; };
  auto issue = [&](int kx) {
    const int st = kx % kFStages;
    const int y = static_cast<int>(row_base + static_cast<int64_t>(block_of(kx)) * kBlock);
    uint8_t* t = tiles + (warp * kFStages + st) * Cfg::kTile;
    mbar_arrive_expect_tx(&bars[warp][st], Cfg::kTile);
#pragma unroll
    for (int hf = 0; hf < Cfg::kHalves; ++hf) {
      tma_load_2d(t + hf * Cfg::kHalf, &tmK, hf * 64, y, &bars[warp][st]);
      tma_load_2d(t + (Cfg::kHalves + hf) * Cfg::kHalf, &tmV, hf * 64, y, &bars[warp][st]);
    }
  };
  // the key buffer above aliased the tiles: order those generic accesses
  // before the first TMA writes
  fence_proxy_async_smem();
  asm volatile("fence.proxy.async.global;" ::: "memory");
  __syncthreads();
  if (lane == 0) {
    for (int kx = 0; kx < my_count && kx < kFStages; ++kx) issue(kx);
  }
  float o[KT][4];
#pragma unroll
  for (int mt = 0; mt < KT; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const float sl2 = a.scale_log2;
  const int kq_row = (lane & 7) + (((lane >> 3) & 1) << 3);
  const int kq_chk = lane >> 4;
  const int vt_row = (lane & 7) + ((lane >> 4) << 3);
  const int vt_chk = (lane >> 3) & 1;
  int kx = 0;
  for (; kx < my_count; ++kx) {
    const int st = kx % kFStages;
    const bool arrived = mbar_wait_bounded(&bars[warp][st], (kx / kFStages) & 1, a.ctrl);
    if (!__all_sync(0xffffffffu, arrived)) { ok = false; break; }
    const int j = block_of(kx);
    uint8_t* tp = tiles + (warp * kFStages + st) * Cfg::kTile;
    const uint32_t tbase = smem_u32(tp);
    const uint32_t vbase = tbase + Cfg::kHalves * Cfg::kHalf;
    const int valid_rows = static_cast<int>(len - static_cast<int64_t>(j) * kBlock);
    if (valid_rows < kBlock) {
      uint8_t* vt = tp + Cfg::kHalves * Cfg::kHalf;
      for (int idx = lane; idx < Cfg::kHalves * kBlock * 8; idx += 32) {
        const int hf = idx / (kBlock * 8), rrow = (idx / 8) % kBlock, c = idx % 8;
        if (rrow >= valid_rows)
          *reinterpret_cast<uint4*>(vt + hf * Cfg::kHalf + rrow * 128 + c * 16) = make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
    }
    float sacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < KT; ++kk) {
      const int chunk = 2 * kk + kq_chk;
      const uint32_t addr = tbase + (chunk >> 3) * Cfg::kHalf + kq_row * 128 +
                            (((chunk & 7) ^ (kq_row & 7)) << 4);
      uint32_t af[4];
      ldmatrix_x4(af, addr);
      mma_bf16_16816(sacc, af, qb[kk][0], qb[kk][1]);
    }
    const int64_t t_lo = static_cast<int64_t>(j) * kBlock + gq;
    float s0 = sacc[0] * sl2, s1 = sacc[1] * sl2, s2 = sacc[2] * sl2, s3 = sacc[3] * sl2;
    if (t_lo >= len) { s0 = -INFINITY; s1 = -INFINITY; }
    if (t_lo + 8 >= len) { s2 = -INFINITY; s3 = -INFINITY; }
    float mx0 = warp_max_xor(fmaxf(s0, s2), 16, 4), mx1 = warp_max_xor(fmaxf(s1, s3), 16, 4);
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float al0 = exp2f(m0 - mn0), al1 = exp2f(m1 - mn1);
    const float p0 = exp2f(s0 - mn0), p2 = exp2f(s2 - mn0);
    const float p1 = exp2f(s1 - mn1), p3 = exp2f(s3 - mn1);
    l0 = fmaf(l0, al0, p0 + p2);
    l1 = fmaf(l1, al1, p1 + p3);
    m0 = mn0;
    m1 = mn1;
#pragma unroll
    for (int mt = 0; mt < KT; ++mt) {
      o[mt][0] *= al0; o[mt][2] *= al0;
      o[mt][1] *= al1; o[mt][3] *= al1;
    }
    const uint32_t pb0 = movmatrix_trans(pack_bf16x2(p0, p1));
    const uint32_t pb1 = movmatrix_trans(pack_bf16x2(p2, p3));
#pragma unroll
    for (int mt = 0; mt < KT; ++mt) {
      const int chunk = 2 * mt + vt_chk;
      const uint32_t addr = vbase + (chunk >> 3) * Cfg::kHalf + vt_row * 128 +
                            (((chunk & 7) ^ (vt_row & 7)) << 4);
      uint32_t af[4];
      ldmatrix_x4_trans(af, addr);
      mma_bf16_16816(o[mt], af, pb0, pb1);
    }
    __syncwarp();
    if (lane == 0 && kx + kFStages < my_count) {
      fence_proxy_async_smem();
      issue(kx + kFStages);
    }
  }
  if (!ok) {
    for (int k2 = kx; k2 < my_count && k2 < kx + kFStages; ++k2)
      mbar_wait_bounded(&bars[warp][k2 % kFStages], (k2 / kFStages) & 1, a.ctrl);
  }
  if (!__syncthreads_and(ok)) return;
#pragma unroll
  for (int o2 = 4; o2 <= 16; o2 <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o2);
  }
  float* sm = reinterpret_cast<float*>(tiles);
  float* sm_o = sm;                       // [kFW][8][D]
  float* sm_m = sm + kFW * 8 * D;
  float* sm_l = sm_m + kFW * 8;
  const int h0 = 2 * cq, h1 = 2 * cq + 1;
  if (gq == 0) {
    sm_m[warp * 8 + h0] = m0; sm_l[warp * 8 + h0] = l0;
    sm_m[warp * 8 + h1] = m1; sm_l[warp * 8 + h1] = l1;
  }
#pragma unroll
  for (int mt = 0; mt < KT; ++mt) {
    const int ch = mt * 16 + gq;
    sm_o[(warp * 8 + h0) * D + ch] = o[mt][0];
    sm_o[(warp * 8 + h1) * D + ch] = o[mt][1];
    sm_o[(warp * 8 + h0) * D + ch + 8] = o[mt][2];
    sm_o[(warp * 8 + h1) * D + ch + 8] = o[mt][3];
  }
  __syncthreads();
  // ------------------------------------------------------------ 5. merge
  const int64_t head0 = static_cast<int64_t>(b) * a.Hq + g * a.G;
  for (int idx = tid; idx < a.G * D; idx += kFThreads) {
    const int h = idx / D, ch = idx % D;
    float mstar = -INFINITY;
#pragma unroll
    for (int w = 0; w < kFW; ++w) mstar = fmaxf(mstar, sm_m[w * 8 + h]);
    float ov = 0.f, lv = 0.f;
#pragma unroll
    for (int w = 0; w < kFW; ++w) {
      const float f = mstar == -INFINITY ? 0.f : exp2f(sm_m[w * 8 + h] - mstar);
      ov = fmaf(f, sm_o[(w * 8 + h) * D + ch], ov);
      lv = fmaf(f, sm_l[w * 8 + h], lv);
    }
    if (a.cpg == 1) {
      a.out[(head0 + h) * D + ch] = __float2bfloat16_rn(ov / lv);
      if (a.lse != nullptr && ch == 0) a.lse[head0 + h] = (mstar + log2f(lv)) * 0.69314718055994531f;
    } else {
      const int64_t row = (head0 + h) * a.cpg + slot;
      a.part_o[row * D + ch] = ov;
      if (ch == 0) {
        a.part_ml[row * 2] = mstar;
        a.part_ml[row * 2 + 1] = lv;
      }
    }
  }
  if (a.cpg == 1) return;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(merge_cnt, 1) == a.cpg - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int idx = tid; idx < a.G * D; idx += kFThreads) {
    const int h = idx / D, ch = idx % D;
    const float* po = a.part_o + (head0 + h) * a.cpg * D + ch;
    const float* ml = a.part_ml + (head0 + h) * a.cpg * 2;
    float run_m = -INFINITY, run_l = 0.f, run_o = 0.f;
    for (int sp0 = 0; sp0 < a.cpg; sp0 += 32) {
      float x[32], mv[32], lv[32];
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const bool in = sp0 + u < a.cpg;
        x[u] = in ? __ldcg(po + static_cast<int64_t>(sp0 + u) * D) : 0.f;
        mv[u] = in ? __ldcg(ml + 2 * (sp0 + u)) : -INFINITY;
        lv[u] = in ? __ldcg(ml + 2 * (sp0 + u) + 1) : 0.f;
      }
      float cm = run_m;
#pragma unroll
      for (int u = 0; u < 32; ++u) cm = fmaxf(cm, mv[u]);
      const float s = run_m == -INFINITY ? 0.f : exp2f(run_m - cm);
      run_o *= s;
      run_l *= s;
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const float w = mv[u] == -INFINITY ? 0.f : exp2f(mv[u] - cm);
        run_o = fmaf(w, x[u], run_o);
        run_l = fmaf(w, lv[u], run_l);
      }
      run_m = cm;
    }
    a.out[(head0 + h) * D + ch] = __float2bfloat16_rn(run_o / run_l);
    if (a.lse != nullptr && ch == 0) a.lse[head0 + h] = (run_m + log2f(run_l)) * 0.69314718055994531f;
  }
  if (tid == 0) {
    *bar_cnt = 0;
    *merge_cnt = 0;
  }
}

template <int D>
static cudaError_t fused_t(const FusedLaunch& f, cudaStream_t st) {
  using Cfg = FCfg<D>;
  static std::atomic<bool> attr_set[64];   // per device; launches may come from several host threads
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(decode_fused_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  FusedArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(f.q);
  a.k_new = static_cast<const __nv_bfloat16*>(f.k_new);
  a.v_new = static_cast<const __nv_bfloat16*>(f.v_new);
  a.k = static_cast<__nv_bfloat16*>(f.k);
  a.v = static_cast<__nv_bfloat16*>(f.v);
  a.desc = static_cast<__nv_bfloat16*>(f.desc);
  a.out = static_cast<__nv_bfloat16*>(f.out);
  a.lse = f.lse;
  a.sel = f.sel;
  a.scores = f.scores;
  a.part_o = f.part_o;
  a.part_ml = f.part_ml;
  a.sync = f.sync;
  a.ctrl = f.ctrl;
  a.len = f.len;
  a.L_max = f.s.L_max;
  a.H = f.s.H;
  a.Hq = f.s.Hq;
  a.G = f.s.G;
  a.Mmax = f.s.Mmax;
  a.M = f.M;
  a.n = f.n;
  a.cpg = f.cpg;
  a.scale_log2 = f.scale * 1.4426950408889634f;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(f.s.B * f.s.H * f.cpg);
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = Cfg::kSmem;
  cfg.stream = st;
  // the CTAs of a group wait on one another: all of them must be resident
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = f.cpg > 1 ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, decode_fused_kernel<D>, *f.tm_k, *f.tm_v, a);
}

// largest M-1 whose keys and bitmap fit the tiles, and largest CTA share
int fused_max_keys(int D) {
  const int bytes = kFW * kFStages * (D == 128 ? FCfg<128>::kTile : FCfg<64>::kTile);
  int mo = bytes / 4 - bytes / 128 - 1;            // keys + bitmap words
  if (mo > kFMaxRounds * kFThreads) mo = kFMaxRounds * kFThreads;
  return mo;
}
int fused_max_share() { return kFMaxIds; }

cudaError_t launch_decode_fused(const FusedLaunch& f, cudaStream_t st) {
  return f.s.D == 128 ? fused_t<128>(f, st) : fused_t<64>(f, st);
}

}  // namespace resa
