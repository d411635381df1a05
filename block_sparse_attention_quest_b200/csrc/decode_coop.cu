// One-launch GBSA decode step (bf16): append, pooled Quest scores, exact
// top-n selection, split-KV attention and the log-sum-exp merge in a single
// grid whose CTAs of one KV group cooperate on the selection.
//
// "Rectified Sparse Attention" (pith.science review), section "What carries
// the argument": each GQA group ranks its key blocks with the pooled Quest
// bound, keeps the top n = max(n_min, ceil(M p)) (Eq. 5, p read as the active
// ratio) with the newest block always among them, and all of its query heads
// attend to those blocks (Eq. 2); the split/merge schedule follows
// Flash-Decoding.
//
// Grid (S, H, B), one CTA per SM. CTA s of group (b, g) owns the slice
// [s Mo / S, (s + 1) Mo / S) of the Mo = M - 1 scored blocks:
//   1. it streams its slice's descriptors into shared memory as 2-D tensor
//      boxes and scores them there (the keys stay on the chip; CTA S - 1 also
//      appends the new token and owns the newest block);
//   2. the group's S CTAs find the exact top n - 1 (key descending, block
//      index ascending) in three rounds through L2, each ended by a release
//      arrival on the group's counter and a bounded acquire wait:
//        A  the group's key range (atomic max of ~min and of max),
//        B  a 2048-bin histogram of the key offsets: every block in a bin
//           above the threshold bin is kept, and its K/V tiles are prefetched
//           into L2 at once,
//        C  each CTA's kept blocks above the threshold bin (in index order,
//           with their count) and the threshold bin's members, which every
//           CTA ranks to the same (key, index) cut;
//      a threshold bin too crowded to rank is resolved instead by radix
//      passes that every CTA runs over all of the group's scores;
//   3. CTA s then attends to positions [s n / S, (s + 1) n / S) of the
//      ascending list (an equal share; it also writes that part of the list
//      to `sel`), and the last CTA to arrive merges the group's partials and
//      returns the group's state to zero.
// Selection and attention match score_kernel + select_reg_kernel +
// attend_bf16_kernel; only the order of the sums inside a split differs.
#include "attend_core.cuh"
#include "select_core.cuh"

namespace resa {

namespace {

constexpr int kCW = 8;                   // warps per CTA
constexpr int kCThreads = kCW * 32;
constexpr int kCStages = 2;              // K/V tiles in flight per warp
constexpr int kCKpt = 8;                 // keys per thread
constexpr int kCSlice = kCThreads * kCKpt;   // largest slice: 2048 blocks
constexpr int kCChunk = 64;              // descriptor blocks per ring slot (128 rows)
constexpr int kCRing = 4;                // ring slots in flight
constexpr int kCBoxRows = 32;            // rows of one descriptor box (64 channels x 32 rows)
constexpr int kCMaxKeys = 32768;         // keys of a group held for the crowded-bin passes
constexpr int kCMaxShare = 2048;         // blocks one CTA attends to

template <int D>
struct CoopCfg {
  using Attn = Bf16Cfg<D, kCW, kCStages>;
  static constexpr int kTiles = kCW * kCStages * Attn::kTile;
  static constexpr int kBlockBytes = 2 * D * 2;            // one descriptor (min and max rows)
  static constexpr int kHalves = D / 64;                   // 64-channel boxes per row
  static constexpr int kBox = kCBoxRows * 64 * 2;          // 4 KB
  static constexpr int kChunkBytes = kCChunk * kBlockBytes;
  static_assert(kChunkBytes == (2 * kCChunk / kCBoxRows) * kHalves * kBox, "chunk = whole boxes");
  static constexpr int kDyn0 = kTiles > kCRing * kChunkBytes ? kTiles : kCRing * kChunkBytes;
  static constexpr int kDyn = (kDyn0 > kCMaxKeys * 4 ? kDyn0 : kCMaxKeys * 4) + 1024;
};

}  // namespace

// Per-group state in the workspace (its zero-initialised prefix); every call
// leaves it at zero again.
struct CoopGroup {
  int ctr;                 // round arrivals of the group's CTAs
  unsigned mninv;          // max over CTAs of ~(smallest key): zero is neutral
  unsigned mx;             // max over CTAs of the largest key
  int ccount;              // threshold-bin members gathered
  int pad[12];
  int above[kMaxSplits];   // per CTA: kept blocks above the threshold bin (every call)
  unsigned hist[kBins];
  unsigned cand_rel[kCand];
  int cand_j[kCand];
  int cand_pos[kCand];     // its CTA's kept blocks above the threshold bin before it
};

struct CoopArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k;
  __nv_bfloat16* v;
  __nv_bfloat16* desc;
  int32_t* sel;            // [B][H][n] ascending list (caller's or the workspace's)
  float* scores;           // [B][H][M] (read back only by the crowded-bin passes)
  int32_t* kept;           // [B][H][M] each CTA's blocks above the threshold bin, at its slice
  CoopGroup* grp;          // [B][H]
  AttnK a;                 // attention and merge arguments (R = 1)
  int64_t len;
  int Mmax, M, n, S;
};

namespace {

// The CTA's arrival on the group counter: a CTA barrier, then one release add
// that publishes every thread's prior writes, then a bounded acquire wait for
// all S CTAs of this round; `target` grows by S per round on every thread.
__device__ __forceinline__ bool group_round(CoopGroup* G, int& target, int S, Ctrl* ctrl,
                                            int* s_fail) {
  __syncthreads();
  target += S;
  if (threadIdx.x == 0) {
    red_release_add(&G->ctr, 1);
    *s_fail = wait_count_bounded(&G->ctr, target, kWaitLimitNs, ctrl) ? 0 : 1;
  }
  __syncthreads();
  return *s_fail == 0;
}

__device__ __forceinline__ int slice_begin(int r, int Mo, int S) {
  return static_cast<int>(static_cast<int64_t>(r) * Mo / S);
}
// Crowded threshold bin: every CTA runs the remaining radix passes over all
// Mo key offsets of the group (keys[], from the scores every CTA wrote before
// round A) and ends with the (key offset, index) cut of the need-th key.
__device__ void crowded_cut(const uint32_t* keys, int Mo, uint32_t prefix, uint32_t remaining,
                            int top, uint32_t* hist, uint32_t* wtot, uint32_t* s_vals,
                            int* s_cut_j) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) { s_vals[0] = prefix; s_vals[1] = remaining; s_vals[2] = 0u; }
  __syncthreads();
  while (top > 0) {
    const int sh = top > 8 ? top - 8 : 0;
    const int width = top - sh;
    hist[tid] = 0u;
    __syncthreads();
    const uint32_t pre = s_vals[0];
    const uint32_t hi_mask = top >= 32 ? 0u : ~((1u << top) - 1u);
    for (int j = tid; j < Mo; j += kCThreads) {
      const uint32_t rel = keys[j];
      if ((rel & hi_mask) == pre) atomicAdd(&hist[(rel >> sh) & ((1u << width) - 1u)], 1u);
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
      const uint32_t rem = s_vals[1];
      if (before < rem && rem <= inc) {
        uint32_t acc = before;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (acc < rem && rem <= acc + c[i]) {
            s_vals[0] = pre | (static_cast<uint32_t>(255 - 8 * lane - i) << sh);
            s_vals[1] = rem - acc;
            if (rem - acc == c[i]) s_vals[2] = 1u;
          }
          acc += c[i];
        }
      }
    }
    __syncthreads();
    top = s_vals[2] ? 0 : sh;
  }
  if (s_vals[2]) {                                 // the bin at s_vals[0] is kept whole
    if (tid == 0) *s_cut_j = 0x7fffffff;
    __syncthreads();
    return;
  }
  // the need_eq-th lowest index among the keys equal to T
  const uint32_t T = s_vals[0];
  const uint32_t need_eq = s_vals[1];
  const int per = (Mo + kCThreads - 1) / kCThreads;
  const int jb = min(Mo, tid * per), je = min(Mo, jb + per);
  uint32_t cnt = 0;
  for (int j = jb; j < je; ++j) cnt += keys[j] == T;
  const uint32_t before = block_exclusive_scan(cnt, wtot, &s_vals[3]);
  if (before < need_eq && need_eq <= before + cnt) {
    uint32_t seen = before;
    for (int j = jb; j < je; ++j) {
      if (keys[j] == T && ++seen == need_eq) { *s_cut_j = j; break; }
    }
  }
  __syncthreads();
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(kCThreads, 1) decode_coop_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const __grid_constant__ CUtensorMap tmD, const CoopArgs c) {
  using Cfg = CoopCfg<D>;
  constexpr int KT = D / 16;
  constexpr int CH = 8;                          // bf16 per 16-byte chunk
  constexpr int CPB = 2 * D / CH;                // chunks per descriptor block
  constexpr int W = CPB < 32 ? CPB : 32;         // lanes per block
  constexpr int BPL = 32 / W;                    // blocks per warp-wide load
  constexpr int BPW = kCChunk / kCW;             // blocks of a ring slot each warp scores
  constexpr int U = BPW / BPL;                   // loads per warp per slot
  static_assert(CPB / W == 1, "one 16-byte chunk per lane and block");
  static_assert(BPW % BPL == 0 && U >= 1 && (U & (U - 1)) == 0, "whole warp-wide loads per slot");

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[kCW][kCStages];
  __shared__ __align__(8) uint64_t dbar[kCRing];
  __shared__ float coef[2 * D];
  __shared__ float sc[kCSlice];
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t cand_rel[kCand];
  __shared__ int cand_j[kCand];
  __shared__ int cand_pos[kCand];
  __shared__ int ids[kCMaxShare];
  __shared__ uint32_t tab[kCKpt * kCW];
  __shared__ uint32_t wtot[32];
  __shared__ uint32_t red_a[kCW], red_b[kCW];
  __shared__ int pre[kMaxSplits + 1];
  __shared__ int kc_beg[kMaxSplits + 1];         // kept candidates of slice r: [kc_beg[r], kc_beg[r+1])
  __shared__ uint32_t s_vals[8];
  __shared__ int s_fail, s_mode, s_cut_j, s_nkc;
  __shared__ uint32_t s_base, s_cut_rel;
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));

  const AttnK& a = c.a;
  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int S = c.S, M = c.M, n = c.n;
  const int Mo = M - 1, need = n - 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t bh = static_cast<int64_t>(b) * a.H + g;
  CoopGroup* G = c.grp + bh;
  const int j0 = slice_begin(s, Mo, S);
  const int m = slice_begin(s + 1, Mo, S) - j0;
  const bool rounds = need > 0 && need < Mo;     // otherwise the list is known up front
  const int64_t drow0 = (bh * c.Mmax + j0) * 2;  // first descriptor row of the slice
  const int nchunks = (m + kCChunk - 1) / kCChunk;

  if (lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
#pragma unroll
    for (int st = 0; st < kCStages; ++st) mbar_init(&bars[warp][st], 1);
  }
  if (tid == 0) {
    prefetch_tmap(&tmD);
#pragma unroll
    for (int i = 0; i < kCRing; ++i) mbar_init(&dbar[i], 1);
    s_fail = 0;
    s_mode = 0;
    s_nkc = 0;
  }
  if (lane == 0 || tid == 0) fence_mbar_init();
  for (int i = tid; i < kBins; i += kCThreads) hist[i] = 0u;
  __syncthreads();
  // launched as a programmatic dependent of whatever precedes it: nothing is
  // read (or copied) before the dependency wait
  grid_dependency_wait();

  // ------------------------------------------------------ 1. own slice's scores
  // ring slot ch % kCRing holds blocks [ch * 64, ch * 64 + 64) of the slice as
  // (row group, 64-channel half) boxes of 32 descriptor rows
  auto issue_chunk = [&](int ch) {
    const int nb = min(kCChunk, m - ch * kCChunk);
    const int groups = (2 * nb + kCBoxRows - 1) / kCBoxRows;
    uint64_t* bar = &dbar[ch % kCRing];
    uint8_t* dst = tiles + (ch % kCRing) * Cfg::kChunkBytes;
    mbar_arrive_expect_tx(bar, groups * Cfg::kHalves * Cfg::kBox);
    for (int rg = 0; rg < groups; ++rg)
#pragma unroll
      for (int h = 0; h < Cfg::kHalves; ++h)
        tma_load_2d(dst + (rg * Cfg::kHalves + h) * Cfg::kBox, &tmD, h * 64,
                    static_cast<int>(drow0 + ch * 2 * kCChunk + rg * kCBoxRows), bar);
  };
  if (rounds && tid == 0)
    for (int ch = 0; ch < nchunks && ch < kCRing; ++ch) issue_chunk(ch);

  // q: score coefficients (N for the min rows, P for the max rows) and the
  // MMA fragments
  const __nv_bfloat16* qg = c.q + (bh * a.G) * D;
  if (tid < D) {
    float nsum = 0.f, psum = 0.f;
    for (int h = 0; h < a.G; ++h) {
      const float x = __bfloat162float(qg[h * D + tid]);
      nsum += fminf(x, 0.f);
      psum += fmaxf(x, 0.f);
    }
    coef[tid] = nsum;
    coef[D + tid] = psum;
  }
  uint32_t qb[KT][2];
  load_q_frags<D>(qg, a.G, qb);

  // the new token goes to slot len-1 and into the descriptor of the newest
  // block; CTA S-1 owns that block (it is the last entry of the list), so the
  // writes and the tile copies that read them stay in one CTA
  if (s == S - 1 && c.k_new != nullptr && tid < D) {
    const int64_t t = c.len - 1;
    const __nv_bfloat16 kn = c.k_new[bh * D + tid];
    c.k[(bh * a.L_max + t) * D + tid] = kn;
    c.v[(bh * a.L_max + t) * D + tid] = c.v_new[bh * D + tid];
    __nv_bfloat16* d = c.desc + (bh * c.Mmax + t / kBlock) * 2 * D;
    if (t % kBlock == 0) {
      d[tid] = kn;
      d[D + tid] = kn;
    } else {
      const float x = __bfloat162float(kn);
      d[tid] = __float2bfloat16_rn(fminf(__bfloat162float(d[tid]), x));
      d[D + tid] = __float2bfloat16_rn(fmaxf(__bfloat162float(d[D + tid]), x));
    }
    asm volatile("fence.proxy.async.global;" ::: "memory");
  }
  __syncthreads();

  int target = 0;
  const uint32_t lt = (1u << lane) - 1u;
  int crowded = 0;                               // the list comes from all keys in shared memory
  int all_equal = 0;                             // every key of the group is equal
  int mode = 0;
  if (rounds) {
    float cf[CH];
#pragma unroll
    for (int e = 0; e < CH; ++e) cf[e] = coef[(lane % W) * CH + e];
    // this lane's 16 bytes of a block: row (min or max) and 64-channel half
    const int e0 = (lane % W) * CH;
    const int row_sel = e0 / D, half = (e0 % D) / 64, col = e0 % 64;
    float* gsc = c.scores + bh * M;
    const int seg = lane / W;
    int ch = 0;
    for (; ch < nchunks; ++ch) {
      if (!mbar_wait_bounded(&dbar[ch % kCRing], (ch / kCRing) & 1, a.ctrl)) s_fail = 1;
      __syncthreads();
      if (s_fail) break;
      const uint8_t* buf = tiles + (ch % kCRing) * Cfg::kChunkBytes;
      const int nb = min(kCChunk, m - ch * kCChunk);
      float v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int jb = warp * BPW + u * BPL + seg;        // block within the slot
        float acc = 0.f;
        if (jb < nb) {
          const int rg = (2 * jb) / kCBoxRows, rr = (2 * jb) % kCBoxRows + row_sel;
          const uint4 raw = *reinterpret_cast<const uint4*>(
              buf + ((rg * Cfg::kHalves + half) * kCBoxRows + rr) * 128 + col * 2);
          float f[CH];
          Chunk<__nv_bfloat16>::unpack(raw, f);
#pragma unroll
          for (int e = 0; e < CH; ++e) acc = fmaf(cf[e], f[e], acc);
        }
        v[u] = acc;
      }
      transpose_reduce<U, W>(v, lane);
      if (seg_value_owner<U, W>(lane)) {
        const int u = seg_value_index<U, W>(lane);
        const int jb = warp * BPW + u * BPL + seg;
        if (jb < nb) {
          const int i = ch * kCChunk + jb;
          sc[i] = v[0];
          gsc[j0 + i] = v[0];
        }
      }
      __syncthreads();                                   // the slot is free again
      if (tid == 0 && ch + kCRing < nchunks) {
        fence_proxy_async_smem();
        issue_chunk(ch + kCRing);
      }
    }
    if (s_fail) {
      // drain the copies still in flight (bounded), then leave: the host sees
      // the error flag; the group's other CTAs time out in their rounds
      if (tid == 0)
        for (int k2 = ch; k2 < nchunks && k2 < ch + kCRing; ++k2)
          mbar_wait_bounded(&dbar[k2 % kCRing], (k2 / kCRing) & 1, a.ctrl);
      return;
    }

    // ------------------------------------------------------ 2. the exact cut
    uint32_t kr[kCKpt];
    uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
    for (int k = 0; k < kCKpt; ++k) {
      const int i = tid + k * kCThreads;
      kr[k] = i < m ? score_key(sc[i]) : 0u;
      if (i < m) { kmin = min(kmin, kr[k]); kmax = max(kmax, kr[k]); }
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) { red_a[warp] = kmin; red_b[warp] = kmax; }
    __syncthreads();
    if (tid == 0) {
      uint32_t x0 = red_a[0], x1 = red_b[0];
      for (int w = 1; w < kCW; ++w) { x0 = min(x0, red_a[w]); x1 = max(x1, red_b[w]); }
      if (m > 0) {
        atomicMax(&G->mninv, ~x0);
        atomicMax(&G->mx, x1);
      }
    }
    if (!group_round(G, target, S, a.ctrl, &s_fail)) return;                 // round A
    if (tid == 0) {
      s_base = ~static_cast<uint32_t>(ld_acquire(reinterpret_cast<const int*>(&G->mninv)));
      s_vals[4] = static_cast<uint32_t>(ld_acquire(reinterpret_cast<const int*>(&G->mx)));
    }
    __syncthreads();
    const uint32_t base = s_base;
    const uint32_t range = s_vals[4] - base;
    auto valid = [&](int k) { return tid + k * kCThreads < m; };
#pragma unroll
    for (int k = 0; k < kCKpt; ++k) kr[k] -= base;       // key offsets from the group minimum
    const int top = 32 - __clz(range);
    const int shift = top > 11 ? top - 11 : 0;
    if (top == 0) {
      all_equal = 1;                                     // the lowest indices are kept
    } else {
#pragma unroll
      for (int k = 0; k < kCKpt; ++k)
        if (valid(k)) atomicAdd(&hist[kr[k] >> shift], 1u);
      __syncthreads();
      for (int i = tid; i < kBins; i += kCThreads) {
        const uint32_t cnt = hist[i];
        if (cnt) atomicAdd(&G->hist[i], cnt);
      }
      if (!group_round(G, target, S, a.ctrl, &s_fail)) return;               // round B
      uint32_t cb[8], local = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) { cb[e] = __ldcg(&G->hist[kBins - 1 - 8 * tid - e]); local += cb[e]; }
      const uint32_t before = block_exclusive_scan(local, wtot, &s_vals[5]);
      const uint32_t rem = static_cast<uint32_t>(need);
      uint32_t acc = before;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (acc < rem && rem <= acc + cb[e]) {
          const uint32_t digit = static_cast<uint32_t>(kBins - 1 - 8 * tid - e);
          s_vals[0] = digit;                             // the threshold bin
          s_vals[1] = rem - acc;                         // keys still to take from it
          s_mode = (rem - acc == cb[e]) ? 1 : (cb[e] <= static_cast<uint32_t>(kCand) && shift > 0 ? 2 : 0);
        }
        acc += cb[e];
      }
      __syncthreads();
      const uint32_t tbin = s_vals[0];
      mode = s_mode;
      // blocks above the threshold bin are kept (the whole bin too in mode 1)
      uint32_t above = 0u, inbin = 0u;
#pragma unroll
      for (int k = 0; k < kCKpt; ++k) {
        if (!valid(k)) continue;
        const uint32_t bin = kr[k] >> shift;
        if (bin > tbin || (mode == 1 && bin == tbin)) above |= 1u << k;
        else if (bin == tbin) inbin |= 1u << k;
      }
      // their K/V tiles go into L2 now, while the cut is still being found
#pragma unroll
      for (int k = 0; k < kCKpt; ++k) {
        if ((above >> k) & 1u) {
          const int y = static_cast<int>(bh * a.L_max +
                                         static_cast<int64_t>(j0 + tid + k * kCThreads) * kBlock);
#pragma unroll
          for (int hf = 0; hf < D / 64; ++hf) {
            tma_prefetch_2d(&tmK, hf * 64, y);
            tma_prefetch_2d(&tmV, hf * 64, y);
          }
        }
      }
      if (mode != 0) {
        // ---------------------------------------------------- round C
        // this CTA's blocks above the threshold bin, ascending, and their
        // count; the threshold bin's members with the count of this CTA's
        // kept blocks before each
#pragma unroll
        for (int k = 0; k < kCKpt; ++k) {
          const uint32_t tb = __ballot_sync(0xffffffffu, (above >> k) & 1u);
          if (lane == 0) tab[k * kCW + warp] = __popc(tb);
        }
        __syncthreads();
        if (warp == 0) {
          // exclusive scan of the (round, warp) counts in index order
          const uint32_t v0 = tab[2 * lane], v1 = tab[2 * lane + 1];
          uint32_t inc = v0 + v1;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
          }
          const uint32_t ex = inc - v0 - v1;
          tab[2 * lane] = ex;
          tab[2 * lane + 1] = ex + v0;
          if (lane == 31) G->above[s] = static_cast<int>(inc);
        }
        __syncthreads();
        int32_t* kept = c.kept + bh * M + j0;
#pragma unroll
        for (int k = 0; k < kCKpt; ++k) {
          const bool t = (above >> k) & 1u;
          const uint32_t tb = __ballot_sync(0xffffffffu, t);
          const uint32_t pos = tab[k * kCW + warp] + __popc(tb & lt);
          if (t) kept[pos] = j0 + tid + k * kCThreads;
          if ((inbin >> k) & 1u) {
            const int slot = atomicAdd(&G->ccount, 1);
            if (slot < kCand) {
              G->cand_rel[slot] = kr[k];
              G->cand_j[slot] = j0 + tid + k * kCThreads;
              G->cand_pos[slot] = static_cast<int>(pos);
            }
          }
        }
        if (!group_round(G, target, S, a.ctrl, &s_fail)) return;             // round C
        const int cnt = mode == 2 ? min(__ldcg(&G->ccount), kCand) : 0;
        if (warp == 0) {
          // prefix of the CTAs' counts above the threshold bin
          const int v0 = lane < S ? __ldcg(&G->above[lane]) : 0;
          const int v1 = lane + 32 < S ? __ldcg(&G->above[lane + 32]) : 0;
          int inc0 = v0, inc1 = v1;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y0 = __shfl_up_sync(0xffffffffu, inc0, o);
            const int y1 = __shfl_up_sync(0xffffffffu, inc1, o);
            if (lane >= o) { inc0 += y0; inc1 += y1; }
          }
          const int tot0 = __shfl_sync(0xffffffffu, inc0, 31);
          pre[lane] = inc0 - v0;
          pre[lane + 32] = tot0 + inc1 - v1;
          if (lane == 31) pre[kMaxSplits] = tot0 + inc1;
        }
        for (int i = tid; i < cnt; i += kCThreads) {
          cand_rel[i] = __ldcg(&G->cand_rel[i]);
          cand_j[i] = __ldcg(&G->cand_j[i]);
          cand_pos[i] = __ldcg(&G->cand_pos[i]);
        }
        __syncthreads();
        int* kc_j = reinterpret_cast<int*>(hist);        // the histogram's memory is free now
        int* kc_pos = kc_j + kCand;
        if (mode == 2) {
          rank_cut(cand_rel, cand_j, cnt, s_vals[1], &s_cut_rel, &s_cut_j);
          __syncthreads();
          // the kept members sorted by index (hence grouped by CTA slice)
          const uint32_t crel = s_cut_rel;
          const int cj = s_cut_j;
          for (int i = tid; i < cnt; i += kCThreads) {
            if (!at_or_above(cand_rel[i], cand_j[i], crel, cj)) continue;
            int rank = 0;
            for (int q = 0; q < cnt; ++q)
              rank += cand_j[q] < cand_j[i] && at_or_above(cand_rel[q], cand_j[q], crel, cj);
            kc_j[rank] = cand_j[i];
            kc_pos[rank] = cand_pos[i];
          }
          if (tid == 0) s_nkc = need - pre[kMaxSplits];
        } else if (tid == 0) {
          s_nkc = 0;
        }
        __syncthreads();
        // kc_beg[r]: kept members in the slices before r
        const int nkc = s_nkc;
        for (int r = tid; r <= S; r += kCThreads) {
          const int jr = slice_begin(r, Mo, S);
          int cntr = 0;
          for (int q = 0; q < nkc; ++q) cntr += kc_j[q] < jr;
          kc_beg[r] = cntr;
        }
        __syncthreads();
      } else {
        crowded = 1;
      }
    }
  }

  // ------------------------------------------------------ this CTA's share
  const int lo = static_cast<int>(static_cast<int64_t>(s) * n / S);
  const int hi = static_cast<int>(static_cast<int64_t>(s + 1) * n / S);
  const int share = hi - lo;
  int32_t* sel_out = c.sel + bh * n;
  if (crowded) {
    // all key offsets of the group in shared memory, the cut by radix passes,
    // then the kept blocks in index order
    uint32_t* keys = reinterpret_cast<uint32_t*>(tiles);
    const uint32_t base = s_base;
    for (int j = tid; j < Mo; j += kCThreads) keys[j] = score_key(__ldcg(c.scores + bh * M + j)) - base;
    __syncthreads();
    const int top = 32 - __clz(s_vals[4] - base);
    const int shift = top > 11 ? top - 11 : 0;
    crowded_cut(keys, Mo, s_vals[0] << shift, s_vals[1], shift, hist, wtot, s_vals, &s_cut_j);
    const uint32_t crel = s_vals[0];
    const int cj = s_cut_j;
    const int per = (Mo + kCThreads - 1) / kCThreads;
    const int jb = min(Mo, tid * per), je = min(Mo, jb + per);
    uint32_t cnt = 0;
    for (int j = jb; j < je; ++j) cnt += at_or_above(keys[j], j, crel, cj);
    uint32_t pos = block_exclusive_scan(cnt, wtot, &s_vals[6]);
    for (int j = jb; j < je; ++j) {
      if (at_or_above(keys[j], j, crel, cj)) {
        if (static_cast<int>(pos) >= lo && static_cast<int>(pos) < hi) ids[pos - lo] = j;
        ++pos;
      }
    }
    __syncthreads();
    for (int p = lo + tid; p < hi; p += kCThreads) {
      if (p == need) ids[p - lo] = M - 1;
      sel_out[p] = ids[p - lo];
    }
  } else {
    const int* kc_j = reinterpret_cast<const int*>(hist);
    const int* kc_pos = kc_j + kCand;
    for (int p = lo + tid; p < hi; p += kCThreads) {
      int id;
      if (p == need) {
        id = M - 1;                                // the newest block, always kept
      } else if (!rounds || all_equal) {
        id = p;                                    // every block (n = M) or the lowest indices
      } else {
        // slice r: the last with pre[r] + kc_beg[r] <= p
        int r = 0, r_hi = S;
        while (r_hi - r > 1) {
          const int mid = (r + r_hi) >> 1;
          if (pre[mid] + kc_beg[mid] <= p) r = mid; else r_hi = mid;
        }
        const int o = p - pre[r] - kc_beg[r];
        id = -1;
        int before = 0;
        for (int q = kc_beg[r]; q < kc_beg[r + 1]; ++q) {
          const int mp = kc_pos[q] + (q - kc_beg[r]);  // its place in the slice's list
          if (mp == o) { id = kc_j[q]; break; }
          before += mp < o;
        }
        if (id < 0) id = __ldcg(c.kept + bh * M + slice_begin(r, Mo, S) + (o - before));
      }
      ids[p - lo] = id;
      sel_out[p] = id;
    }
  }
  // the tile area was last written by copies and read by this CTA's threads;
  // order those accesses before the tile copies that reuse it
  fence_proxy_async_smem();
  __syncthreads();

  // ------------------------------------------------------ 3. attention and merge
  const int my_count = share > warp ? (share - warp + kCW - 1) / kCW : 0;
  const int64_t row_base = bh * a.L_max;
  auto block_of = [&](int k) -> int {
    const int j = ids[warp + k * kCW];
    return (j >= 0 && j < M) ? j : -1;
  };
  float o[KT][4];
  float m0, m1, l0, l1;
  const bool ok = stream_bf16<D, kCW, kCStages>(&tmK, &tmV, tiles, bars, block_of, my_count,
                                                row_base, c.len, qb, a.scale_log2, a.ctrl, o, m0,
                                                m1, l0, l1);
  grid_launch_dependents();
  const bool merged = finish_bf16<D, kCW, kCStages>(a, tiles, ok, o, m0, m1, l0, l1, b, g, s);
  if (merged) {
    // every CTA of the group has passed all rounds: return its state to zero
    for (int i = tid; i < kBins; i += kCThreads) G->hist[i] = 0u;
    if (tid == 0) {
      G->ctr = 0;
      G->mninv = 0u;
      G->mx = 0u;
      G->ccount = 0;
    }
  }
}

// ---------------------------------------------------------------------- host
size_t coop_group_bytes() { return (sizeof(CoopGroup) + 255) / 256 * 256; }

bool coop_supported(const Shape& s, int M, int n, int S) {
  if (!s.bf16 || S < 1 || S > kMaxSplits) return false;
  const int Mo = M - 1;
  if (Mo > kCMaxKeys) return false;
  if ((Mo + S - 1) / S > kCSlice) return false;
  if ((n + S - 1) / S > kCMaxShare) return false;
  return true;
}

template <int D>
static cudaError_t coop_t(const CoopLaunch& L, cudaStream_t st) {
  using Cfg = CoopCfg<D>;
  static std::atomic<bool> attr_set[64];   // per device; launches may come from several host threads
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(decode_coop_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kDyn);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const Shape& s = L.s;
  CoopArgs c{};
  c.q = static_cast<const __nv_bfloat16*>(L.q);
  c.k_new = static_cast<const __nv_bfloat16*>(L.k_new);
  c.v_new = static_cast<const __nv_bfloat16*>(L.v_new);
  c.k = static_cast<__nv_bfloat16*>(L.k);
  c.v = static_cast<__nv_bfloat16*>(L.v);
  c.desc = static_cast<__nv_bfloat16*>(L.desc);
  c.sel = L.sel;
  c.scores = L.scores;
  c.kept = L.kept;
  c.grp = reinterpret_cast<CoopGroup*>(L.groups);
  c.len = L.len;
  c.Mmax = s.Mmax;
  c.M = L.M;
  c.n = L.n;
  c.S = L.S;
  AttnK& a = c.a;
  a.q = L.q; a.sel = nullptr; a.part_o = L.part_o; a.part_ml = L.part_ml; a.counters = L.counters;
  a.ctrl = L.ctrl; a.k = L.k; a.v = L.v; a.out = L.out; a.lse = L.lse;
  a.len0 = L.len; a.L_max = s.L_max; a.R = 1; a.Hq = s.Hq; a.H = s.H; a.G = s.G;
  a.n_sel = L.n; a.S = L.S;
  a.scale_log2 = L.scale * 1.4426950408889634f;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.S, s.H, s.B);
  cfg.blockDim = dim3(kCThreads);
  cfg.dynamicSmemBytes = Cfg::kDyn;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_coop_kernel<D>, *L.tm_k, *L.tm_v, *L.tm_d, c);
}

cudaError_t launch_decode_coop(const CoopLaunch& L, cudaStream_t st) {
  return L.s.D == 128 ? coop_t<128>(L, st) : coop_t<64>(L, st);
}

}  // namespace resa
