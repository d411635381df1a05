// Dense rectification attention on the 5th-generation tensor cores.
//
// "Rectified Sparse Attention" (pith.science review), section "What carries
// the argument": after every f decode steps the newest f tokens are encoded
// again by one dense causal pass. For one KV head the f query rows of its G
// query heads attend to the same keys, so the f*G rows form the M dimension
// of a real dense contraction: S = Q K^T (M = 128 rows, N = 128 keys,
// K = head_dim) and O += P V (M = 128, N = head_dim, K = 128 keys).
//
// One CTA per (KV split, KV head, batch x 128-row tile); 9 warps:
//   warps 0-3 and 4-7  two softmax warpgroups; group w takes the key tiles
//              t = w (mod 2) with its own S and O accumulators in TMEM, so one
//              group's softmax overlaps the other group's MMAs. One query row
//              per thread (= TMEM lane): row maximum, causal mask on the tiles
//              that cross it only, P = 2^(s * scale - m) written as bf16 pairs
//              into tensor memory over the S columns it was computed from (the
//              A operand of the PV product), O rescaled in TMEM only when the
//              running maximum grows by more than 2^8; the two groups'
//              (m, l, O) are merged at the end;
//   warp 8     one thread issues the TMA copies (Q once; K and V of each tile
//              into a ring of three shared-memory stages, K and V on separate
//              barriers so the next keys stream in while a tile is in its
//              softmax) and the tcgen05.mma instructions, with completion
//              signalled by tcgen05.commit on mbarriers.
// The row order inside a tile is m = i * G + h (query i of head h of the
// group), which is exactly the layout of q_f[b][i][g*G + h][:] viewed as a
// 3-D tensor, so Q arrives by one box per 64-channel half.
//
// Keys past the end of the cache (the padded tail of the last tile) are
// masked in S and their V rows are zeroed in shared memory before the PV
// product, so stale cache contents never reach an output.
//
// In a rectification the kernel is launched as a programmatic dependent of
// the kernel that writes the f new rows into the cache: only the CTAs whose
// key range reaches those rows wait for it before their first copy, the rest
// start streaming at once. The split merge is launched the same way and
// waits for this grid before reading the partials.
#include <type_traits>

#include "launch.h"
#include "tc.cuh"

namespace resa {

struct RectK {
  void* out;             // [B][f][Hq][D] bf16 (used when S == 1)
  float* part_o;         // [S][units][128][D], each row's float4 units swizzled
  float* part_ml;        // [S][units][128][2]
  Ctrl* ctrl;
  int64_t len;
  int64_t L_max;
  const int32_t* lens;   // optional per-row lengths [B] (len: their bound)
  const int32_t* windows;  // optional per-row windows [B] in [0, f]
  __nv_bfloat16* desc;   // prefill: descriptors of the queries' own tokens, or nullptr
  int64_t Mmax;
  int B, H, Hq, G, f, S, mtiles;   // units = B * H * mtiles: (b, g, m-tile) = unit
  float scale_log2;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// A staged output row of D fp32 values occupies its own D * 4 bytes as D/4
// float4 units, unit j of row r at j ^ (r mod D/4): conflict-free both when
// one thread writes its own row and when one warp reads a whole row. The
// split partials keep this order in global memory (the merge undoes it).
template <int D>
__device__ __forceinline__ int stage_slot(int r, int j) {
  constexpr int NJ = D / 4;
  return r * NJ + (j ^ (r & (NJ - 1)));
}

// First row of the partials of split s for unit (b, g, m-tile).
__device__ __forceinline__ int64_t partial_row(const RectK& a, int s, int b, int g, int mt) {
  const int64_t units = static_cast<int64_t>(a.B) * a.H * a.mtiles;
  const int64_t unit = (static_cast<int64_t>(b) * a.H + g) * a.mtiles + mt;
  return (s * units + unit) * 128;
}


template <int D>
struct RectCfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kHalfBytes = 128 * 128;            // [128 rows][64 bf16]
  static constexpr int kQBytes = kHalves * kHalfBytes;
  static constexpr int kKBytes = kHalves * kHalfBytes;    // K (or V) of one 128-key tile
  // K/V ring: tile t uses stage t % kStages (P lives in tensor memory)
  static constexpr int kStages = 3;
  static constexpr int kStageBytes = 2 * kKBytes;
  // at least 116 KB, so that one CTA fits an SM: a second would wait in
  // its tensor-memory allocation for the first one's 512 columns
  static constexpr int kSmem = kQBytes + kStages * kStageBytes + 1024 > 116 * 1024
                                   ? kQBytes + kStages * kStageBytes + 1024
                                   : 116 * 1024;
  static constexpr uint32_t kTmemCols = 512;              // S0 S1 O0 O1, 128 columns each
};

template <int D>
__global__ void __launch_bounds__(288, 1) rectify_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                            const __grid_constant__ CUtensorMap tmK,
                                                            const __grid_constant__ CUtensorMap tmV,
                                                            RectK a) {
  using C = RectCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_q;
  __shared__ __align__(8) uint64_t bar_kfull[C::kStages], bar_kempty[C::kStages];
  __shared__ __align__(8) uint64_t bar_vfull[C::kStages], bar_vempty[C::kStages];
  __shared__ __align__(8) uint64_t bar_s[2], bar_p[2], bar_pv[2];
  __shared__ uint32_t tmem_base_sh;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = base;
  uint8_t* sStage = sQ + C::kQBytes;
  auto sK = [&](int st) { return sStage + st * C::kStageBytes; };
  auto sV = [&](int st) { return sStage + st * C::kStageBytes + C::kKBytes; };

  // Prefill: grid z runs over (m-tile, batch row) with the m-tiles that see
  // the most keys first. Rectification: grid x runs over (m-tile, split)
  // with the m-tile fastest, so the m-tiles of one split, which stream the
  // same key tiles, run side by side and the second read of a tile hits L2.
  const bool prefill = a.desc != nullptr;
  const int s_idx = prefill ? blockIdx.x : blockIdx.x / a.mtiles, g = blockIdx.y;
  const int b = prefill ? blockIdx.z % a.B : blockIdx.z;
  const int mt = prefill ? a.mtiles - 1 - static_cast<int>(blockIdx.z / a.B)
                         : static_cast<int>(blockIdx.x % a.mtiles);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t len = row_len(a.lens, a.len, b);
  const int win = row_window(a.windows, a.f, b);   // query rows in use: 0 .. win-1
  // Launched after the kernel that writes the rectified rows into the cache
  // (programmatic dependent launch): a CTA waits for it before reading any
  // of those rows, and before it exits in any case (no-op otherwise).
  if (win == 0 || len < win || mt * 128 >= win * a.G) {   // not rectified, or no row in use
    grid_dependency_wait();
    return;
  }
  grid_launch_dependents();
  // positions of this m-tile's first and last query rows; keys past the last
  // are masked for every row, so their tiles are not visited
  const int64_t qpos_lo = len - win + (mt * 128) / a.G;
  const int rows_hi = (mt + 1) * 128 < win * a.G ? (mt + 1) * 128 : win * a.G;
  const int64_t qpos_hi = len - win + (rows_hi - 1) / a.G;
  const int n_tiles = static_cast<int>(qpos_hi / 128) + 1;
  const int t0 = static_cast<int>(static_cast<int64_t>(s_idx) * n_tiles / a.S);
  const int t1 = static_cast<int>(static_cast<int64_t>(s_idx + 1) * n_tiles / a.S);
  const int nt = t1 - t0;

  if (threadIdx.x == 0) {
    mbar_init(&bar_q, 1);
#pragma unroll
    for (int st = 0; st < C::kStages; ++st) {
      mbar_init(&bar_kfull[st], 1);
      mbar_init(&bar_kempty[st], 1);
      mbar_init(&bar_vfull[st], 1);
      mbar_init(&bar_vempty[st], 1);
    }
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      mbar_init(&bar_s[w], 1);
      mbar_init(&bar_p[w], 128);
      mbar_init(&bar_pv[w], 1);
    }
    fence_mbar_init();
  }
  if (warp == 0) tc::alloc(&tmem_base_sh, C::kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_sh;
  auto tS = [&](int w) { return tmem + 128u * w; };
  auto tO = [&](int w) { return tmem + 256u + 128u * w; };

  if (warp == 8) {
    // ------------------------------------------------------------ control
    if (lane == 0 && nt > 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const int rows_per_q = 128 / a.G;
      mbar_arrive_expect_tx(&bar_q, C::kQBytes);
#pragma unroll
      for (int hf = 0; hf < C::kHalves; ++hf)
        tma_load_3d(sQ + hf * C::kHalfBytes, &tmQ, hf * 64, g * a.G, b * a.f + mt * rows_per_q,
                    &bar_q);
      const int64_t row0 = (static_cast<int64_t>(b) * a.H + g) * a.L_max;
      // rows from len - win on are rewritten by the kernel this one may
      // overlap: the first copy of a tile that reaches them waits for it
      bool waited = false;
      auto load = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int t) {
        if (!waited && static_cast<int64_t>(t0 + t + 1) * 128 > len - win) {
          grid_dependency_wait();
          waited = true;
        }
        const int y = static_cast<int>(row0 + static_cast<int64_t>(t0 + t) * 128);
        mbar_arrive_expect_tx(bar, C::kKBytes);
#pragma unroll
        for (int hf = 0; hf < C::kHalves; ++hf) tma_load_2d(dst + hf * C::kHalfBytes, map, hf * 64, y, bar);
      };
      for (int t = 0; t < nt && t < C::kStages; ++t) {
        load(&tmK, sK(t), &bar_kfull[t], t);
        load(&tmV, sV(t), &bar_vfull[t], t);
      }
      constexpr uint32_t idS = tc::idesc_bf16(128, 128, false);
      constexpr uint32_t idO = tc::idesc_bf16(128, D, true);
      const uint32_t q_addr = smem_u32(sQ);
      auto issue_qk = [&](int t) {
        const int w = t & 1, st = t % C::kStages;
        const uint32_t k_addr = smem_u32(sK(st));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kHalfBytes + (kk & 3) * 32;
          tc::mma_ss(tS(w), tc::smem_desc(q_addr + off, 16, 1024),
                     tc::smem_desc(k_addr + off, 16, 1024), idS, kk > 0);
        }
        tc::commit(&bar_s[w]);
        tc::commit(&bar_kempty[st]);
      };
      // P of tile t sits in tensor memory over S of its group: 16 keys per
      // k-step = 8 columns of bf16 pairs
      auto issue_pv = [&](int t) {
        const int w = t & 1, st = t % C::kStages;
        const uint32_t v_addr = smem_u32(sV(st));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_ts(tO(w), tS(w) + 8u * kk, tc::smem_desc(v_addr + kk * 2048, C::kHalfBytes, 1024),
                     idO, t >= 2 || kk > 0);
        tc::commit(&bar_pv[w]);
        tc::commit(&bar_vempty[st]);
      };
      bool ok = mbar_wait_bounded(&bar_q, 0, a.ctrl);
      for (int t = 0; ok && t < nt && t < 2; ++t) {
        ok = mbar_wait_bounded(&bar_kfull[t], 0, a.ctrl);
        if (!ok) break;
        tc::fence_after_sync();
        issue_qk(t);
      }
      for (int t = 0; ok && t < nt; ++t) {
        const int w = t & 1, st = t % C::kStages;
        const uint32_t ph = (t / C::kStages) & 1;      // phase of stage st for tile t
        const bool refill = t + C::kStages < nt;
        // K of tile t is no longer needed once QK(t) completed
        if (refill) {
          if (!(ok = mbar_wait_bounded(&bar_kempty[st], ph, a.ctrl))) break;
          load(&tmK, sK(st), &bar_kfull[st], t + C::kStages);
        }
        if (!(ok = mbar_wait_bounded(&bar_p[w], (t >> 1) & 1, a.ctrl))) break;
        if (!(ok = mbar_wait_bounded(&bar_vfull[st], ph, a.ctrl))) break;
        tc::fence_after_sync();
        issue_pv(t);
        // PV(t) reads P from this group's S columns, which QK(t + 2) rewrites:
        // it is issued only once PV(t) has completed
        if (!(ok = mbar_wait_bounded(&bar_vempty[st], ph, a.ctrl))) break;
        if (refill) load(&tmV, sV(st), &bar_vfull[st], t + C::kStages);
        if (t + 2 < nt) {
          const int st2 = (t + 2) % C::kStages;
          if (!(ok = mbar_wait_bounded(&bar_kfull[st2], ((t + 2) / C::kStages) & 1, a.ctrl))) break;
          tc::fence_after_sync();
          issue_qk(t + 2);
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int w = warp >> 2;                               // warpgroup: tiles t = w (mod 2)
    const int row = threadIdx.x & 127;                     // TMEM lane / tile row
    const int rg = mt * 128 + row;
    const int qi = rg / a.G;
    const int64_t qpos = len - win + qi;                   // causal limit of this row
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float sl2 = a.scale_log2;
    float m_ref = -INFINITY, l = 0.f;                      // reference max (log2 units), sum
    bool ok = true;
    int u = 0;
    for (int t = w; t < nt; t += 2, ++u) {
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar_s[w], u & 1, a.ctrl));
      if (!ok) break;
      tc::fence_after_sync();
      const int64_t key0 = static_cast<int64_t>(t0 + t) * 128;
      // keys above the smallest causal limit of the tile (or past the end of
      // the cache) exist only in the last tiles
      const bool masked = key0 + 127 > qpos_lo;
      const int lim = masked ? static_cast<int>(qpos - key0 < 127 ? qpos - key0 : 127) : 127;
      // masked keys become -inf, which the exponential below turns into 0
      auto mask = [&](float (&x)[32], int c4) {
        if (masked) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c4 * 32 + i > lim) x[i] = -INFINITY;
        }
      };
      // pass 1: row maximum as eight independent chains (a single chain of
      // 128 dependent maxima is latency-bound)
      float va[2][32];
      float mp[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) mp[j] = -INFINITY;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        tc::ld32(tS(w) + lane_off + 64 * h, va[0]);
        tc::ld32(tS(w) + lane_off + 64 * h + 32, va[1]);
        tc::wait_ld();
        mask(va[0], 2 * h);
        mask(va[1], 2 * h + 1);
#pragma unroll
        for (int i = 0; i < 32; ++i) mp[i & 7] = fmaxf(mp[i & 7], fmaxf(va[0][i], va[1][i]));
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) mp[j] = fmaxf(mp[j], mp[j + 4]);
      float mx = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])) * sl2;
      if (u > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar_pv[w], (u - 1) & 1, a.ctrl));
        if (!ok) break;
        tc::fence_after_sync();
      }
      // move the reference only when the row maximum grew by more than 2^8
      const bool need = mx > m_ref + 8.f;
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? mx : m_ref;
        const float alpha = need ? (m_ref == -INFINITY ? 0.f : ex2(m_ref - m_new)) : 1.f;
        if (u > 0) {
#pragma unroll
          for (int c4 = 0; c4 < D / 32; ++c4) {
            float o[32];
            tc::ld32(tO(w) + lane_off + c4 * 32, o);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tc::st32(tO(w) + lane_off + c4 * 32, o);
          }
          tc::wait_st();
        }
        l *= alpha;
        m_ref = m_new;
      }
      // pass 2: P = 2^(s * scale - m_ref) as bf16 pairs into TMEM columns
      // 16 c4 .. 16 c4 + 15 of S (keys 32 c4 .. 32 c4 + 31): below the columns
      // still to be read, above none the A operand needs later
      const bool live = m_ref != -INFINITY;
      const float nm = live ? -m_ref : 0.f;
      float sum = 0.f;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        float x[32];
        tc::ld32(tS(w) + lane_off + c4 * 32, x);
        tc::wait_ld();
        mask(x, c4);
        uint32_t wd[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float p0 = ex2(fmaf(x[2 * e], sl2, nm));
          float p1 = ex2(fmaf(x[2 * e + 1], sl2, nm));
          if (!live) { p0 = 0.f; p1 = 0.f; }
          sum += p0 + p1;
          wd[e] = pack_bf16x2(p0, p1);
        }
        tc::st16(tS(w) + lane_off + c4 * 16, wd);
      }
      tc::wait_st();
      l += sum;
      // V rows past the end of the cache are zeroed (0 * stale data must not
      // reach an output), once the tile's V copy, which may still be in
      // flight when its S is ready, has landed
      if (key0 + 127 >= len) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar_vfull[t % C::kStages],
                                                       (t / C::kStages) & 1, a.ctrl));
        if (!ok) break;
        if (key0 + row >= len) {
          uint8_t* vt = sV(t % C::kStages);
#pragma unroll
          for (int hf = 0; hf < C::kHalves; ++hf)
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(vt + hf * C::kHalfBytes + row * 128 + c * 16) =
                  make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      tc::fence_before_sync();
      mbar_arrive(&bar_p[w]);
    }
    const bool has = u > 0;
    if (ok && has) {
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar_pv[w], (u - 1) & 1, a.ctrl));
      tc::fence_after_sync();
    }
    // prefill: the descriptors of this m-tile's own tokens (min and max of
    // their keys per 16-token block), read from the last key tile, which holds
    // them and receives no further copy, so K is read from HBM only once
    if (a.desc != nullptr && nt > 0 && s_idx == a.S - 1 && w == ((nt - 1) & 1)) {
      const int64_t key_last = static_cast<int64_t>(t0 + nt - 1) * 128;
      const int r0 = static_cast<int>(qpos_lo - key_last);       // its first token's row
      const int ntok = 128 / a.G;
      if (row < D) {
        const uint8_t* kt = sK((nt - 1) % C::kStages);
        const int half = row >> 6, chunk = (row & 63) >> 3, e = row & 7;
        const int64_t bh = static_cast<int64_t>(b) * a.H + g;
        for (int blk = 0; blk * 16 < ntok; ++blk) {
          const int64_t tb = qpos_lo + blk * 16;
          if (tb >= len) break;
          const int cnt = len - tb < 16 ? static_cast<int>(len - tb) : 16;
          float mn = INFINITY, mx = -INFINITY;
          for (int rr = 0; rr < cnt; ++rr) {
            const int kr = r0 + blk * 16 + rr;
            const float x = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                kt + half * C::kHalfBytes + kr * 128 + ((chunk ^ (kr & 7)) << 4) + e * 2));
            mn = fminf(mn, x);
            mx = fmaxf(mx, x);
          }
          __nv_bfloat16* d = a.desc + (bh * a.Mmax + tb / 16) * 2 * D;
          d[row] = __float2bfloat16_rn(mn);
          d[D + row] = __float2bfloat16_rn(mx);
        }
      }
      // group 1 reuses this stage for its hand-over below: every thread of
      // the group has read it first
      if (w == 1) asm volatile("bar.sync 2, 128;" ::: "memory");
    }
    // combine the two warpgroups: group 1 hands O over through the K/V
    // stage of its last tile, idle once that tile's PV product has
    // completed (no copy targets it afterwards, and group 0's remaining tile
    // uses another stage); with no tile of its own, through stage 1, which
    // is never loaded then. A row's D values sit in its own D * 4 bytes of
    // the stage as float4 units, unit j at j ^ (row mod D/4): conflict-free
    // both for one thread per row and for one warp per row.
    constexpr int NJ = D / 4;                                // float4 units per row
    const int t_last1 = (nt & 1) ? nt - 2 : nt - 1;          // last odd tile
    float4* sO1 = reinterpret_cast<float4*>(sK(nt >= 2 ? t_last1 % C::kStages : 1));
    auto slot = [](int r, int j) { return stage_slot<D>(r, j); };
    if (w == 1) {
      // (m, l) of the row go to the first two columns of the group's S block,
      // unused once its last PV product has completed
      tc::st2(tS(1) + lane_off, has ? m_ref : -INFINITY, has ? l : 0.f);
#pragma unroll
      for (int c4 = 0; c4 < D / 32; ++c4) {
        float o[32];
        if (has && ok) {
          tc::ld32(tO(1) + lane_off + c4 * 32, o);
          tc::wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
          sO1[slot(row, c4 * 8 + k)] = make_float4(o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
      }
    }
    if (w == 1) tc::wait_st();
    tc::fence_before_sync();
    asm volatile("bar.sync 1, 256;" ::: "memory");
    tc::fence_after_sync();
    if (w == 0 && ok) {
      float m1, l1;
      tc::ld2(tS(1) + lane_off, m1, l1);
      tc::wait_ld();
      const float m0 = has ? m_ref : -INFINITY, l0 = has ? l : 0.f;
      const float m = fmaxf(m0, m1);
      const float a0 = m0 == -INFINITY ? 0.f : ex2(m0 - m);
      const float a1 = m1 == -INFINITY ? 0.f : ex2(m1 - m);
      const float lt = a0 * l0 + a1 * l1;
      // the combined row replaces group 1's in the stage (normalised when it
      // is the final output) ...
      const float sc = a.S == 1 ? 1.f / lt : 1.f;
      const float b0 = a0 * sc, b1 = a1 * sc;
#pragma unroll
      for (int c4 = 0; c4 < D / 32; ++c4) {
        float o[32];
        if (has) {
          tc::ld32(tO(0) + lane_off + c4 * 32, o);
          tc::wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        }
        // all eight units are read before any is written back (the
        // compiler cannot tell the slots apart, so interleaved they would
        // serialise on shared-memory latency)
        float4 y[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) y[k] = sO1[slot(row, c4 * 8 + k)];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          sO1[slot(row, c4 * 8 + k)] =
              make_float4(b0 * o[4 * k] + b1 * y[k].x, b0 * o[4 * k + 1] + b1 * y[k].y,
                          b0 * o[4 * k + 2] + b1 * y[k].z, b0 * o[4 * k + 3] + b1 * y[k].w);
      }
      // (each warp's lanes wrote exactly the 32 rows the warp stores below)
      fence_proxy_async_smem();
      __syncwarp();
      if (a.S > 1) {
        // ... and a split's partial rows of this unit form one contiguous
        // block of the workspace, copied as the stage holds it (rows past
        // the window included; the merge never reads them): one bulk copy
        // of 32 rows per warp
        const int64_t prow = partial_row(a, s_idx, b, g, mt);
        reinterpret_cast<float2*>(a.part_ml)[prow + row] = make_float2(m, lt);
        if (lane == 0) {
          const int r0 = (warp & 3) * 32;
          bulk_store(a.part_o + (prow + r0) * D, sO1 + r0 * NJ, 32 * D * 4);
          bulk_commit();
          bulk_wait_read();
        }
        __syncwarp();
      } else {
        // ... and each warp writes its 32 rows out whole (32 / NJ rows per
        // store instruction, each a contiguous run of global memory)
        constexpr int RPI = 32 / NJ;
        const int j = lane % NJ;
#pragma unroll 4
        for (int it = 0; it < 32 / RPI; ++it) {
          const int r = (warp & 3) * 32 + it * RPI + lane / NJ;
          const int rgr = mt * 128 + r;
          const int qr = rgr / a.G;
          if (qr >= win) continue;
          const int64_t orow = (static_cast<int64_t>(b) * a.f + qr) * a.Hq + g * a.G + rgr % a.G;
          const float4 x = sO1[slot(r, j)];
          *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + orow * D + 4 * j) =
              make_uint2(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w));
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::dealloc(tmem, C::kTmemCols);
  }
  grid_dependency_wait();
}

// Merge of split partials for independent rows: one warp per output row,
// each lane owning D/32 of its columns. Split s of the unit (b, g, m-tile)
// holding tile row r left (m, l) at part_ml[(s * units + unit) * 128 + r] and
// its D values at the same row of part_o, float4 unit j at position
// j ^ (r mod D/4). The merge runs online over groups of up to 32 splits
// (running maximum, rescaled sum), so every load of a group is issued before
// any is used and no separate pass over the maxima comes first.
template <int D>
__global__ void __launch_bounds__(128) merge_rows_kernel(const float* __restrict__ part_o,
                                                         const float* __restrict__ part_ml,
                                                         __nv_bfloat16* __restrict__ out,
                                                         int64_t rows, int S, int64_t units,
                                                         const int32_t* lens, int64_t len,
                                                         const int32_t* windows, int f, int H,
                                                         int Hq, int G, int mtiles) {
  constexpr int CPL = D / 32;
  constexpr int NJ = D / 4;
  using Vec = typename std::conditional<CPL == 4, float4, float2>::type;
  // the partials come from the previous kernel (programmatic dependent launch)
  grid_dependency_wait();
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int64_t rows_per_b = static_cast<int64_t>(f) * Hq;
  const int b = static_cast<int>(row / rows_per_b);
  const int qi = static_cast<int>((row % rows_per_b) / Hq);
  const int h = static_cast<int>(row % Hq);
  if (lens != nullptr || windows != nullptr) {
    const int w = row_window(windows, f, b);
    if (qi >= w || row_len(lens, len, b) < w) return;   // row not rectified
  }
  const int rg = qi * G + h % G;                         // row within the unit's tiles
  const int r = rg & 127;
  const int64_t unit = (static_cast<int64_t>(b) * H + h / G) * mtiles + (rg >> 7);
  // this lane's columns: float4 unit j (whole for D = 128, half for D = 64)
  const int j = lane * CPL / 4;
  const int col = ((j ^ (r & (NJ - 1))) * 4) + (lane * CPL) % 4;
  const float2* ml = reinterpret_cast<const float2*>(part_ml) + unit * 128 + r;
  const float* po = part_o + (unit * 128 + r) * D + col;
  const int64_t split_rows = units * 128;                 // rows between splits
  float m_run = -INFINITY, l_run = 0.f;
  float acc[CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) acc[i] = 0.f;
  for (int s0 = 0; s0 < S; s0 += 32) {
    const int ns = S - s0 < 32 ? S - s0 : 32;
    // lane u holds (m, l) of split s0 + u; every lane loads its columns of
    // all the group's splits before any is used
    const float2 p = lane < ns ? ml[(s0 + lane) * split_rows] : make_float2(-INFINITY, 0.f);
    Vec x[32];
#pragma unroll
    for (int u = 0; u < 32; ++u)
      if (u < ns) x[u] = *reinterpret_cast<const Vec*>(po + (s0 + u) * split_rows * D);
    const float m_new = fmaxf(m_run, warp_max_xor(p.x, 16, 1));
    if (m_new == -INFINITY) continue;                    // no live split yet
    const float alpha = m_run == -INFINITY ? 0.f : exp2f(m_run - m_new);
    const float w = p.x == -INFINITY ? 0.f : exp2f(p.x - m_new);
    float wl = w * p.y;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) wl += __shfl_xor_sync(0xffffffffu, wl, o);
    l_run = fmaf(l_run, alpha, wl);
#pragma unroll
    for (int i = 0; i < CPL; ++i) acc[i] *= alpha;
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const float wu = __shfl_sync(0xffffffffu, w, u);
      if (u < ns && wu != 0.f) {                        // (a split without keys adds nothing)
        const float* xv = reinterpret_cast<const float*>(&x[u]);
#pragma unroll
        for (int i = 0; i < CPL; ++i) acc[i] = fmaf(wu, xv[i], acc[i]);
      }
    }
    m_run = m_new;
  }
  const float inv = 1.f / l_run;
  __nv_bfloat16* orow = out + row * D + lane * CPL;
#pragma unroll
  for (int i = 0; i < CPL; ++i) orow[i] = __float2bfloat16_rn(acc[i] * inv);
}

// The merge is launched as a programmatic dependent of the rectification
// kernel (it waits for that grid before reading the partials), so its launch
// overlaps the kernel's tail; with the same shared-memory carveout its CTAs
// can wait on SMs that still hold a rectification CTA.
template <int D>
static cudaError_t merge_rows_t(const RectArgs& r, cudaStream_t st) {
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(merge_rows_kernel<D>,
                                         cudaFuncAttributePreferredSharedMemoryCarveout,
                                         cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  const int64_t rows = static_cast<int64_t>(r.B) * r.f * r.Hq;
  cudaLaunchConfig_t mcfg = {};
  mcfg.gridDim = dim3(static_cast<unsigned>((rows + 3) / 4));
  mcfg.blockDim = dim3(128);
  mcfg.stream = st;
  mcfg.attrs = attr;
  mcfg.numAttrs = 1;
  const int64_t units = static_cast<int64_t>(r.B) * r.H * r.mtiles;
  return cudaLaunchKernelEx(&mcfg, merge_rows_kernel<D>, static_cast<const float*>(r.part_o),
                            static_cast<const float*>(r.part_ml),
                            static_cast<__nv_bfloat16*>(r.out), rows, r.S, units, r.lens, r.len,
                            r.windows, r.f, r.H, r.Hq, r.G, r.mtiles);
}

static RectK rect_kernel_args(const RectArgs& r) {
  RectK k{};
  k.out = r.out; k.part_o = r.part_o; k.part_ml = r.part_ml; k.ctrl = r.ctrl;
  k.len = r.len; k.L_max = r.L_max; k.H = r.H; k.Hq = r.Hq; k.G = r.G; k.f = r.f; k.S = r.S;
  k.lens = r.lens; k.windows = r.windows;
  k.desc = static_cast<__nv_bfloat16*>(r.desc); k.Mmax = r.L_max / 16; k.B = r.B;
  k.mtiles = r.mtiles; k.scale_log2 = r.scale * 1.4426950408889634f;
  return k;
}

template <int D>
static cudaError_t rectify_tc_t(const RectArgs& r, cudaStream_t st) {
  using C = RectCfg<D>;
  static std::atomic<bool> attr_set[64];   // per device; launches may come from several host threads
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(rectify_tc_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const RectK k = rect_kernel_args(r);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = r.desc != nullptr ? dim3(r.S, r.H, r.B * r.mtiles)
                                   : dim3(r.S * r.mtiles, r.H, r.B);
  cfg.blockDim = dim3(288);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = r.pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, rectify_tc_kernel<D>, *r.tm_q, *r.tm_k, *r.tm_v, k);
  if (e != cudaSuccess || r.S == 1) return e;
  return merge_rows_t<D>(r, st);
}

cudaError_t launch_rectify_tc(const RectArgs& r, cudaStream_t st) {
  return r.D == 128 ? rectify_tc_t<128>(r, st) : rectify_tc_t<64>(r, st);
}

}  // namespace resa
