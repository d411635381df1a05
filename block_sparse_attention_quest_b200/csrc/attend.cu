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
// and V rows of one 16-token block, brought in by 2-D TMA tensor copies with
// 128-byte swizzle (conflict-free ldmatrix). The per-block products
// S^T = K q^T (16 tokens x 8 head columns, k = head_dim) and O^T += V^T P^T
// run on warp-level mma.sync; the softmax is the usual online update in
// float32 and the probabilities enter the second product as bf16.
//
// fp32 path: the same schedule on CUDA cores with plain loads (no tensor
// cores: fp32 inputs must keep fp32 products).
#include "launch.h"

namespace resa {

struct AttnK {
  const void* q;
  const int32_t* sel;
  float* part_o;
  float* part_ml;
  int* counters;     // [B*R*H] arrival counters of the split CTAs (zero between calls)
  Ctrl* ctrl;
  const void* k;
  const void* v;
  void* out;         // [B*R][Hq][D] in the cache dtype
  float* lse;        // [B*R][Hq] or nullptr
  int64_t len0;
  int64_t L_max;
  const int32_t* lens;   // optional per-row lengths [B] (see AttnArgs)
  const int32_t* windows;  // optional per-row query counts [B] (see AttnArgs)
  double r;
  int n_min;
  int R, Hq, H, G, n_sel, S;
  float scale_log2;
};

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

// Row stride (floats) of the per-warp outputs in shared memory: 4 floats of
// padding put the rows of heads 2c and 2c + 1 of the tensor-core layout on
// different banks.
__host__ __device__ constexpr int merge_row(int D) { return D + 4; }
// floats of shared memory the per-warp merge needs
__host__ __device__ constexpr int merge_floats(int D, int NW) { return NW * 8 * merge_row(D) + 2 * NW * 8; }

// Merge the per-warp (m, l, O) of one CTA through shared memory. With one
// split the CTA writes the normalised output; otherwise it writes its partial
// and the last CTA of the (row, group) to arrive merges all S partials
// (log-sum-exp weights) into the output and resets the arrival counter.
// sm must hold merge_floats(D, NW) floats; it is reused by the final merge.
template <typename T, int D, int NW>
__device__ __forceinline__ void cta_finish(const AttnK& a, float* sm, int br, int g, int s_idx) {
  constexpr int OR = merge_row(D);
  float* sm_o = sm;                       // [NW][8][OR]
  float* sm_m = sm + NW * 8 * OR;         // [NW][8]
  float* sm_l = sm_m + NW * 8;            // [NW][8]
  __shared__ int s_last;
  T* out = static_cast<T*>(a.out);
  const int64_t head0 = static_cast<int64_t>(br) * a.Hq + g * a.G;
  constexpr int NT = NW * 32;
  constexpr int HALF = D / 2;
  // One output channel pair (c, c + HALF) of one head per thread when the
  // group fits (G * D / 2 <= threads), so the warp weights are computed once
  // per pair; otherwise a strided walk over single channels.
  const bool paired = a.G * HALF <= NT;
  const int n_items = paired ? a.G * HALF : a.G * D;
  for (int idx = threadIdx.x; idx < n_items; idx += NT) {
    const int h = paired ? idx / HALF : idx / D;
    const int ch = paired ? idx % HALF : idx % D;
    float mstar = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) mstar = fmaxf(mstar, sm_m[w * 8 + h]);
    float o0 = 0.f, o1 = 0.f, l = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float sc = mstar == -INFINITY ? 0.f : exp2f(sm_m[w * 8 + h] - mstar);
      o0 = fmaf(sc, sm_o[(w * 8 + h) * OR + ch], o0);
      if (paired) o1 = fmaf(sc, sm_o[(w * 8 + h) * OR + ch + HALF], o1);
      l = fmaf(sc, sm_l[w * 8 + h], l);
    }
    if (a.S == 1) {
      out[(head0 + h) * D + ch] = Dt<T>::from_f(o0 / l);
      if (paired) out[(head0 + h) * D + ch + HALF] = Dt<T>::from_f(o1 / l);
      if (a.lse != nullptr && ch == 0) a.lse[head0 + h] = (mstar + log2f(l)) * 0.69314718055994531f;
    } else {
      const int64_t row = (head0 + h) * a.S + s_idx;
      a.part_o[row * D + ch] = o0;
      if (paired) a.part_o[row * D + ch + HALF] = o1;
      if (ch == 0) {
        a.part_ml[row * 2] = mstar;
        a.part_ml[row * 2 + 1] = l;
      }
    }
  }
  if (a.S == 1) return;
  // arrival: one acquire-release add after the CTA barrier releases every
  // thread's partial (cumulativity) and, for the last CTA, acquires all others'
  __syncthreads();
  int* counter = a.counters + static_cast<int64_t>(br) * a.H + g;
  if (threadIdx.x == 0) s_last = atomic_add_acq_rel(counter, 1) == a.S - 1;
  __syncthreads();
  if (!s_last) return;
  // last CTA: each thread merges its outputs over all splits.
  if (paired && a.S <= 32) {
    // common case (at most two outputs per thread, at most 32 splits): every
    // partial output and every (m, l) pair is requested before any is used,
    // so the merge costs one round trip to L2
    float x[2][32];
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int idx = threadIdx.x + it * NT;
      const int h = idx / D, ch = idx % D;
      const float* po = a.part_o + (head0 + h) * a.S * D + ch;
#pragma unroll
      for (int u = 0; u < 32; ++u)
        x[it][u] = (idx < a.G * D && u < a.S) ? __ldcg(po + static_cast<int64_t>(u) * D) : 0.f;
    }
    float* pml = sm;                                   // [G][S][2]
    float* w_s = sm + 8 * kMaxSplits * 2;             // [S][8]
    float* l_h = w_s + kMaxSplits * 8;                // [8]
    float* m_h = l_h + 8;                             // [8]
    for (int i = threadIdx.x; i < a.G * a.S * 2; i += NT) pml[i] = __ldcg(a.part_ml + head0 * a.S * 2 + i);
    __syncthreads();
    {
      const int lane = threadIdx.x & 31;
      for (int h = threadIdx.x >> 5; h < a.G; h += NW) {
        const float mv = lane < a.S ? pml[(h * a.S + lane) * 2] : -INFINITY;
        const float lv = lane < a.S ? pml[(h * a.S + lane) * 2 + 1] : 0.f;
        const float mstar = warp_max_xor(mv, 16, 1);
        const float w = mv == -INFINITY ? 0.f : exp2f(mv - mstar);
        if (lane < a.S) w_s[lane * 8 + h] = w;
        float l = w * lv;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (lane == 0) { l_h[h] = l; m_h[h] = mstar; }
      }
    }
    __syncthreads();
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int idx = threadIdx.x + it * NT;
      if (idx < a.G * D) {
        const int h = idx / D, ch = idx % D;
        float o = 0.f;
#pragma unroll
        for (int u = 0; u < 32; ++u)
          if (u < a.S) o = fmaf(w_s[u * 8 + h], x[it][u], o);
        out[(head0 + h) * D + ch] = Dt<T>::from_f(o / l_h[h]);
        if (a.lse != nullptr && ch == 0) a.lse[head0 + h] = (m_h[h] + log2f(l_h[h])) * 0.69314718055994531f;
      }
    }
    if (threadIdx.x == 0) *counter = 0;
    return;
  }
  // general case: chunks of up to 32 splits, each loaded in one round trip
  // and folded in with an online log-sum-exp
  for (int idx = threadIdx.x; idx < a.G * D; idx += NT) {
    const int h = idx / D, ch = idx % D;
    const float* po = a.part_o + (head0 + h) * a.S * D + ch;
    const float* ml = a.part_ml + (head0 + h) * a.S * 2;
    float run_m = -INFINITY, run_l = 0.f, run_o = 0.f;
    for (int sp0 = 0; sp0 < a.S; sp0 += 32) {
      float x[32], mv[32], lv[32];
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const bool in = sp0 + u < a.S;
        x[u] = in ? __ldcg(po + static_cast<int64_t>(sp0 + u) * D) : 0.f;
        mv[u] = in ? __ldcg(ml + 2 * (sp0 + u)) : -INFINITY;
        lv[u] = in ? __ldcg(ml + 2 * (sp0 + u) + 1) : 0.f;
      }
      float cm = run_m;
#pragma unroll
      for (int u = 0; u < 32; ++u) cm = fmaxf(cm, mv[u]);
      const float sc = run_m == -INFINITY ? 0.f : exp2f(run_m - cm);
      run_o *= sc;
      run_l *= sc;
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const float w = mv[u] == -INFINITY ? 0.f : exp2f(mv[u] - cm);
        run_o = fmaf(w, x[u], run_o);
        run_l = fmaf(w, lv[u], run_l);
      }
      run_m = cm;
    }
    out[(head0 + h) * D + ch] = Dt<T>::from_f(run_o / run_l);
    if (a.lse != nullptr && ch == 0) a.lse[head0 + h] = (run_m + log2f(run_l)) * 0.69314718055994531f;
  }
  if (threadIdx.x == 0) *counter = 0;
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
struct Bf16Cfg {
  static constexpr int kHalf = 16 * 64 * 2;            // one 16 x 64 bf16 box (2 KB)
  static constexpr int kHalves = D / 64;
  static constexpr int kTile = 2 * kHalves * kHalf;    // K and V of one block
  static constexpr int kSmem = NW * STAGES * kTile + 1024;
};

template <int D, int NW, int STAGES>
__global__ void __launch_bounds__(NW * 32) attend_bf16_kernel(const __grid_constant__ CUtensorMap tmK,
                                                              const __grid_constant__ CUtensorMap tmV,
                                                              AttnK a) {
  using Cfg = Bf16Cfg<D, NW, STAGES>;
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

  // q^T as the B operand: lane (gq = lane / 4, c = lane % 4) holds head gq,
  // channels kk*16 + 2c, +1 (b0) and kk*16 + 8 + 2c, +1 (b1)
  const int gq = lane >> 2, cq = lane & 3;
  uint32_t qb[KT][2];
  {
    const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(a.q) +
                                (static_cast<int64_t>(br) * a.Hq + g * a.G + gq) * D;
#pragma unroll
    for (int kk = 0; kk < KT; ++kk) {
      if (gq < a.G) {
        qb[kk][0] = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * cq);
        qb[kk][1] = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 8 + 2 * cq);
      } else {
        qb[kk][0] = 0u;
        qb[kk][1] = 0u;
      }
    }
  }

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
  auto issue = [&](int k) {
    const int st = k % STAGES;
    const int j = max(block_of(k), 0);   // a bad id still completes the stage (block 0)
    const int y = static_cast<int>(row_base + static_cast<int64_t>(j) * kBlock);
    uint8_t* t = tiles + (warp * STAGES + st) * Cfg::kTile;
    mbar_arrive_expect_tx(&bars[warp][st], Cfg::kTile);
#pragma unroll
    for (int hf = 0; hf < Cfg::kHalves; ++hf) {
      tma_load_2d(t + hf * Cfg::kHalf, &tmK, hf * 64, y, &bars[warp][st]);
      tma_load_2d(t + (Cfg::kHalves + hf) * Cfg::kHalf, &tmV, hf * 64, y, &bars[warp][st]);
    }
  };
  if (lane == 0) {
    for (int k = 0; k < my_count && k < STAGES; ++k) issue(k);
  }

  float o[KT][4];
#pragma unroll
  for (int mt = 0; mt < KT; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const float sl2 = a.scale_log2;
  // ldmatrix row/chunk owned by this lane
  const int kq_row = (lane & 7) + (((lane >> 3) & 1) << 3);   // K (non-trans) row
  const int kq_chk = lane >> 4;                                // + 2*kk
  const int vt_row = (lane & 7) + ((lane >> 4) << 3);          // V (trans) row
  const int vt_chk = (lane >> 3) & 1;                          // + 2*mt
  bool ok = true;
  int k = 0;
  for (; k < my_count; ++k) {
    const int st = k % STAGES;
    const bool arrived = mbar_wait_bounded(&bars[warp][st], (k / STAGES) & 1, a.ctrl);
    if (!__all_sync(0xffffffffu, arrived)) { ok = false; break; }
    const int j = block_of(k);
    if (j < 0) {                               // skip the block, report it
      if (lane == 0) raise_error(a.ctrl, kErrBadIndex);
      __syncwarp();
      if (lane == 0 && k + STAGES < my_count) {
        fence_proxy_async_smem();
        issue(k + STAGES);
      }
      continue;
    }
    const uint32_t tbase = smem_u32(tiles + (warp * STAGES + st) * Cfg::kTile);
    const uint32_t vbase = tbase + Cfg::kHalves * Cfg::kHalf;
    const int valid_rows = static_cast<int>(len_r - static_cast<int64_t>(j) * kBlock);
    if (valid_rows < kBlock) {
      // slots past the end of the cache: zero their V rows so that 0 * stale
      // data cannot reach the output
      uint8_t* vt = tiles + (warp * STAGES + st) * Cfg::kTile + Cfg::kHalves * Cfg::kHalf;
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
    // sacc: (token gq, head 2cq), (gq, 2cq+1), (gq+8, 2cq), (gq+8, 2cq+1)
    const int64_t t_lo = static_cast<int64_t>(j) * kBlock + gq;
    float s0 = sacc[0] * sl2, s1 = sacc[1] * sl2, s2 = sacc[2] * sl2, s3 = sacc[3] * sl2;
    if (t_lo >= len_r) { s0 = -INFINITY; s1 = -INFINITY; }
    if (t_lo + 8 >= len_r) { s2 = -INFINITY; s3 = -INFINITY; }
    float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
    mx0 = warp_max_xor(mx0, 16, 4);
    mx1 = warp_max_xor(mx1, 16, 4);
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
    // P^T as the B operand of O^T += V^T P^T
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
    if (lane == 0 && k + STAGES < my_count) {
      fence_proxy_async_smem();
      issue(k + STAGES);
    }
  }
  // The next kernel in the stream may launch once every CTA has streamed its
  // blocks (whatever it reads from this kernel it reads after its own
  // dependency wait); launched earlier its prologue would compete with the
  // stream, launched here it overlaps the merge tail.
  grid_launch_dependents();
  if (!ok) {
    // drain the copies this warp still has in flight (bounded), then leave
    // without writing a partial; the host sees the error flag
    for (int kk = k; kk < my_count && kk < k + STAGES; ++kk)
      mbar_wait_bounded(&bars[warp][kk % STAGES], (kk / STAGES) & 1, a.ctrl);
  }
  const bool cta_ok = __syncthreads_and(ok);
  if (!cta_ok) return;

  l0 += __shfl_xor_sync(0xffffffffu, l0, 4);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 8);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 16);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 4);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 8);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 16);

  // per-warp partials; head columns past G (padding of the n = 8 product)
  // are never read and not stored
  static_assert(merge_floats(D, NW) * 4 <= NW * STAGES * Cfg::kTile, "merge area");
  constexpr int OR = merge_row(D);
  float* sm = reinterpret_cast<float*>(tiles);
  float* sm_o = sm;
  float* sm_m = sm + NW * 8 * OR;
  float* sm_l = sm_m + NW * 8;
  const int h0 = 2 * cq, h1 = 2 * cq + 1;
  if (gq == 0 && h0 < a.G) {
    sm_m[warp * 8 + h0] = m0; sm_l[warp * 8 + h0] = l0;
    sm_m[warp * 8 + h1] = m1; sm_l[warp * 8 + h1] = l1;
  }
  if (h0 < a.G) {
#pragma unroll
    for (int mt = 0; mt < KT; ++mt) {
      const int ch = mt * 16 + gq;
      sm_o[(warp * 8 + h0) * OR + ch] = o[mt][0];
      sm_o[(warp * 8 + h1) * OR + ch] = o[mt][1];
      sm_o[(warp * 8 + h0) * OR + ch + 8] = o[mt][2];
      sm_o[(warp * 8 + h1) * OR + ch + 8] = o[mt][3];
    }
  }
  __syncthreads();
  cta_finish<__nv_bfloat16, D, NW>(a, sm, br, g, s_idx);
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
