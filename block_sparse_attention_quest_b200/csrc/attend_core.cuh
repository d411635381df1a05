// Pieces of the split-KV attention shared by the attention kernels of
// attend.cu and the one-launch decode kernel of decode_coop.cu: the kernel
// argument block, the per-warp bf16 streaming loop (TMA tile ring, warp MMA,
// online softmax) and the merge of the per-warp and per-CTA partials.
//
// "Rectified Sparse Attention" (pith.science review), section "What carries
// the argument": all heads of a GQA group read the same selected key blocks;
// Eq. 2 (minor comment 3) masks token k through its block floor(k / b); the
// split/merge schedule follows Flash-Decoding (reference list of the page).
#pragma once

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
// Returns true in the CTA that wrote the group's final output (the only CTA
// when S == 1, else the last one to arrive); false in the others.
template <typename T, int D, int NW>
__device__ __forceinline__ bool cta_finish(const AttnK& a, float* sm, int br, int g, int s_idx) {
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
  if (a.S == 1) return true;
  // arrival: one acquire-release add after the CTA barrier releases every
  // thread's partial (cumulativity) and, for the last CTA, acquires all others'
  __syncthreads();
  int* counter = a.counters + static_cast<int64_t>(br) * a.H + g;
  if (threadIdx.x == 0) s_last = atomic_add_acq_rel(counter, 1) == a.S - 1;
  __syncthreads();
  if (!s_last) return false;
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
    return true;
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
  return true;
}

// ---------------------------------------------------------------------- bf16
template <int D, int NW, int STAGES>
struct Bf16Cfg {
  static constexpr int kHalf = 16 * 64 * 2;            // one 16 x 64 bf16 box (2 KB)
  static constexpr int kHalves = D / 64;
  static constexpr int kTile = 2 * kHalves * kHalf;    // K and V of one block
  static constexpr int kSmem = NW * STAGES * kTile + 1024;
};


// Stream one warp's blocks through its private ring of STAGES K/V tiles and
// fold them into the online softmax. block_of(k) gives the warp's k-th block
// id (k < my_count); -1 marks an id out of range, which is skipped and
// flagged. Tiles are 2-D TMA copies with 128-byte swizzle (conflict-free
// ldmatrix). S^T = K q^T (16 tokens x 8 head columns, k = head_dim) and
// O^T += V^T P^T run on warp-level mma.sync; P enters the second product as
// bf16. Tokens at or past len_r are masked and their V rows zeroed. Returns
// false (time-out raised) when a tile did not arrive in time; the copies
// still in flight are drained before returning.
template <int D, int NW, int STAGES, typename BlockOf>
__device__ __forceinline__ bool stream_bf16(const CUtensorMap* tmK, const CUtensorMap* tmV,
                                            uint8_t* tiles, uint64_t (*bars)[STAGES],
                                            BlockOf block_of, int my_count, int64_t row_base,
                                            int64_t len_r, const uint32_t (&qb)[D / 16][2],
                                            float sl2, Ctrl* ctrl, float (&o)[D / 16][4],
                                            float& m0, float& m1, float& l0, float& l1) {
  using Cfg = Bf16Cfg<D, NW, STAGES>;
  constexpr int KT = D / 16;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gq = lane >> 2;
  auto issue = [&](int k) {
    const int st = k % STAGES;
    const int j = max(block_of(k), 0);   // a bad id still completes the stage (block 0)
    const int y = static_cast<int>(row_base + static_cast<int64_t>(j) * kBlock);
    uint8_t* t = tiles + (warp * STAGES + st) * Cfg::kTile;
    mbar_arrive_expect_tx(&bars[warp][st], Cfg::kTile);
#pragma unroll
    for (int hf = 0; hf < Cfg::kHalves; ++hf) {
      tma_load_2d(t + hf * Cfg::kHalf, tmK, hf * 64, y, &bars[warp][st]);
      tma_load_2d(t + (Cfg::kHalves + hf) * Cfg::kHalf, tmV, hf * 64, y, &bars[warp][st]);
    }
  };
  if (lane == 0) {
    for (int k = 0; k < my_count && k < STAGES; ++k) issue(k);
  }
#pragma unroll
  for (int mt = 0; mt < KT; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  m0 = -INFINITY; m1 = -INFINITY; l0 = 0.f; l1 = 0.f;
  // ldmatrix row/chunk owned by this lane
  const int kq_row = (lane & 7) + (((lane >> 3) & 1) << 3);   // K (non-trans) row
  const int kq_chk = lane >> 4;                                // + 2*kk
  const int vt_row = (lane & 7) + ((lane >> 4) << 3);          // V (trans) row
  const int vt_chk = (lane >> 3) & 1;                          // + 2*mt
  bool ok = true;
  int k = 0;
  for (; k < my_count; ++k) {
    const int st = k % STAGES;
    const bool arrived = mbar_wait_bounded(&bars[warp][st], (k / STAGES) & 1, ctrl);
    if (!__all_sync(0xffffffffu, arrived)) { ok = false; break; }
    const int j = block_of(k);
    if (j < 0) {                               // skip the block, report it
      if (lane == 0) raise_error(ctrl, kErrBadIndex);
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
  if (!ok) {
    // drain the copies this warp still has in flight (bounded), then leave
    // without writing a partial; the host sees the error flag
    for (int kk = k; kk < my_count && kk < k + STAGES; ++kk)
      mbar_wait_bounded(&bars[warp][kk % STAGES], (kk / STAGES) & 1, ctrl);
  }
  return ok;
}

// The q^T fragments of the B operand: lane (gq = lane / 4, c = lane % 4)
// holds head gq, channels kk*16 + 2c, +1 (b0) and kk*16 + 8 + 2c, +1 (b1);
// heads at or past G are zero.
template <int D>
__device__ __forceinline__ void load_q_frags(const __nv_bfloat16* qgroup, int G,
                                             uint32_t (&qb)[D / 16][2]) {
  const int lane = threadIdx.x & 31;
  const int gq = lane >> 2, cq = lane & 3;
  const __nv_bfloat16* qrow = qgroup + static_cast<int64_t>(gq) * D;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    if (gq < G) {
      qb[kk][0] = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * cq);
      qb[kk][1] = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 8 + 2 * cq);
    } else {
      qb[kk][0] = 0u;
      qb[kk][1] = 0u;
    }
  }
}

// After the streaming loops of all warps: merge the warps' partials in shared
// memory (reusing the tile area) and the CTAs' through cta_finish. Returns
// true in the CTA that wrote the group's output; false in the others and when
// any warp of the CTA failed (nothing is written then).
template <int D, int NW, int STAGES>
__device__ __forceinline__ bool finish_bf16(const AttnK& a, uint8_t* tiles, bool ok,
                                            float (&o)[D / 16][4], float m0, float m1, float l0,
                                            float l1, int br, int g, int s_idx) {
  using Cfg = Bf16Cfg<D, NW, STAGES>;
  constexpr int KT = D / 16;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gq = lane >> 2, cq = lane & 3;
  const bool cta_ok = __syncthreads_and(ok);
  if (!cta_ok) return false;

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
  return cta_finish<__nv_bfloat16, D, NW>(a, sm, br, g, s_idx);
}

}  // namespace resa
