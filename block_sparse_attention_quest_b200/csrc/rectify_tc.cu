// Dense rectification attention on the 5th-generation tensor cores.
//
// "Rectified Sparse Attention" (pith.science review), section "What carries
// the argument": after every f decode steps the newest f tokens are encoded
// again by one dense causal pass. For one KV head the f query rows of its G
// query heads attend to the same keys, so the f*G rows form the M dimension
// of a real dense contraction: S = Q K^T (M = 128 rows, N = 128 keys,
// K = head_dim) and O += P V (M = 128, N = head_dim, K = 128 keys).
//
// One CTA per (KV split, KV head, batch x 128-row tile); 5 warps:
//   warps 0-3  one query row per thread (= TMEM lane): read S from TMEM,
//              causal mask, online softmax in float32, write P (bf16) to
//              shared memory, rescale O in TMEM when the running maximum
//              moves by more than 2^8, and write the result at the end;
//   warp 4     one elected thread issues the TMA copies (Q once, K/V tiles of
//              128 keys in a two-stage ring) and the tcgen05.mma instructions;
//              completion is signalled with tcgen05.commit on mbarriers.
// The row order inside a tile is m = i * G + h (query i of head h of the
// group), which is exactly the layout of q_f[b][i][g*G + h][:] viewed as a
// 3-D tensor, so Q arrives by one box per 64-channel half.
//
// Keys past the end of the cache (the padded tail of the last tile) are
// masked in S and their V rows are zeroed in shared memory before the PV
// product, so stale cache contents never reach an output.
#include "launch.h"
#include "tc.cuh"

namespace resa {

struct RectK {
  void* out;             // [B][f][Hq][D] bf16 (used when S == 1)
  float* part_o;         // [B*f*Hq][S][D]
  float* part_ml;        // [B*f*Hq][S][2]
  Ctrl* ctrl;
  int64_t len;
  int64_t L_max;
  int H, Hq, G, f, S, mtiles;
  float scale_log2;
};

template <int D>
struct RectCfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kHalfBytes = 128 * 128;            // [128 rows][64 bf16]
  static constexpr int kQBytes = kHalves * kHalfBytes;
  static constexpr int kKVBytes = 2 * kHalves * kHalfBytes;
  static constexpr int kPBytes = 2 * kHalfBytes;          // [128 rows][128 keys]
  static constexpr int kStages = 2;
  static constexpr int kSmem = kQBytes + kStages * kKVBytes + kPBytes + 1024;
  static constexpr uint32_t kTmemCols = 256;              // S: cols 0..127, O: 128..
};

template <int D>
__global__ void __launch_bounds__(160, 1) rectify_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                            const __grid_constant__ CUtensorMap tmK,
                                                            const __grid_constant__ CUtensorMap tmV,
                                                            RectK a) {
  using C = RectCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_q, bar_s, bar_p, bar_pv;
  __shared__ __align__(8) uint64_t bar_full[C::kStages], bar_empty[C::kStages];
  __shared__ uint32_t tmem_base_sh;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = base;
  uint8_t* sKV = sQ + C::kQBytes;
  uint8_t* sP = sKV + C::kStages * C::kKVBytes;

  const int s_idx = blockIdx.x, g = blockIdx.y;
  const int b = blockIdx.z / a.mtiles, mt = blockIdx.z % a.mtiles;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t len = a.len;
  const int n_tiles = static_cast<int>((len + 127) / 128);
  const int t0 = static_cast<int>(static_cast<int64_t>(s_idx) * n_tiles / a.S);
  const int t1 = static_cast<int>(static_cast<int64_t>(s_idx + 1) * n_tiles / a.S);
  const int nt = t1 - t0;

  if (threadIdx.x == 0) {
    mbar_init(&bar_q, 1);
    mbar_init(&bar_s, 1);
    mbar_init(&bar_p, 128);
    mbar_init(&bar_pv, 1);
#pragma unroll
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_empty[i], 1);
    }
    fence_mbar_init();
  }
  if (warp == 0) tc::alloc(&tmem_base_sh, C::kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t tS = tmem, tO = tmem + 128;

  if (warp == 4) {
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
      auto load_kv = [&](int t) {
        const int st = t % C::kStages;
        const int y = static_cast<int>(row0 + static_cast<int64_t>(t0 + t) * 128);
        uint8_t* kv = sKV + st * C::kKVBytes;
        mbar_arrive_expect_tx(&bar_full[st], C::kKVBytes);
#pragma unroll
        for (int hf = 0; hf < C::kHalves; ++hf) {
          tma_load_2d(kv + hf * C::kHalfBytes, &tmK, hf * 64, y, &bar_full[st]);
          tma_load_2d(kv + (C::kHalves + hf) * C::kHalfBytes, &tmV, hf * 64, y, &bar_full[st]);
        }
      };
      for (int t = 0; t < nt && t < C::kStages; ++t) load_kv(t);
      constexpr uint32_t idS = tc::idesc_bf16(128, 128, false);
      constexpr uint32_t idO = tc::idesc_bf16(128, D, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t p_addr = smem_u32(sP);
      auto issue_qk = [&](int t) {
        const uint32_t k_addr = smem_u32(sKV + (t % C::kStages) * C::kKVBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kHalfBytes + (kk & 3) * 32;
          tc::mma_ss(tS, tc::smem_desc(q_addr + off, 16, 1024), tc::smem_desc(k_addr + off, 16, 1024),
                     idS, kk > 0);
        }
        tc::commit(&bar_s);
      };
      auto issue_pv = [&](int t) {
        const int st = t % C::kStages;
        const uint32_t v_addr = smem_u32(sKV + st * C::kKVBytes + C::kHalves * C::kHalfBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t poff = (kk >> 2) * C::kHalfBytes + (kk & 3) * 32;
          tc::mma_ss(tO, tc::smem_desc(p_addr + poff, 16, 1024),
                     tc::smem_desc(v_addr + kk * 2048, C::kHalfBytes, 1024), idO, t > 0 || kk > 0);
        }
        tc::commit(&bar_pv);
        tc::commit(&bar_empty[st]);
      };
      bool ok = mbar_wait_bounded(&bar_q, 0, a.ctrl) && mbar_wait_bounded(&bar_full[0], 0, a.ctrl);
      if (ok) {
        tc::fence_after_sync();
        issue_qk(0);
      }
      for (int t = 1; ok && t <= nt; ++t) {
        if (!mbar_wait_bounded(&bar_p, (t - 1) & 1, a.ctrl)) { ok = false; break; }
        tc::fence_after_sync();
        issue_pv(t - 1);
        if (t < nt) {
          if (!mbar_wait_bounded(&bar_full[t % C::kStages], (t / C::kStages) & 1, a.ctrl)) {
            ok = false;
            break;
          }
          issue_qk(t);
        }
        const int refill = t - 1 + C::kStages;
        if (refill < nt) {
          const int st = (t - 1) % C::kStages;
          if (!mbar_wait_bounded(&bar_empty[st], ((t - 1) / C::kStages) & 1, a.ctrl)) {
            ok = false;
            break;
          }
          load_kv(refill);
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax rows
    const int row = threadIdx.x;                          // TMEM lane / tile row
    const int rg = mt * 128 + row;
    const int qi = rg / a.G, hh = rg % a.G;
    const int64_t qpos = len - a.f + qi;                   // causal limit of this row
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < nt; ++t) {
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar_s, t & 1, a.ctrl));
      if (!ok) break;
      tc::fence_after_sync();
      float sv[128];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        float chunk[32];
        tc::ld32(tS + lane_off + c4 * 32, chunk);
        tc::wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[c4 * 32 + i] = chunk[i];
      }
      const int64_t key0 = static_cast<int64_t>(t0 + t) * 128;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        const float z = key0 + c > qpos ? -INFINITY : sv[c] * a.scale_log2;
        sv[c] = z;
        mx = fmaxf(mx, z);
      }
      if (t > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar_pv, (t - 1) & 1, a.ctrl));
        if (!ok) break;
        tc::fence_after_sync();
      }
      // new reference maximum only when the row maximum grew by more than 2^8
      const bool need = mx > m_ref + 8.f;
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? mx : m_ref;
        const float alpha = need ? (m_ref == -INFINITY ? 0.f : exp2f(m_ref - m_new)) : 1.f;
        if (t > 0) {
#pragma unroll
          for (int c4 = 0; c4 < D / 32; ++c4) {
            float o[32];
            tc::ld32(tO + lane_off + c4 * 32, o);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tc::st32(tO + lane_off + c4 * 32, o);
          }
          tc::wait_st();
        }
        l *= alpha;
        m_ref = m_new;
      }
      // P = exp2(s - m_ref) as bf16, K-major with 128-byte swizzle
      float sum = 0.f;
      const bool live = m_ref != -INFINITY;
#pragma unroll
      for (int c8 = 0; c8 < 16; ++c8) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float z0 = sv[c8 * 8 + 2 * e], z1 = sv[c8 * 8 + 2 * e + 1];
          const float p0 = live && z0 != -INFINITY ? exp2f(z0 - m_ref) : 0.f;
          const float p1 = live && z1 != -INFINITY ? exp2f(z1 - m_ref) : 0.f;
          sum += p0 + p1;
          w[e] = pack_bf16x2(p0, p1);
        }
        uint8_t* dst = sP + (c8 >> 3) * C::kHalfBytes + row * 128 + (((c8 & 7) ^ (row & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      l += sum;
      // V rows past the end of the cache are zeroed (0 * stale data must not
      // reach an output)
      if (key0 + row >= len) {
        uint8_t* v = sKV + ((t % C::kStages) * C::kKVBytes) + C::kHalves * C::kHalfBytes;
#pragma unroll
        for (int hf = 0; hf < C::kHalves; ++hf)
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(v + hf * C::kHalfBytes + row * 128 + c * 16) =
                make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();
      tc::fence_before_sync();
      mbar_arrive(&bar_p);
    }
    if (ok && nt > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar_pv, (nt - 1) & 1, a.ctrl));
      tc::fence_after_sync();
    }
    if (ok) {
      const bool valid = qi < a.f;
      const int64_t orow = (static_cast<int64_t>(b) * a.f + qi) * a.Hq + g * a.G + hh;
#pragma unroll
      for (int c4 = 0; c4 < D / 32; ++c4) {
        float o[32];
        if (nt > 0) {
          tc::ld32(tO + lane_off + c4 * 32, o);
          tc::wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        }
        if (valid) {
          if (a.S == 1) {
            const float inv = 1.f / l;
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + orow * D + c4 * 32;
#pragma unroll
            for (int i = 0; i < 32; i += 2)
              *reinterpret_cast<uint32_t*>(dst + i) = pack_bf16x2(o[i] * inv, o[i + 1] * inv);
          } else {
            float* dst = a.part_o + (orow * a.S + s_idx) * D + c4 * 32;
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(dst + i) = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
          }
        }
      }
      if (valid && a.S > 1) {
        a.part_ml[(orow * a.S + s_idx) * 2] = m_ref;
        a.part_ml[(orow * a.S + s_idx) * 2 + 1] = l;
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::dealloc(tmem, C::kTmemCols);
  }
}

// Merge of split partials for independent rows: one warp per row.
template <int D>
__global__ void __launch_bounds__(128) merge_rows_kernel(const float* __restrict__ part_o,
                                                         const float* __restrict__ part_ml,
                                                         __nv_bfloat16* __restrict__ out,
                                                         int64_t rows, int S) {
  constexpr int CPL = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float* ml = part_ml + row * S * 2;
  float mstar = -INFINITY;
  for (int s = lane; s < S; s += 32) mstar = fmaxf(mstar, ml[2 * s]);
  mstar = warp_max_xor(mstar, 16, 1);
  float lsum = 0.f;
  for (int s = lane; s < S; s += 32) {
    const float m = ml[2 * s];
    lsum += m == -INFINITY ? 0.f : exp2f(m - mstar) * ml[2 * s + 1];
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  float acc[CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) acc[i] = 0.f;
  const float* po = part_o + row * S * D + lane * CPL;
  int s = 0;
  for (; s + 4 <= S; s += 4) {
    float w[4], x[4][CPL];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float m = ml[2 * (s + u)];
      w[u] = m == -INFINITY ? 0.f : exp2f(m - mstar);
#pragma unroll
      for (int i = 0; i < CPL; ++i) x[u][i] = po[static_cast<int64_t>(s + u) * D + i];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int i = 0; i < CPL; ++i) acc[i] = fmaf(w[u], x[u][i], acc[i]);
  }
  for (; s < S; ++s) {
    const float m = ml[2 * s];
    const float w = m == -INFINITY ? 0.f : exp2f(m - mstar);
#pragma unroll
    for (int i = 0; i < CPL; ++i) acc[i] = fmaf(w, po[static_cast<int64_t>(s) * D + i], acc[i]);
  }
  const float inv = 1.f / lsum;
  __nv_bfloat16* orow = out + row * D + lane * CPL;
#pragma unroll
  for (int i = 0; i < CPL; ++i) orow[i] = __float2bfloat16_rn(acc[i] * inv);
}

template <int D>
static cudaError_t rectify_tc_t(const RectArgs& r, cudaStream_t st) {
  using C = RectCfg<D>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(rectify_tc_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  RectK k{};
  k.out = r.out; k.part_o = r.part_o; k.part_ml = r.part_ml; k.ctrl = r.ctrl;
  k.len = r.len; k.L_max = r.L_max; k.H = r.H; k.Hq = r.Hq; k.G = r.G; k.f = r.f; k.S = r.S;
  k.mtiles = r.mtiles; k.scale_log2 = r.scale * 1.4426950408889634f;
  dim3 grid(r.S, r.H, r.B * r.mtiles);
  rectify_tc_kernel<D><<<grid, 160, C::kSmem, st>>>(*r.tm_q, *r.tm_k, *r.tm_v, k);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || r.S == 1) return e;
  const int64_t rows = static_cast<int64_t>(r.B) * r.f * r.Hq;
  merge_rows_kernel<D><<<static_cast<unsigned>((rows + 3) / 4), 128, 0, st>>>(
      r.part_o, r.part_ml, static_cast<__nv_bfloat16*>(r.out), rows, r.S);
  return cudaGetLastError();
}

cudaError_t launch_rectify_tc(const RectArgs& r, cudaStream_t st) {
  return r.D == 128 ? rectify_tc_t<128>(r, st) : rectify_tc_t<64>(r, st);
}

}  // namespace resa
