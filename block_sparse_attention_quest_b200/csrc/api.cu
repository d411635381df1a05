// C ABI of libresa: argument validation, workspace layout, launch plans.
// Declarations and the meaning of every argument are in include/resa.h.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdlib>
#include <mutex>

#include "../../include/resa.h"
#include "launch.h"

using namespace resa;

namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxDevices = 64;
// upper bound on co-resident CTAs assumed when sizing split partials
constexpr int kSplitCtaBound = 1024;
// largest rectification window (f) a call accepts
constexpr int kMaxRectifyRows = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DeviceInfo {
  int num_sms = 0;
};
std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_dev[dev].num_sms == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    g_dev[dev].num_sms = n;
  }
  return g_dev[dev].num_sms;
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  return g_encode;
}

// 2-D view [B*H*L_max rows][D cols] of a bf16 cache, (box_rows x 64) boxes,
// 128-byte swizzle
bool make_cache_map(CUtensorMap* m, const void* base, const Shape& s, uint32_t box_rows = 16) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(s.D),
                        static_cast<cuuint64_t>(s.B) * s.H * static_cast<cuuint64_t>(s.L_max)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(s.D) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D view [B*H*Mmax*2 rows][D cols] of bf16 descriptors (min and max rows of
// every block), 64 x 32 boxes without swizzle
bool make_desc_map(CUtensorMap* m, const void* base, const Shape& s) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(s.D),
                        static_cast<cuuint64_t>(s.B) * s.H * static_cast<cuuint64_t>(s.Mmax) * 2};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(s.D) * 2};
  cuuint32_t box[2] = {64, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D view [B*f][Hq][D] of bf16 rectify queries; a (64 x G x 128/G) box is
// one 128-row tile in the order row = query * G + head
bool make_query_map(CUtensorMap* m, const void* base, const Shape& s, int f) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(s.D), static_cast<cuuint64_t>(s.Hq),
                        static_cast<cuuint64_t>(s.B) * static_cast<cuuint64_t>(f)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(s.D) * 2,
                           static_cast<cuuint64_t>(s.Hq) * s.D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(s.G), static_cast<cuuint32_t>(128 / s.G)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool rectify_on_tensor_cores(const Shape& s) {
  return s.bf16 && (s.G == 1 || s.G == 2 || s.G == 4 || s.G == 8);
}
int rect_mtiles(const Shape& s, int f) { return (f * s.G + 127) / 128; }

int check_dims(const resa_dims* d, Shape* s) {
  if (d == nullptr) return RESA_ERR_INVALID_ARG;
  if (d->batch < 1 || d->n_kv_heads < 1 || d->n_q_heads < 1 || d->max_len < 16 ||
      d->max_len % 16 != 0)
    return RESA_ERR_INVALID_ARG;
  if (d->n_q_heads % d->n_kv_heads != 0) return RESA_ERR_INVALID_ARG;
  if (d->dtype != RESA_F32 && d->dtype != RESA_BF16) return RESA_ERR_INVALID_ARG;
  if (d->block_size != 16) return RESA_ERR_UNSUPPORTED;
  if (d->head_dim != 64 && d->head_dim != 128) return RESA_ERR_UNSUPPORTED;
  const int G = d->n_q_heads / d->n_kv_heads;
  if (G > 8) return RESA_ERR_UNSUPPORTED;
  // TMA row coordinates are signed 32-bit
  const double rows = static_cast<double>(d->batch) * d->n_kv_heads * static_cast<double>(d->max_len);
  if (rows >= 2147483648.0) return RESA_ERR_UNSUPPORTED;
  // grid.y / grid.z limits
  if (d->n_kv_heads > 65535 || static_cast<int64_t>(d->batch) * 1024 > 65535 * 1024LL)
    return RESA_ERR_UNSUPPORTED;
  s->B = d->batch;
  s->Hq = d->n_q_heads;
  s->H = d->n_kv_heads;
  s->G = G;
  s->D = d->head_dim;
  s->L_max = d->max_len;
  s->Mmax = static_cast<int>(d->max_len / 16);
  s->bf16 = d->dtype == RESA_BF16;
  return RESA_OK;
}

int64_t blocks_of(int64_t len) { return (len + 15) / 16; }

// Decode steps run as the three-kernel chain (score, select, attend, chained
// by programmatic dependent launch). RESA_DECODE_ONE_LAUNCH=1 in the
// environment runs bf16 steps at one length as one launch instead
// (decode_coop.cu), where the shape allows it: the same step, measured slower
// on B200 (its one CTA per SM streams the descriptors more slowly than the
// score kernel, and its selection rounds through L2 cost more than the
// chain's single-CTA selection).
bool one_launch_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("RESA_DECODE_ONE_LAUNCH");
    return e != nullptr && e[0] == '1';
  }();
  return on;
}

int splits_for(int units, int64_t min_blocks, int num_sms, const Shape& s) {
  const int target = num_sms * attend_ctas_per_sm(s);
  int S = units >= target ? 1 : target / units;
  const int bound = units >= kSplitCtaBound ? 1 : kSplitCtaBound / units;
  if (S > bound) S = bound;
  if (S > kMaxSplits) S = kMaxSplits;
  if (S > min_blocks) S = static_cast<int>(min_blocks);
  return S < 1 ? 1 : S;
}

// bound used for workspace sizing (independent of the device)
int64_t split_bound(int64_t units) {
  int64_t S = units >= kSplitCtaBound ? 1 : kSplitCtaBound / units;
  return S > kMaxSplits ? kMaxSplits : S;
}

struct WsLayout {
  size_t scores, sel, kept, counters, coop, part_ml, part_o, total;
};

bool coop_groups_fit(const Shape& s) {
  return s.bf16 && static_cast<int64_t>(s.B) * s.H <= kCoopMaxGroups;
}

// Control block and arrival counters come first, at offsets that depend on
// the dims only: they must stay put (and zero) from call to call. The scratch
// regions after them are rewritten by every call.
WsLayout ws_layout(const Shape& s, int64_t len, int32_t f) {
  WsLayout w{};
  const int64_t M = blocks_of(len);
  size_t off = kCtrlBytes;
  w.counters = off;
  off = align_up(off + static_cast<size_t>(s.B) * s.H * kMaxRectifyRows * sizeof(int));
  // per-group state of the one-launch decode step (zero between calls)
  w.coop = off;
  if (coop_groups_fit(s)) off = align_up(off + static_cast<size_t>(s.B) * s.H * coop_group_bytes());
  w.scores = off;
  off = align_up(off + static_cast<size_t>(s.B) * s.H * M * sizeof(float));
  w.sel = off;
  off = align_up(off + static_cast<size_t>(s.B) * s.H * M * sizeof(int32_t));
  w.kept = off;
  if (coop_groups_fit(s)) off = align_up(off + static_cast<size_t>(s.B) * s.H * M * sizeof(int32_t));
  // decode rows: B*Hq with units B*H; rectify rows: B*f*Hq with units B*H*f
  const int64_t dec = static_cast<int64_t>(s.B) * s.Hq * split_bound(static_cast<int64_t>(s.B) * s.H);
  // a smaller window can take more splits, so size for the largest need of
  // every window up to f (none for a decode-only workspace, f = 0)
  int64_t rec = 0;
  for (int64_t fr = 1; fr <= f; ++fr) {
    const int64_t sb = split_bound(static_cast<int64_t>(s.B) * s.H * fr);
    const int64_t need = static_cast<int64_t>(s.B) * fr * s.Hq * sb;
    if (need > rec) rec = need;
    // tensor-core path: 128 rows per (batch row, KV head, m-tile) and split
    const int64_t tc_units = static_cast<int64_t>(s.B) * s.H * rect_mtiles(s, static_cast<int>(fr));
    const int64_t need_tc = tc_units * 128 * split_bound(tc_units);
    if (need_tc > rec) rec = need_tc;
  }
  const int64_t rows = dec > rec ? dec : rec;
  w.part_ml = off;
  off = align_up(off + static_cast<size_t>(rows) * 2 * sizeof(float));
  w.part_o = off;
  off = align_up(off + static_cast<size_t>(rows) * s.D * sizeof(float));
  w.total = off;
  return w;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? RESA_OK : RESA_ERR_CUDA; }

// split-KV attention over `R` query rows + merge
int run_attention(const Shape& s, const void* q, int R, int64_t len0, const int32_t* sel, int n_sel,
                  float scale, const void* k, const void* v, void* out, float* lse, uint8_t* ws,
                  const WsLayout& w, int num_sms, cudaStream_t st, bool pdl = false,
                  const int32_t* lens = nullptr, double r = 0.0, int n_min = 0,
                  const int32_t* windows = nullptr) {
  const int64_t min_blocks = sel ? n_sel : blocks_of(len0);
  const int S = splits_for(s.B * s.H * R, min_blocks, num_sms, s);
  AttnArgs a{};
  a.q = q; a.R = R; a.len0 = len0; a.sel = sel; a.n_sel = n_sel; a.S = S; a.scale = scale;
  a.part_o = reinterpret_cast<float*>(ws + w.part_o);
  a.part_ml = reinterpret_cast<float*>(ws + w.part_ml);
  a.counters = reinterpret_cast<int*>(ws + w.counters);
  a.out = out;
  a.lse = lse;
  a.ctrl = reinterpret_cast<Ctrl*>(ws);
  a.k = k; a.v = v;
  a.pdl = pdl;
  a.lens = lens; a.windows = windows; a.r = r; a.n_min = n_min;
  CUtensorMap tk, tv;
  if (s.bf16) {
    if (!make_cache_map(&tk, k, s) || !make_cache_map(&tv, v, s)) return RESA_ERR_CUDA;
    a.tm_k = &tk;
    a.tm_v = &tv;
  }
  return cuda_status(launch_attend(s, a, st));
}

}  // namespace

namespace resa {
size_t workspace_zero_prefix(const Shape& s) { return ws_layout(s, 1, 0).scores; }
}  // namespace resa

extern "C" {

int32_t resa_num_selected(int64_t len, int32_t block_size, double r, int32_t n_min) {
  if (len < 1 || block_size != 16 || !(r > 0.0 && r <= 1.0) || n_min < 1) return RESA_ERR_INVALID_ARG;
  const int64_t M = blocks_of(len);
  int64_t n = static_cast<int64_t>(std::ceil(static_cast<double>(M) * r - 1e-9));
  if (n < n_min) n = n_min;
  if (n > M) n = M;
  return static_cast<int32_t>(n);
}

size_t resa_workspace_bytes(const resa_dims* dims, int64_t len, int32_t f) {
  Shape s;
  if (check_dims(dims, &s) != RESA_OK || len < 1 || f < 0 || f > kMaxRectifyRows) return 0;
  return ws_layout(s, len, f).total;
}

static int build_desc_impl(const resa_dims* dims, const void* k_cache, int64_t len, void* desc,
                           void* stream, const int32_t* lens) {
  Shape s;
  int rc = check_dims(dims, &s);
  if (rc != RESA_OK) return rc;
  if (!k_cache || !desc || !aligned16(k_cache) || !aligned16(desc) || len < 1) return RESA_ERR_INVALID_ARG;
  if (len > s.L_max) return RESA_ERR_CAPACITY;
  return cuda_status(
      launch_build_desc(s, k_cache, desc, len, static_cast<cudaStream_t>(stream), lens));
}

int resa_build_desc(const resa_dims* dims, const void* k_cache, int64_t len, void* desc,
                    void* stream) {
  return build_desc_impl(dims, k_cache, len, desc, stream, nullptr);
}

static bool lens_ok(const int32_t* lens) {
  return lens != nullptr && (reinterpret_cast<uintptr_t>(lens) & 3u) == 0;
}

int resa_build_desc_varlen(const resa_dims* dims, const void* k_cache, const int32_t* lens,
                           int64_t len_bound, void* desc, void* stream) {
  if (!lens_ok(lens)) return RESA_ERR_INVALID_ARG;
  return build_desc_impl(dims, k_cache, len_bound, desc, stream, lens);
}

static int check_decode_common(const resa_dims* dims, Shape* s, const void* q, const void* k_new,
                               const void* v_new, const void* k_cache, const void* v_cache,
                               int64_t len, const void* out, const void* workspace,
                               size_t workspace_bytes, int32_t f_for_ws) {
  int rc = check_dims(dims, s);
  if (rc != RESA_OK) return rc;
  if (!q || !k_cache || !v_cache || !out || !workspace) return RESA_ERR_INVALID_ARG;
  if ((k_new == nullptr) != (v_new == nullptr)) return RESA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      (k_new && (!aligned16(k_new) || !aligned16(v_new))) ||
      (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return RESA_ERR_INVALID_ARG;
  if (len < 1) return RESA_ERR_INVALID_ARG;
  if (len > s->L_max) return RESA_ERR_CAPACITY;
  if (workspace_bytes < ws_layout(*s, len, f_for_ws).total) return RESA_ERR_WORKSPACE;
  return RESA_OK;
}

static int select_impl(const resa_dims* dims, const void* q, const void* k_new,
                       const void* v_new, void* k_cache, void* v_cache, void* desc,
                       int64_t len, double r, int32_t n_min, int32_t* sel, void* workspace,
                       size_t workspace_bytes, void* stream, const int32_t* lens) {
  Shape s;
  int rc = check_decode_common(dims, &s, q, k_new, v_new, k_cache, v_cache, len, q, workspace,
                               workspace_bytes, 0);
  if (rc != RESA_OK) return rc;
  if (!desc || !aligned16(desc) || !sel) return RESA_ERR_INVALID_ARG;
  if (!(r > 0.0 && r <= 1.0) || n_min < 1) return RESA_ERR_INVALID_ARG;
  if (blocks_of(len) > 262144) return RESA_ERR_UNSUPPORTED;
  const int num_sms = device_sms();
  if (num_sms <= 0) return RESA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int M = static_cast<int>(blocks_of(len));
  const int n = resa_num_selected(len, 16, r, n_min);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const WsLayout w = ws_layout(s, len, 0);
  float* scores = reinterpret_cast<float*>(ws + w.scores);
  cudaError_t e = launch_score(s, q, desc, scores, k_new, v_new, k_cache, v_cache, desc, len,
                               num_sms, st, lens, reinterpret_cast<Ctrl*>(ws));
  if (e != cudaSuccess) return RESA_ERR_CUDA;
  return cuda_status(launch_select(s, scores, sel, M, n, st, lens, len, r, n_min));
}

int resa_select_blocks(const resa_dims* dims, const void* q, const void* k_new,
                       const void* v_new, void* k_cache, void* v_cache, void* desc,
                       int64_t len, double r, int32_t n_min, int32_t* sel, void* workspace,
                       size_t workspace_bytes, void* stream) {
  return select_impl(dims, q, k_new, v_new, k_cache, v_cache, desc, len, r, n_min, sel,
                     workspace, workspace_bytes, stream, nullptr);
}

static int attend_blocks_impl(const resa_dims* dims, const void* q, const void* k_cache,
                              const void* v_cache, int64_t len, const int32_t* sel, int32_t n_sel,
                              float softmax_scale, void* out, float* lse, void* workspace,
                              size_t workspace_bytes, void* stream, bool pdl,
                              const int32_t* lens = nullptr, double r = 0.0, int32_t n_min = 0) {
  Shape s;
  int rc = check_decode_common(dims, &s, q, nullptr, nullptr, k_cache, v_cache, len, out,
                               workspace, workspace_bytes, 0);
  if (rc != RESA_OK) return rc;
  if (!sel || n_sel < 1 || n_sel > blocks_of(len) || !(std::isfinite(softmax_scale) && softmax_scale > 0.f))
    return RESA_ERR_INVALID_ARG;
  const int num_sms = device_sms();
  if (num_sms <= 0) return RESA_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const WsLayout w = ws_layout(s, len, 0);
  return run_attention(s, q, 1, len, sel, n_sel, softmax_scale, k_cache, v_cache, out, lse, ws, w,
                       num_sms, static_cast<cudaStream_t>(stream), pdl, lens, r, n_min);
}

int resa_attend_blocks(const resa_dims* dims, const void* q, const void* k_cache,
                       const void* v_cache, int64_t len, const int32_t* sel, int32_t n_sel,
                       float softmax_scale, void* out, float* lse, void* workspace,
                       size_t workspace_bytes, void* stream) {
  return attend_blocks_impl(dims, q, k_cache, v_cache, len, sel, n_sel, softmax_scale, out, lse,
                            workspace, workspace_bytes, stream, false);
}

static int decode_sparse_impl(const resa_dims* dims, const void* q, const void* k_new,
                              const void* v_new, void* k_cache, void* v_cache, void* desc,
                              int64_t len, double r, int32_t n_min, float softmax_scale,
                              void* out, float* lse, int32_t* sel, void* workspace,
                              size_t workspace_bytes, void* stream, const int32_t* lens) {
  Shape s;
  int rc = check_decode_common(dims, &s, q, k_new, v_new, k_cache, v_cache, len, out, workspace,
                               workspace_bytes, 0);
  if (rc != RESA_OK) return rc;
  if (!desc || !aligned16(desc)) return RESA_ERR_INVALID_ARG;
  if (!(r > 0.0 && r <= 1.0) || n_min < 1 || !(std::isfinite(softmax_scale) && softmax_scale > 0.f)) return RESA_ERR_INVALID_ARG;
  const int n = resa_num_selected(len, 16, r, n_min);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const WsLayout w = ws_layout(s, len, 0);
  int32_t* selp = sel ? sel : reinterpret_cast<int32_t*>(ws + w.sel);
  if (s.bf16 && lens == nullptr && one_launch_enabled() && coop_groups_fit(s)) {
    // one launch: the CTAs of each KV group score their slices, agree on the
    // exact top-n cut through the workspace and attend to equal shares
    const int num_sms = device_sms();
    if (num_sms <= 0) return RESA_ERR_CUDA;
    const int M = static_cast<int>(blocks_of(len));
    const int S = splits_for(s.B * s.H, n, num_sms, s);
    if (coop_supported(s, M, n, S)) {
      CoopLaunch c{};
      c.s = s; c.q = q; c.k_new = k_new; c.v_new = v_new; c.k = k_cache; c.v = v_cache;
      c.desc = desc; c.out = out; c.lse = lse; c.sel = selp;
      c.scores = reinterpret_cast<float*>(ws + w.scores);
      c.kept = reinterpret_cast<int32_t*>(ws + w.kept);
      c.groups = ws + w.coop;
      c.part_o = reinterpret_cast<float*>(ws + w.part_o);
      c.part_ml = reinterpret_cast<float*>(ws + w.part_ml);
      c.counters = reinterpret_cast<int*>(ws + w.counters);
      c.ctrl = reinterpret_cast<Ctrl*>(ws);
      c.len = len; c.M = M; c.n = n; c.S = S; c.scale = softmax_scale;
      CUtensorMap tk, tv, td;
      if (!make_cache_map(&tk, k_cache, s) || !make_cache_map(&tv, v_cache, s) ||
          !make_desc_map(&td, desc, s))
        return RESA_ERR_CUDA;
      c.tm_k = &tk; c.tm_v = &tv; c.tm_d = &td;
      return cuda_status(launch_decode_coop(c, static_cast<cudaStream_t>(stream)));
    }
  }
  rc = select_impl(dims, q, k_new, v_new, k_cache, v_cache, desc, len, r, n_min, selp,
                   workspace, workspace_bytes, stream, lens);
  if (rc != RESA_OK) return rc;
  // the attention kernel is a programmatic dependent of the select kernel:
  // its prologue overlaps the selection, it reads the block list after it
  return attend_blocks_impl(dims, q, k_cache, v_cache, len, selp, n, softmax_scale, out, lse,
                            workspace, workspace_bytes, stream, true, lens, r, n_min);
}

int resa_decode_sparse(const resa_dims* dims, const void* q, const void* k_new,
                       const void* v_new, void* k_cache, void* v_cache, void* desc,
                       int64_t len, double r, int32_t n_min, float softmax_scale, void* out,
                       float* lse, int32_t* sel, void* workspace, size_t workspace_bytes,
                       void* stream) {
  return decode_sparse_impl(dims, q, k_new, v_new, k_cache, v_cache, desc, len, r, n_min,
                            softmax_scale, out, lse, sel, workspace, workspace_bytes, stream,
                            nullptr);
}

int resa_decode_sparse_varlen(const resa_dims* dims, const void* q, const void* k_new,
                              const void* v_new, void* k_cache, void* v_cache, void* desc,
                              const int32_t* lens, int64_t len_bound, double r, int32_t n_min,
                              float softmax_scale, void* out, float* lse, int32_t* sel,
                              void* workspace, size_t workspace_bytes, void* stream) {
  if (!lens_ok(lens)) return RESA_ERR_INVALID_ARG;
  return decode_sparse_impl(dims, q, k_new, v_new, k_cache, v_cache, desc, len_bound, r, n_min,
                            softmax_scale, out, lse, sel, workspace, workspace_bytes, stream,
                            lens);
}

static int decode_dense_impl(const resa_dims* dims, const void* q, const void* k_new,
                             const void* v_new, void* k_cache, void* v_cache, void* desc,
                             int64_t len, float softmax_scale, void* out, float* lse,
                             void* workspace, size_t workspace_bytes, void* stream,
                             const int32_t* lens) {
  Shape s;
  int rc = check_decode_common(dims, &s, q, k_new, v_new, k_cache, v_cache, len, out, workspace,
                               workspace_bytes, 0);
  if (rc != RESA_OK) return rc;
  if (desc && !aligned16(desc)) return RESA_ERR_INVALID_ARG;
  if (!(std::isfinite(softmax_scale) && softmax_scale > 0.f)) return RESA_ERR_INVALID_ARG;
  const int num_sms = device_sms();
  if (num_sms <= 0) return RESA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const WsLayout w = ws_layout(s, len, 0);
  if (k_new) {
    cudaError_t e = launch_append(s, k_new, v_new, k_cache, v_cache, desc, len, st, lens);
    if (e != cudaSuccess) return RESA_ERR_CUDA;
  }
  return run_attention(s, q, 1, len, nullptr, 0, softmax_scale, k_cache, v_cache, out, lse, ws, w,
                       num_sms, st, false, lens);
}

int resa_decode_dense(const resa_dims* dims, const void* q, const void* k_new,
                      const void* v_new, void* k_cache, void* v_cache, void* desc, int64_t len,
                      float softmax_scale, void* out, float* lse, void* workspace,
                      size_t workspace_bytes, void* stream) {
  return decode_dense_impl(dims, q, k_new, v_new, k_cache, v_cache, desc, len, softmax_scale, out,
                           lse, workspace, workspace_bytes, stream, nullptr);
}

int resa_decode_dense_varlen(const resa_dims* dims, const void* q, const void* k_new,
                             const void* v_new, void* k_cache, void* v_cache, void* desc,
                             const int32_t* lens, int64_t len_bound, float softmax_scale,
                             void* out, float* lse, void* workspace, size_t workspace_bytes,
                             void* stream) {
  if (!lens_ok(lens)) return RESA_ERR_INVALID_ARG;
  return decode_dense_impl(dims, q, k_new, v_new, k_cache, v_cache, desc, len_bound,
                           softmax_scale, out, lse, workspace, workspace_bytes, stream, lens);
}

static int rectify_impl(const resa_dims* dims, const void* q_f, const void* k_f, const void* v_f,
                        void* k_cache, void* v_cache, void* desc, int64_t len, int32_t f,
                        float softmax_scale, void* out_f, void* workspace,
                        size_t workspace_bytes, void* stream, const int32_t* lens,
                        const int32_t* windows) {
  Shape s;
  int rc = check_dims(dims, &s);
  if (rc != RESA_OK) return rc;
  if (f < 1 || f > kMaxRectifyRows) return RESA_ERR_INVALID_ARG;
  rc = check_decode_common(dims, &s, q_f, k_f, v_f, k_cache, v_cache, len, out_f, workspace,
                               workspace_bytes, f);
  if (rc != RESA_OK) return rc;
  if (!k_f || !desc || !aligned16(desc)) return RESA_ERR_INVALID_ARG;
  if (f > len || !(std::isfinite(softmax_scale) && softmax_scale > 0.f)) return RESA_ERR_INVALID_ARG;
  const int num_sms = device_sms();
  if (num_sms <= 0) return RESA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const WsLayout w = ws_layout(s, len, f);
  cudaError_t e = launch_rectify_write(s, k_f, v_f, k_cache, v_cache, desc, len, f, st, lens,
                                       windows, reinterpret_cast<Ctrl*>(ws));
  if (e != cudaSuccess) return RESA_ERR_CUDA;
  if (rectify_on_tensor_cores(s)) {
    RectArgs r{};
    r.B = s.B; r.H = s.H; r.Hq = s.Hq; r.G = s.G; r.D = s.D; r.f = f;
    r.mtiles = rect_mtiles(s, f);
    const int units = s.B * s.H * r.mtiles;
    const int64_t n_tiles = (len + 127) / 128;
    int64_t S = units >= num_sms ? 1 : num_sms / units;
    if (S > kMaxSplits) S = kMaxSplits;
    if (S > n_tiles) S = n_tiles;
    r.S = static_cast<int>(S);
    r.len = len; r.lens = lens; r.windows = windows; r.L_max = s.L_max; r.scale = softmax_scale; r.out = out_f;
    r.part_o = reinterpret_cast<float*>(ws + w.part_o);
    r.part_ml = reinterpret_cast<float*>(ws + w.part_ml);
    r.ctrl = reinterpret_cast<Ctrl*>(ws);
    CUtensorMap tq, tk, tv;
    if (!make_query_map(&tq, q_f, s, f) || !make_cache_map(&tk, k_cache, s, 128) ||
        !make_cache_map(&tv, v_cache, s, 128))
      return RESA_ERR_CUDA;
    r.tm_q = &tq; r.tm_k = &tk; r.tm_v = &tv;
    r.pdl = true;
    return cuda_status(launch_rectify_tc(r, st));
  }
  return run_attention(s, q_f, f, len - f + 1, nullptr, 0, softmax_scale, k_cache, v_cache, out_f,
                       nullptr, ws, w, num_sms, st, false, lens, 0.0, 0, windows);
}

int resa_rectify(const resa_dims* dims, const void* q_f, const void* k_f, const void* v_f,
                 void* k_cache, void* v_cache, void* desc, int64_t len, int32_t f,
                 float softmax_scale, void* out_f, void* workspace, size_t workspace_bytes,
                 void* stream) {
  return rectify_impl(dims, q_f, k_f, v_f, k_cache, v_cache, desc, len, f, softmax_scale, out_f,
                      workspace, workspace_bytes, stream, nullptr, nullptr);
}

int resa_rectify_varlen(const resa_dims* dims, const void* q_f, const void* k_f,
                        const void* v_f, void* k_cache, void* v_cache, void* desc,
                        const int32_t* lens, const int32_t* windows, int64_t len_bound,
                        int32_t f, float softmax_scale, void* out_f, void* workspace,
                        size_t workspace_bytes, void* stream) {
  if (!lens_ok(lens) || (windows != nullptr && !lens_ok(windows))) return RESA_ERR_INVALID_ARG;
  return rectify_impl(dims, q_f, k_f, v_f, k_cache, v_cache, desc, len_bound, f, softmax_scale,
                      out_f, workspace, workspace_bytes, stream, lens, windows);
}

int resa_prefill(const resa_dims* dims, const void* q, const void* k_cache, const void* v_cache,
                 void* desc, int64_t len, float softmax_scale, void* out, void* workspace,
                 size_t workspace_bytes, void* stream) {
  Shape s;
  int rc = check_decode_common(dims, &s, q, nullptr, nullptr, k_cache, v_cache, len, out,
                               workspace, workspace_bytes, 0);
  if (rc != RESA_OK) return rc;
  if (!desc || !aligned16(desc) || !(std::isfinite(softmax_scale) && softmax_scale > 0.f))
    return RESA_ERR_INVALID_ARG;
  if (!rectify_on_tensor_cores(s)) return RESA_ERR_UNSUPPORTED;   // bf16, group 1/2/4/8
  const int64_t mt64 = (len * s.G + 127) / 128;
  if (mt64 > 65535) return RESA_ERR_UNSUPPORTED;
  const int mtiles = static_cast<int>(mt64);
  if (static_cast<int64_t>(s.B) * mtiles > 65535 || len * s.B > 2147483647LL) return RESA_ERR_UNSUPPORTED;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const WsLayout w = ws_layout(s, len, 0);
  RectArgs r{};
  r.B = s.B; r.H = s.H; r.Hq = s.Hq; r.G = s.G; r.D = s.D;
  r.f = static_cast<int>(len);          // every position is a query row
  r.mtiles = mtiles;
  r.S = 1;                              // m-tiles give the parallelism: no key splits
  r.len = len; r.L_max = s.L_max; r.scale = softmax_scale; r.out = out;
  r.part_o = reinterpret_cast<float*>(ws + w.part_o);
  r.part_ml = reinterpret_cast<float*>(ws + w.part_ml);
  r.ctrl = reinterpret_cast<Ctrl*>(ws);
  r.desc = desc;
  CUtensorMap tq, tk, tv;
  if (!make_query_map(&tq, q, s, static_cast<int>(len)) || !make_cache_map(&tk, k_cache, s, 128) ||
      !make_cache_map(&tv, v_cache, s, 128))
    return RESA_ERR_CUDA;
  r.tm_q = &tq; r.tm_k = &tk; r.tm_v = &tv;
  return cuda_status(launch_rectify_tc(r, static_cast<cudaStream_t>(stream)));
}

int resa_wait_check(const int32_t* flag, int32_t target, uint32_t limit_us, void* workspace,
                    void* stream) {
  if (!flag || (reinterpret_cast<uintptr_t>(flag) & 3u) != 0 || !workspace ||
      (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 || limit_us < 1 ||
      limit_us > 2000000u)
    return RESA_ERR_INVALID_ARG;
  return cuda_status(launch_wait_check(flag, target, static_cast<unsigned long long>(limit_us) * 1000ull,
                                       reinterpret_cast<Ctrl*>(workspace),
                                       static_cast<cudaStream_t>(stream)));
}

int resa_workspace_status(void* workspace, void* stream) {
  if (!workspace) return RESA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return RESA_ERR_CUDA;
  int err = 0;
  if (cudaMemcpy(&err, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return RESA_ERR_CUDA;
  if (err != 0) {
    const int zero = 0;
    if (cudaMemcpy(workspace, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return RESA_ERR_CUDA;
    return (err & kErrTimeout) ? RESA_ERR_TIMEOUT : RESA_ERR_BAD_INDEX;
  }
  return RESA_OK;
}

const char* resa_status_string(int status) {
  switch (status) {
    case RESA_OK: return "ok";
    case RESA_ERR_INVALID_ARG: return "invalid argument";
    case RESA_ERR_UNSUPPORTED: return "unsupported shape (head_dim 64/128, group <= 8, block 16)";
    case RESA_ERR_CAPACITY: return "len exceeds cache capacity";
    case RESA_ERR_WORKSPACE: return "workspace too small";
    case RESA_ERR_CUDA: return "CUDA error";
    case RESA_ERR_TIMEOUT: return "device-side wait timed out";
    case RESA_ERR_BAD_INDEX: return "block id or per-row length out of range";
    default: return "unknown status";
  }
}

}  // extern "C"
