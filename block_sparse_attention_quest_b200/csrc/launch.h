// Internal launchers of libresa (host side). Every launcher enqueues on
// `stream` and returns the cudaError_t of the launch.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "common.cuh"

namespace resa {

struct Shape {
  int B, Hq, H, G, D;
  int64_t L_max;   // cache capacity (tokens)
  int Mmax;        // L_max / 16
  bool bf16;
};

// descriptors ----------------------------------------------------------------
// lens: optional per-row lengths [B] on the device (len is then their bound)
cudaError_t launch_build_desc(const Shape& s, const void* k, void* desc, int64_t len,
                              cudaStream_t st, const int32_t* lens = nullptr);
cudaError_t launch_append(const Shape& s, const void* k_new, const void* v_new, void* k, void* v,
                          void* desc, int64_t len, cudaStream_t st, const int32_t* lens = nullptr);
cudaError_t launch_rectify_write(const Shape& s, const void* k_f, const void* v_f, void* k, void* v,
                                 void* desc, int64_t len, int f, cudaStream_t st,
                                 const int32_t* lens = nullptr, const int32_t* windows = nullptr,
                                 Ctrl* ctrl = nullptr);

// scoring + selection ----------------------------------------------------------
// scores: [B][H][M] float; the CTA that owns the last chunk also performs the
// append of (k_new, v_new) when k_new != nullptr.
cudaError_t launch_score(const Shape& s, const void* q, const void* desc, float* scores,
                         const void* k_new, const void* v_new, void* k, void* v, void* desc_w,
                         int64_t len, int num_sms, cudaStream_t st,
                         const int32_t* lens = nullptr, Ctrl* ctrl = nullptr);
// with lens, each row's M and n follow its own length (r, n_min: Eq. 5)
cudaError_t launch_select(const Shape& s, const float* scores, int32_t* sel, int M, int n,
                          cudaStream_t st, const int32_t* lens = nullptr, int64_t len = 0,
                          double r = 0.0, int n_min = 0);

// attention ---------------------------------------------------------------------
struct AttnArgs {
  const void* q;          // element (b, r, h, c) at ((b*R + r)*Hq + h)*D + c
  int R;                  // query rows per batch entry
  int64_t len0;           // row r sees tokens t < len0 + r
  const int32_t* sel;     // [B][H][n_sel] or nullptr (dense: every block)
  int n_sel;
  int S;                  // splits per (b, r, KV head)
  float scale;            // softmax scale (natural units)
  float* part_o;          // [B*R*Hq][S][D]
  float* part_ml;         // [B*R*Hq][S][2]  (max in log2 units, sum)
  int* counters;          // [B*R*H], zero between calls
  void* out;              // [B*R][Hq][D] in the cache dtype
  float* lse;             // [B*R][Hq] or nullptr
  Ctrl* ctrl;
  const CUtensorMap* tm_k;  // bf16 only (host copies, passed by value to the kernel)
  const CUtensorMap* tm_v;
  const void* k;          // cache base pointers (fp32 path)
  const void* v;
  bool pdl;               // launched as a programmatic dependent of the select kernel
  // optional per-row lengths [B]: row b's last query row sees lens[b] tokens
  // (len0 + R - 1 is then their bound); selected rows hold Eq. 5's n for
  // their own length (r, n_min), n_sel being the list stride
  const int32_t* lens;
  // optional per-row query counts [B] (rectify windows, clamped to [0, R]):
  // row b uses query rows 0 .. w-1 at positions lens[b] - w .. lens[b] - 1;
  // without it every row uses all R. A batch row shorter than its count
  // (or with count 0) is skipped.
  const int32_t* windows;
  double r;
  int n_min;
};
cudaError_t launch_attend(const Shape& s, const AttnArgs& a, cudaStream_t st);

// one-launch decode step (bf16): append, score, cooperative exact top-n
// selection, attention and merge (decode_coop.cu); S CTAs per KV group
struct CoopLaunch {
  Shape s;
  const void* q;
  const void* k_new;
  const void* v_new;
  void* k;
  void* v;
  void* desc;
  void* out;
  float* lse;
  int32_t* sel;           // [B][H][n] list written by the step
  float* scores;          // [B][H][M] workspace
  int32_t* kept;          // [B][H][M] workspace
  void* groups;           // [B*H] per-group state, zero between calls
  float* part_o;
  float* part_ml;
  int* counters;          // [B*H] merge arrivals, zero between calls
  Ctrl* ctrl;
  int64_t len;
  int M, n, S;
  float scale;
  const CUtensorMap* tm_k;
  const CUtensorMap* tm_v;
  const CUtensorMap* tm_d;  // descriptors as [B*H*Mmax*2][D], 64 x 32 boxes
};
cudaError_t launch_decode_coop(const CoopLaunch& c, cudaStream_t st);
// whether the one-launch kernel takes M blocks, n selected, S CTAs per group
bool coop_supported(const Shape& s, int M, int n, int S);
// workspace bytes of one group's state (256-byte multiple)
size_t coop_group_bytes();
constexpr int kCoopMaxGroups = 64;   // groups (batch x KV heads) the one-launch path serves

// rectification attention on tcgen05 (bf16, group size 1, 2, 4 or 8)
struct RectArgs {
  int B, H, Hq, G, D, f, S, mtiles;
  int64_t len, L_max;     // len: the cache length (with lens: the bound on the rows')
  const int32_t* lens;    // optional per-row lengths [B]
  const int32_t* windows; // optional per-row windows [B] in [0, f]; rows with window 0 or
                          // shorter than their window are skipped
  void* desc;             // prefill (f = len, S = 1): descriptors written from the K tiles
  float scale;
  void* out;              // [B][f][Hq][D] bf16
  float* part_o;          // [S][B*H*mtiles][128][D] (S > 1), float4 units swizzled per row
  float* part_ml;         // [S][B*H*mtiles][128][2]
  Ctrl* ctrl;
  const CUtensorMap* tm_q;  // q_f as [B*f][Hq][D], 64 x G x (128/G) boxes
  const CUtensorMap* tm_k;  // cache as [B*H*L_max][D], 64 x 128 boxes
  const CUtensorMap* tm_v;
  bool pdl;               // launched right after the rectify write kernel: CTAs that
                          // do not read the rewritten rows start before it ends
};
// dense rectification / prefill, then the split merge
cudaError_t launch_rectify_tc(const RectArgs& r, cudaStream_t st);
int attend_ctas_per_sm(const Shape& s);

// bounded wait of one thread until *flag >= target (failure-detection check)
cudaError_t launch_wait_check(const int* flag, int target, unsigned long long limit_ns,
                              Ctrl* ctrl, cudaStream_t st);

constexpr int kMaxSplits = 64;

// Bytes at the start of a workspace that must be zero before a call (the
// error word and the arrival counters); 0 for invalid dims.
size_t workspace_zero_prefix(const Shape& s);

}  // namespace resa
