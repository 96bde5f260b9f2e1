// C ABI of the FLARE library: argument validation, workspace carving and
// launch orchestration on the caller's stream.  No allocation, no
// synchronisation (except flare_device_status, documented as such), no
// global mutable state (the one exception, flare_fwd_noalloc's fixed scratch
// array and its address cache, lives in flare_noalloc.cu).
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "flare_plan.cuh"

using namespace flare;

namespace flare {
namespace {
thread_local char g_error_detail[512];
}

void note_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_error_detail, sizeof(g_error_detail), fmt, ap);
  va_end(ap);
}
}  // namespace flare

namespace {

int current_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 148;  // B200
  }
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;
  }
  return n;
}

#define FLARE_TRY(x)                    \
  do {                                  \
    flare_status_t s_ = (x);            \
    if (s_ != FLARE_OK) return s_;      \
  } while (0)

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

flare_status_t check_sizes(int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                           flare_dtype_t dt) {
  if (B < 1 || H < 1 || N < 1 || M < 1 || D < 1) return FLARE_ERR_INVALID_ARG;
  if (dt != FLARE_F32 && dt != FLARE_BF16) return FLARE_ERR_INVALID_ARG;
  if (B > (1LL << 20) || H > (1LL << 16) || N > (1LL << 34)) return FLARE_ERR_INVALID_ARG;
  if (D != 16 && D != 32) return FLARE_ERR_UNSUPPORTED;
  if (M < 16 || M > 256 || (M % 16) != 0) return FLARE_ERR_UNSUPPORTED;
  const double elems = (double)B * (double)H * (double)N * (double)D;
  if (elems >= 1099511627776.0) return FLARE_ERR_INVALID_ARG;  // 2^40
  if (B * H > 65535) return FLARE_ERR_UNSUPPORTED;               // grid.y limit
  return FLARE_OK;
}

flare_status_t check_scale(float scale) {
  return (std::isfinite(scale) && scale > 0.f) ? FLARE_OK : FLARE_ERR_INVALID_ARG;
}

flare_status_t check_ptr(const void* p) {
  return (p != nullptr && aligned16(p)) ? FLARE_OK : FLARE_ERR_INVALID_ARG;
}

flare_status_t check_opt_ptr(const void* p) {
  return (p == nullptr || aligned16(p)) ? FLARE_OK : FLARE_ERR_INVALID_ARG;
}

flare_status_t check_qbs(int64_t qbs, int64_t H, int64_t M, int64_t D) {
  return (qbs == 0 || qbs == H * M * D) ? FLARE_OK : FLARE_ERR_UNSUPPORTED;
}

// One token tensor's strides: each positive, a multiple of 16 bytes and
// below 2^40 bytes (the TMA limits).  The rows of an output may not overlap:
// taken in order of stride, every dimension with more than one index must
// step over all the rows of the dimensions inside it.
flare_status_t tok_from(const flare_strides_t& st, const Dims& d, flare_dtype_t dt,
                        bool output, Tok* out) {
  const int64_t esz = (dt == FLARE_F32) ? 4 : 2;
  const int64_t v[3] = {st.b_stride, st.h_stride, st.n_stride};
  for (int i = 0; i < 3; ++i) {
    if (v[i] < 1 || v[i] >= (1LL << 40) / esz) return FLARE_ERR_INVALID_ARG;
    if ((v[i] * esz) % 16 != 0) return FLARE_ERR_UNSUPPORTED;
  }
  if (output) {
    int64_t s3[3] = {st.b_stride, st.h_stride, st.n_stride}, e3[3] = {d.B, d.H, d.N};
    for (int i = 0; i < 3; ++i)
      for (int j = i + 1; j < 3; ++j)
        if (s3[j] < s3[i]) {
          const int64_t ts = s3[i], te = e3[i];
          s3[i] = s3[j];
          e3[i] = e3[j];
          s3[j] = ts;
          e3[j] = te;
        }
    int64_t span = d.D;   // elements spanned by the dimensions inside
    for (int i = 0; i < 3; ++i) {
      if (e3[i] == 1) continue;
      if (s3[i] < span) return FLARE_ERR_INVALID_ARG;
      span += s3[i] * (e3[i] - 1);
    }
  }
  *out = Tok{st.b_stride, st.h_stride, st.n_stride};
  return FLARE_OK;
}

// The token tensors' layouts: NULL = contiguous; else one flare_strides_t
// per tensor in the order given by `which` (entries of Dims), the last
// `n_out` of them outputs.
flare_status_t apply_strides(const flare_strides_t* st, Tok Dims::* const* which, int n,
                             int n_out, flare_dtype_t dt, Dims* d) {
  if (st == nullptr) return FLARE_OK;
  for (int i = 0; i < n; ++i) FLARE_TRY(tok_from(st[i], *d, dt, i >= n - n_out, &(d->*which[i])));
  return FLARE_OK;
}

flare_status_t check_opt_lens(const int32_t* lens) {
  return (lens == nullptr || ((uintptr_t)lens & 3u) == 0) ? FLARE_OK : FLARE_ERR_INVALID_ARG;
}

flare_status_t check_ws(const void* ws, size_t bytes, size_t need) {
  if (ws == nullptr || ((uintptr_t)ws & 255u) != 0) return FLARE_ERR_WORKSPACE;
  return bytes >= need ? FLARE_OK : FLARE_ERR_WORKSPACE;
}


#define FLARE_CUDA(x)                                                               \
  do {                                                                              \
    cudaError_t e_ = (x);                                                           \
    if (e_ != cudaSuccess) {                                                        \
      if (g_error_detail[0] == 0)                                                   \
        note_error("%s: %s (%s)", #x, cudaGetErrorName(e_), cudaGetErrorString(e_)); \
      return FLARE_ERR_CUDA;                                                        \
    }                                                                               \
  } while (0)

flare_status_t reset_error_word(char* ws, cudaStream_t st) {
  g_error_detail[0] = 0;
  FLARE_CUDA(cudaMemsetAsync(ws, 0, 4, st));
  return FLARE_OK;
}

// Stage launchers shared by the public entry points (arguments validated).
flare_status_t run_encode(const void* Q, int64_t qbs, const void* K, const void* V,
                          const Dims& d, flare_dtype_t dt, float scale, const WsLayout& L,
                          char* ws, cudaStream_t st) {
  const Path path = choose_path(d.N, d.M, d.D, dt);
  float* pml = (float*)(ws + L.part_ml);
  float* pacc = (float*)(ws + L.part_acc);
  if (path.tc_fwd)
    FLARE_CUDA(launch_tc_encode(Q, qbs, K, V, d, scale, L.enc, pml, pacc, (uint32_t*)(ws + L.hdr),
                                st));
  else
    FLARE_CUDA(launch_simt_encode(Q, qbs, K, V, d, dt, scale, L.enc, pml, pacc, st));
  return FLARE_OK;
}

flare_status_t run_combine(const Dims& d, flare_dtype_t dt, float* Z_save, float* lse_save,
                           const void* Qpp, void* Qdyn, const WsLayout& L, char* ws,
                           cudaStream_t st, const PadZero* pz = nullptr) {
  FLARE_CUDA(launch_combine(d, dt, L.enc.slots_per_bh(), L.enc.sub, 1, (const float*)(ws + L.part_ml),
                            (const float*)(ws + L.part_acc), (float*)(ws + L.zf),
                            (__nv_bfloat16*)(ws + L.zb), Z_save, lse_save, Qpp, Qdyn, st, pz));
  return FLARE_OK;
}

flare_status_t run_decode(const void* Q, int64_t qbs, const void* K, void* Y, const Dims& d,
                          flare_dtype_t dt, float scale, const WsLayout& L, char* ws,
                          cudaStream_t st, int sms) {
  const Path path = choose_path(d.N, d.M, d.D, dt);
  if (path.tc_fwd)
    FLARE_CUDA(launch_tc_decode(Q, qbs, K, (const __nv_bfloat16*)(ws + L.zb), Y, d, scale,
                                decode_plan(d.BH(), d.N, sms), (uint32_t*)(ws + L.hdr), st));
  else
    FLARE_CUDA(launch_simt_decode(Q, qbs, K, (const float*)(ws + L.zf), Y, d, dt, scale, st));
  return FLARE_OK;
}

// Validation shared by the two halves of a sharded backward.
flare_status_t check_bwd_shard(const void* Q, int64_t qbs, const void* K, const void* V,
                                      const void* dY, const float* Z_save, const float* lse_save,
                                      int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                                      flare_dtype_t dt, float scale, void* workspace,
                                      size_t workspace_bytes, WsLayout* L) {
  FLARE_TRY(check_sizes(B, H, N, M, D, dt));
  FLARE_TRY(check_scale(scale));
  FLARE_TRY(check_ptr(Q));
  FLARE_TRY(check_ptr(K));
  FLARE_TRY(check_ptr(V));
  FLARE_TRY(check_ptr(dY));
  FLARE_TRY(check_ptr(Z_save));
  FLARE_TRY(check_ptr(lse_save));
  FLARE_TRY(check_qbs(qbs, H, M, D));
  *L = ws_layout(FLARE_OP_BWD, B, H, N, M, D, dt, current_sm_count());
  return check_ws(workspace, workspace_bytes, L->total);
}

// Order of the flare_strides_t entries: forward K, V, Y; backward K, V,
// dY, dK, dV.
Tok Dims::* const kFwdTensors[3] = {&Dims::k, &Dims::v, &Dims::y};
Tok Dims::* const kBwdTensors[5] = {&Dims::k, &Dims::v, &Dims::dy, &Dims::dk, &Dims::dv};

}  // namespace

extern "C" {

int flare_version(void) { return 100; }

const char* flare_last_error_detail(void) { return g_error_detail; }

const char* flare_status_string(flare_status_t s) {
  switch (s) {
    case FLARE_OK: return "FLARE_OK";
    case FLARE_ERR_INVALID_ARG: return "FLARE_ERR_INVALID_ARG: invalid pointer, size or scale";
    case FLARE_ERR_UNSUPPORTED: return "FLARE_ERR_UNSUPPORTED: unsupported D, M or Q stride";
    case FLARE_ERR_WORKSPACE: return "FLARE_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case FLARE_ERR_CUDA: return "FLARE_ERR_CUDA: a CUDA launch failed";
    case FLARE_ERR_DEVICE_TIMEOUT: return "FLARE_ERR_DEVICE_TIMEOUT: a bounded device wait ran out";
  }
  return "FLARE: unknown status";
}

size_t flare_workspace_size(flare_op_t op, int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                            flare_dtype_t dt) {
  if (op != FLARE_OP_FWD && op != FLARE_OP_PP_FWD && op != FLARE_OP_BWD && op != FLARE_OP_PP_BWD)
    return 0;
  if (check_sizes(B, H, N, M, D, dt) != FLARE_OK) return 0;
  return ws_layout(op, B, H, N, M, D, dt, current_sm_count()).total;
}

int flare_fwd_path(int64_t B, int64_t H, int64_t N, int64_t M, int64_t D, flare_dtype_t dt) {
  if (check_sizes(B, H, N, M, D, dt) != FLARE_OK) return -1;
  return choose_path(N, M, D, dt).tc_fwd ? 1 : 0;
}

int flare_bwd_path(int64_t B, int64_t H, int64_t N, int64_t M, int64_t D, flare_dtype_t dt) {
  if (check_sizes(B, H, N, M, D, dt) != FLARE_OK) return -1;
  return choose_path(N, M, D, dt).tc_bwd ? 1 : 0;
}

flare_status_t flare_encode(const void* Q, int64_t qbs, const void* K, const void* V, int64_t B,
                            int64_t H, int64_t N, int64_t M, int64_t D, flare_dtype_t dt,
                            float scale, void* workspace, size_t workspace_bytes, void* stream) {
  FLARE_TRY(check_sizes(B, H, N, M, D, dt));
  FLARE_TRY(check_scale(scale));
  FLARE_TRY(check_ptr(Q));
  FLARE_TRY(check_ptr(K));
  FLARE_TRY(check_ptr(V));
  FLARE_TRY(check_qbs(qbs, H, M, D));
  const WsLayout L = ws_layout(FLARE_OP_FWD, B, H, N, M, D, dt, current_sm_count());
  FLARE_TRY(check_ws(workspace, workspace_bytes, L.total));
  char* ws = (char*)workspace;
  cudaStream_t st = (cudaStream_t)stream;
  FLARE_TRY(reset_error_word(ws, st));
  return run_encode(Q, qbs, K, V, Dims{B, H, N, M, D}, dt, scale, L, ws, st);
}

flare_status_t flare_combine(int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                             flare_dtype_t dt, float* Z_save, float* lse_save, void* workspace,
                             size_t workspace_bytes, void* stream) {
  FLARE_TRY(check_sizes(B, H, N, M, D, dt));
  FLARE_TRY(check_opt_ptr(Z_save));
  FLARE_TRY(check_opt_ptr(lse_save));
  const WsLayout L = ws_layout(FLARE_OP_FWD, B, H, N, M, D, dt, current_sm_count());
  FLARE_TRY(check_ws(workspace, workspace_bytes, L.total));
  g_error_detail[0] = 0;
  return run_combine(Dims{B, H, N, M, D}, dt, Z_save, lse_save, nullptr, nullptr, L,
                     (char*)workspace, (cudaStream_t)stream);
}

flare_status_t flare_decode(const void* Q, int64_t qbs, const void* K, void* Y, int64_t B,
                            int64_t H, int64_t N, int64_t M, int64_t D, flare_dtype_t dt,
                            float scale, void* workspace, size_t workspace_bytes, void* stream) {
  FLARE_TRY(check_sizes(B, H, N, M, D, dt));
  FLARE_TRY(check_scale(scale));
  FLARE_TRY(check_ptr(Q));
  FLARE_TRY(check_ptr(K));
  FLARE_TRY(check_ptr(Y));
  FLARE_TRY(check_qbs(qbs, H, M, D));
  const int sms = current_sm_count();
  const WsLayout L = ws_layout(FLARE_OP_FWD, B, H, N, M, D, dt, sms);
  FLARE_TRY(check_ws(workspace, workspace_bytes, L.total));
  g_error_detail[0] = 0;
  return run_decode(Q, qbs, K, Y, Dims{B, H, N, M, D}, dt, scale, L, (char*)workspace,
                    (cudaStream_t)stream, sms);
}

flare_status_t flare_fwd_ex(const void* Q, int64_t qbs, const void* K, const void* V,
                                 void* Y, const flare_strides_t* strides,
                                 const int32_t* seq_lens, int64_t B, int64_t H,
                                 int64_t N, int64_t M, int64_t D, flare_dtype_t dt, float scale,
                                 float* Z_save, float* lse_save, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  FLARE_TRY(check_sizes(B, H, N, M, D, dt));
  FLARE_TRY(check_scale(scale));
  FLARE_TRY(check_ptr(Q));
  FLARE_TRY(check_ptr(K));
  FLARE_TRY(check_ptr(V));
  FLARE_TRY(check_ptr(Y));
  FLARE_TRY(check_opt_ptr(Z_save));
  FLARE_TRY(check_opt_ptr(lse_save));
  FLARE_TRY(check_qbs(qbs, H, M, D));
  const int sms = current_sm_count();
  const WsLayout L = ws_layout(FLARE_OP_FWD, B, H, N, M, D, dt, sms);
  FLARE_TRY(check_ws(workspace, workspace_bytes, L.total));
  FLARE_TRY(check_opt_lens(seq_lens));
  Dims d{B, H, N, M, D};
  FLARE_TRY(apply_strides(strides, kFwdTensors, 3, 1, dt, &d));
  d.lens = seq_lens;
  char* ws = (char*)workspace;
  cudaStream_t st = (cudaStream_t)stream;
  FLARE_TRY(reset_error_word(ws, st));
  FLARE_CUDA(launch_var_plan(d, L, ws, st, sms));   // lengths: checked, work plans
  FLARE_TRY(run_encode(Q, qbs, K, V, d, dt, scale, L, ws, st));
  // Y = 0 at padding, by extra blocks of the combine
  const PadZero pz = pad_zero(Y, d.y, nullptr, d.y, d, dt, 256);
  FLARE_TRY(run_combine(d, dt, Z_save, lse_save, nullptr, nullptr, L, ws, st, &pz));
  FLARE_TRY(run_decode(Q, qbs, K, Y, d, dt, scale, L, ws, st, sms));
  return FLARE_OK;
}

flare_status_t flare_pp_fwd_ex(const void* Q, const void* K, const void* V, void* Y,
                                    void* Q_dyn_out, const flare_strides_t* strides,
                                 const int32_t* seq_lens, int64_t B,
                                    int64_t H, int64_t N, int64_t M, int64_t D, flare_dtype_t dt,
                                    float scale, float* Z_save, float* lse_save, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  FLARE_TRY(check_sizes(B, H, N, M, D, dt));
  FLARE_TRY(check_scale(scale));
  FLARE_TRY(check_ptr(Q));
  FLARE_TRY(check_ptr(K));
  FLARE_TRY(check_ptr(V));
  FLARE_TRY(check_ptr(Y));
  FLARE_TRY(check_opt_ptr(Q_dyn_out));
  FLARE_TRY(check_opt_ptr(Z_save));
  FLARE_TRY(check_opt_ptr(lse_save));
  const int sms = current_sm_count();
  const WsLayout L = ws_layout(FLARE_OP_PP_FWD, B, H, N, M, D, dt, sms);
  FLARE_TRY(check_ws(workspace, workspace_bytes, L.total));
  FLARE_TRY(check_opt_lens(seq_lens));
  Dims d{B, H, N, M, D};
  FLARE_TRY(apply_strides(strides, kFwdTensors, 3, 1, dt, &d));
  d.lens = seq_lens;
  char* ws = (char*)workspace;
  cudaStream_t st = (cudaStream_t)stream;
  void* qdyn = Q_dyn_out ? Q_dyn_out : (void*)(ws + L.qdyn);
  const int64_t qdyn_bs = H * M * D;
  FLARE_TRY(reset_error_word(ws, st));
  FLARE_CUDA(launch_var_plan(d, L, ws, st, sms));   // lengths: checked, work plans
  // Z1 = encode(Q, K, V); Q_dyn = Q + Z1 (written by the combine)
  FLARE_TRY(run_encode(Q, 0, K, V, d, dt, scale, L, ws, st));
  FLARE_TRY(run_combine(d, dt, nullptr, nullptr, Q, qdyn, L, ws, st));
  // Z = encode(Q_dyn, K, V); Y = decode(Q_dyn, K, Z)
  FLARE_TRY(run_encode(qdyn, qdyn_bs, K, V, d, dt, scale, L, ws, st));
  // Y = 0 at padding, by extra blocks of the combine
  const PadZero pz = pad_zero(Y, d.y, nullptr, d.y, d, dt, 256);
  FLARE_TRY(run_combine(d, dt, Z_save, lse_save, nullptr, nullptr, L, ws, st, &pz));
  FLARE_TRY(run_decode(qdyn, qdyn_bs, K, Y, d, dt, scale, L, ws, st, sms));
  return FLARE_OK;
}

flare_status_t flare_bwd_ex(const void* Q, int64_t qbs, const void* K, const void* V,
                                 const void* dY, const float* Z_save, const float* lse_save,
                                 void* dQ, void* dK, void* dV, const flare_strides_t* strides,
                                 const int32_t* seq_lens,
                                 int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                                 flare_dtype_t dt, float scale, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  FLARE_TRY(check_sizes(B, H, N, M, D, dt));
  FLARE_TRY(check_scale(scale));
  FLARE_TRY(check_ptr(Q));
  FLARE_TRY(check_ptr(K));
  FLARE_TRY(check_ptr(V));
  FLARE_TRY(check_ptr(dY));
  FLARE_TRY(check_ptr(Z_save));
  FLARE_TRY(check_ptr(lse_save));
  FLARE_TRY(check_ptr(dQ));
  FLARE_TRY(check_ptr(dK));
  FLARE_TRY(check_ptr(dV));
  FLARE_TRY(check_qbs(qbs, H, M, D));
  const int sms = current_sm_count();
  const WsLayout L = ws_layout(FLARE_OP_BWD, B, H, N, M, D, dt, sms);
  FLARE_TRY(check_ws(workspace, workspace_bytes, L.total));
  FLARE_TRY(check_opt_lens(seq_lens));
  Dims d{B, H, N, M, D};
  FLARE_TRY(apply_strides(strides, kBwdTensors, 5, 2, dt, &d));
  d.lens = seq_lens;
  char* ws = (char*)workspace;
  cudaStream_t st = (cudaStream_t)stream;
  FLARE_TRY(reset_error_word(ws, st));
  // lengths: checked, work plans (computed inside the backward's first kernel)
  PlanArgs plan;
  FLARE_CUDA(launch_var_plan(d, L, ws, st, sms, &plan));
  // no gradient at padding: dK = dV = 0 there (zeroed by the backward)
  const PadZero pz = pad_zero(dK, d.dk, dV, d.dv, d, dt, (int)M);
  FLARE_CUDA(launch_bwd(Q, qbs, K, V, dY, Z_save, lse_save, dQ, dK, dV, d, dt, scale, L, ws, st,
                        BwdPhase::ALL, nullptr, nullptr, &pz, &plan));
  return FLARE_OK;
}

flare_status_t flare_pp_bwd_ex(const void* Q, const void* K, const void* V, const void* dY,
                                    const void* Q_dyn, const float* Z_save, const float* lse_save,
                                    void* dQ, void* dK, void* dV, const flare_strides_t* strides,
                                 const int32_t* seq_lens,
                                    int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                                    flare_dtype_t dt, float scale, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  FLARE_TRY(check_sizes(B, H, N, M, D, dt));
  FLARE_TRY(check_scale(scale));
  FLARE_TRY(check_ptr(Q));
  FLARE_TRY(check_ptr(K));
  FLARE_TRY(check_ptr(V));
  FLARE_TRY(check_ptr(dY));
  FLARE_TRY(check_ptr(Q_dyn));
  FLARE_TRY(check_ptr(Z_save));
  FLARE_TRY(check_ptr(lse_save));
  FLARE_TRY(check_ptr(dQ));
  FLARE_TRY(check_ptr(dK));
  FLARE_TRY(check_ptr(dV));
  const int sms = current_sm_count();
  const WsLayout L = ws_layout(FLARE_OP_PP_BWD, B, H, N, M, D, dt, sms);
  FLARE_TRY(check_ws(workspace, workspace_bytes, L.total));
  FLARE_TRY(check_opt_lens(seq_lens));
  Dims d{B, H, N, M, D};
  FLARE_TRY(apply_strides(strides, kBwdTensors, 5, 2, dt, &d));
  d.lens = seq_lens;
  char* ws = (char*)workspace;
  cudaStream_t st = (cudaStream_t)stream;
  float* z1 = (float*)(ws + L.z1);
  float* lse1 = (float*)(ws + L.lse1);
  FLARE_TRY(reset_error_word(ws, st));
  FLARE_CUDA(launch_var_plan(d, L, ws, st, sms));   // lengths: checked, work plans
  // the first encode, recomputed: Z1 and its lse
  FLARE_TRY(run_encode(Q, 0, K, V, d, dt, scale, L, ws, st));
  FLARE_TRY(run_combine(d, dt, z1, lse1, nullptr, nullptr, L, ws, st));
  // FLARE's backward with the per-batch latents Q_dyn: dQ_dyn, dK, dV
  // (no gradient at padding: dK = dV = 0 there, zeroed by this backward)
  const PadZero pz = pad_zero(dK, d.dk, dV, d.dv, d, dt, (int)M);
  FLARE_CUDA(launch_bwd(Q_dyn, H * M * D, K, V, dY, Z_save, lse_save, ws + L.dqd, dK, dV, d, dt,
                        scale, L, ws, st, BwdPhase::ALL, nullptr, nullptr, &pz));
  // the first encode's gradient with upstream dQ_dyn (valid rows only), and dQ
  FLARE_CUDA(launch_pp_bwd_tail(Q, K, V, z1, lse1, ws + L.dqd, dQ, dK, dV, d, dt, scale, L, ws, st));
  return FLARE_OK;
}

flare_status_t flare_fwd(const void* Q, int64_t qbs, const void* K, const void* V, void* Y,
                         int64_t B, int64_t H, int64_t N, int64_t M, int64_t D, flare_dtype_t dt,
                         float scale, float* Z_save, float* lse_save, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return flare_fwd_ex(Q, qbs, K, V, Y, nullptr, nullptr, B, H, N, M, D, dt, scale, Z_save, lse_save,
                           workspace, workspace_bytes, stream);
}

// ------------------------------------------------- forward from host memory

}  // extern "C"

namespace {

// Heads per chunk of flare_fwd_host: about 16 chunks, each inside one
// batch element.
int64_t host_chunk_heads(int64_t B, int64_t H) {
  const int64_t hc = (B * H + 15) / 16;
  return hc < 1 ? 1 : (hc > H ? H : hc);
}

}  // namespace

extern "C" {

size_t flare_fwd_host_workspace_size(int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                                     flare_dtype_t dt) {
  if (check_sizes(B, H, N, M, D, dt) != FLARE_OK) return 0;
  return ws_layout(FLARE_OP_FWD, 1, host_chunk_heads(B, H), N, M, D, dt, current_sm_count()).total;
}

flare_status_t flare_fwd_host(const void* Q_host, int64_t qbs, const void* K_host,
                              const void* V_host, void* Y_host, void* Q_dev, void* K_dev,
                              void* V_dev, void* Y_dev, int64_t B, int64_t H, int64_t N, int64_t M,
                              int64_t D, flare_dtype_t dt, float scale, void* workspace,
                              size_t workspace_bytes, void* stream, void* copy_stream) {
  FLARE_TRY(check_sizes(B, H, N, M, D, dt));
  FLARE_TRY(check_scale(scale));
  FLARE_TRY(check_qbs(qbs, H, M, D));
  if (!Q_host || !K_host || !V_host || !Y_host) return FLARE_ERR_INVALID_ARG;
  FLARE_TRY(check_ptr(Q_dev));
  FLARE_TRY(check_ptr(K_dev));
  FLARE_TRY(check_ptr(V_dev));
  FLARE_TRY(check_ptr(Y_dev));
  const int sms = current_sm_count();
  const int64_t hc = host_chunk_heads(B, H);
  const WsLayout L = ws_layout(FLARE_OP_FWD, 1, hc, N, M, D, dt, sms);
  FLARE_TRY(check_ws(workspace, workspace_bytes, L.total));
  char* ws = (char*)workspace;
  cudaStream_t st = (cudaStream_t)stream, cs = (cudaStream_t)copy_stream;
  const int64_t esz = (dt == FLARE_F32) ? 4 : 2;
  const int64_t head_bytes = N * D * esz, lat_bytes = M * D * esz;
  // the copies start after the work already queued on `stream` (which may
  // still use the device buffers)
  cudaEvent_t start = nullptr;
  FLARE_CUDA(cudaEventCreateWithFlags(&start, cudaEventDisableTiming));
  flare_status_t status = FLARE_OK;
  auto fail = [&](cudaError_t e, const char* what) {
    note_error("flare_fwd_host: %s (%s)", what, cudaGetErrorName(e));
    status = FLARE_ERR_CUDA;
  };
  cudaError_t e;
  if ((e = cudaEventRecord(start, st)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(cs, start, 0)) != cudaSuccess)
    fail(e, "stream ordering");
  if (status == FLARE_OK &&
      (e = cudaMemcpyAsync(Q_dev, Q_host, (qbs ? B * H : H) * lat_bytes, cudaMemcpyHostToDevice,
                           cs)) != cudaSuccess)
    fail(e, "Q copy");
  if (status == FLARE_OK) status = reset_error_word(ws, st);
  // chunk k: heads [h0, h1) of batch element b.  Its K and V go in on the
  // copy stream; `stream` waits for them, runs the forward on the chunk (B =
  // 1, shared latents at the chunk's offset) and copies its Y out, while
  // the copy stream already brings in the next chunk.
  for (int64_t b = 0; b < B && status == FLARE_OK; ++b) {
    for (int64_t h0 = 0; h0 < H && status == FLARE_OK; h0 += hc) {
      const int64_t h1 = (h0 + hc < H) ? h0 + hc : H;
      const int64_t off = (b * H + h0) * head_bytes, bytes = (h1 - h0) * head_bytes;
      cudaEvent_t in = nullptr;
      if ((e = cudaEventCreateWithFlags(&in, cudaEventDisableTiming)) != cudaSuccess) {
        fail(e, "event");
        break;
      }
      if ((e = cudaMemcpyAsync((char*)K_dev + off, (const char*)K_host + off, bytes,
                               cudaMemcpyHostToDevice, cs)) != cudaSuccess ||
          (e = cudaMemcpyAsync((char*)V_dev + off, (const char*)V_host + off, bytes,
                               cudaMemcpyHostToDevice, cs)) != cudaSuccess ||
          (e = cudaEventRecord(in, cs)) != cudaSuccess ||
          (e = cudaStreamWaitEvent(st, in, 0)) != cudaSuccess)
        fail(e, "K / V copy");
      cudaEventDestroy(in);   // released once recorded work completes
      if (status != FLARE_OK) break;
      const char* Qc = (const char*)Q_dev + ((qbs ? b * H : 0) + h0) * lat_bytes;
      Dims d{1, h1 - h0, N, M, D};
      if ((status = run_encode(Qc, 0, (const char*)K_dev + off, (const char*)V_dev + off, d, dt,
                               scale, L, ws, st)) != FLARE_OK ||
          (status = run_combine(d, dt, nullptr, nullptr, nullptr, nullptr, L, ws, st)) != FLARE_OK ||
          (status = run_decode(Qc, 0, (const char*)K_dev + off, (char*)Y_dev + off, d, dt, scale, L,
                               ws, st, sms)) != FLARE_OK)
        break;
      if ((e = cudaMemcpyAsync((char*)Y_host + off, (const char*)Y_dev + off, bytes,
                               cudaMemcpyDeviceToHost, st)) != cudaSuccess)
        fail(e, "Y copy");
    }
  }
  cudaEventDestroy(start);
  return status;
}

flare_status_t flare_pp_fwd(const void* Q, const void* K, const void* V, void* Y,
                            void* Q_dyn_out, int64_t B, int64_t H, int64_t N, int64_t M,
                            int64_t D, flare_dtype_t dt, float scale, float* Z_save,
                            float* lse_save, void* workspace, size_t workspace_bytes,
                            void* stream) {
  return flare_pp_fwd_ex(Q, K, V, Y, Q_dyn_out, nullptr, nullptr, B, H, N, M, D, dt, scale, Z_save,
                              lse_save, workspace, workspace_bytes, stream);
}

flare_status_t flare_bwd(const void* Q, int64_t qbs, const void* K, const void* V,
                         const void* dY, const float* Z_save, const float* lse_save, void* dQ,
                         void* dK, void* dV, int64_t B, int64_t H, int64_t N, int64_t M,
                         int64_t D, flare_dtype_t dt, float scale, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return flare_bwd_ex(Q, qbs, K, V, dY, Z_save, lse_save, dQ, dK, dV, nullptr, nullptr, B, H, N, M,
                           D, dt, scale, workspace, workspace_bytes, stream);
}

flare_status_t flare_pp_bwd(const void* Q, const void* K, const void* V, const void* dY,
                            const void* Q_dyn, const float* Z_save, const float* lse_save,
                            void* dQ, void* dK, void* dV, int64_t B, int64_t H, int64_t N,
                            int64_t M, int64_t D, flare_dtype_t dt, float scale, void* workspace,
                            size_t workspace_bytes, void* stream) {
  return flare_pp_bwd_ex(Q, K, V, dY, Q_dyn, Z_save, lse_save, dQ, dK, dV, nullptr, nullptr, B, H, N,
                              M, D, dt, scale, workspace, workspace_bytes, stream);
}

flare_status_t flare_records_layout(int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                                    flare_dtype_t dt, int64_t* records_per_bh, size_t* ml_offset,
                                    size_t* acc_offset) {
  FLARE_TRY(check_sizes(B, H, N, M, D, dt));
  if (!records_per_bh || !ml_offset || !acc_offset) return FLARE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(FLARE_OP_FWD, B, H, N, M, D, dt, current_sm_count());
  *records_per_bh = L.enc.slots_per_bh();
  *ml_offset = L.part_ml;
  *acc_offset = L.part_acc;
  return FLARE_OK;
}

flare_status_t flare_combine_shards(int64_t shards, const float* ml, const float* acc,
                                    int64_t records_per_bh, int64_t B, int64_t H, int64_t N,
                                    int64_t M, int64_t D, flare_dtype_t dt, float* Z_save,
                                    float* lse_save, const void* Q_learned, void* Q_dyn_out,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  FLARE_TRY(check_sizes(B, H, N, M, D, dt));
  if (shards < 1 || shards > 65536 || records_per_bh < 1 || records_per_bh > (1 << 20))
    return FLARE_ERR_INVALID_ARG;
  FLARE_TRY(check_ptr(ml));
  FLARE_TRY(check_ptr(acc));
  FLARE_TRY(check_opt_ptr(Z_save));
  FLARE_TRY(check_opt_ptr(lse_save));
  FLARE_TRY(check_opt_ptr(Q_dyn_out));
  if (Q_dyn_out) FLARE_TRY(check_ptr(Q_learned));
  const WsLayout L = ws_layout(FLARE_OP_FWD, B, H, N, M, D, dt, current_sm_count());
  FLARE_TRY(check_ws(workspace, workspace_bytes, L.total));
  g_error_detail[0] = 0;
  char* ws = (char*)workspace;
  FLARE_CUDA(launch_combine(Dims{B, H, N, M, D}, dt, (int)records_per_bh, 1, (int)shards, ml, acc,
                            (float*)(ws + L.zf), (__nv_bfloat16*)(ws + L.zb), Z_save, lse_save,
                            Q_dyn_out ? Q_learned : nullptr, Q_dyn_out, (cudaStream_t)stream));
  return FLARE_OK;
}

flare_status_t flare_bwd_shard_dz(const void* Q, int64_t qbs, const void* K, const void* V,
                                  const void* dY, const float* Z_save, const float* lse_save,
                                  float* dZ_part, int64_t B, int64_t H, int64_t N, int64_t M,
                                  int64_t D, flare_dtype_t dt, float scale, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  WsLayout L;
  FLARE_TRY(check_bwd_shard(Q, qbs, K, V, dY, Z_save, lse_save, B, H, N, M, D, dt, scale,
                            workspace, workspace_bytes, &L));
  FLARE_TRY(check_ptr(dZ_part));
  char* ws = (char*)workspace;
  cudaStream_t st = (cudaStream_t)stream;
  FLARE_TRY(reset_error_word(ws, st));
  FLARE_CUDA(launch_bwd(Q, qbs, K, V, dY, Z_save, lse_save, nullptr, nullptr, nullptr,
                        Dims{B, H, N, M, D}, dt, scale, L, ws, st, BwdPhase::DZ, dZ_part,
                        nullptr));
  return FLARE_OK;
}

flare_status_t flare_bwd_shard_finish(const void* Q, int64_t qbs, const void* K, const void* V,
                                      const void* dY, const float* Z_save, const float* lse_save,
                                      const float* dZ, float* dQ_part, void* dK, void* dV,
                                      int64_t B, int64_t H, int64_t N, int64_t M, int64_t D,
                                      flare_dtype_t dt, float scale, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  WsLayout L;
  FLARE_TRY(check_bwd_shard(Q, qbs, K, V, dY, Z_save, lse_save, B, H, N, M, D, dt, scale,
                            workspace, workspace_bytes, &L));
  FLARE_TRY(check_ptr(dZ));
  FLARE_TRY(check_ptr(dQ_part));
  FLARE_TRY(check_ptr(dK));
  FLARE_TRY(check_ptr(dV));
  g_error_detail[0] = 0;   // the error word keeps what the first half recorded
  FLARE_CUDA(launch_bwd(Q, qbs, K, V, dY, Z_save, lse_save, nullptr, dK, dV, Dims{B, H, N, M, D},
                        dt, scale, L, (char*)workspace, (cudaStream_t)stream, BwdPhase::FINISH,
                        const_cast<float*>(dZ), dQ_part));
  return FLARE_OK;
}

flare_status_t flare_pp_bwd_shard_tail(const void* Q, const void* K, const void* V,
                                       const float* Z1, const float* lse1, const void* dQ_dyn,
                                       int add_dq_dyn, float* dQ_part, void* dK, void* dV,
                                       int64_t B, int64_t H,
                                       int64_t N, int64_t M, int64_t D, flare_dtype_t dt,
                                       float scale, void* workspace, size_t workspace_bytes,
                                       void* stream) {
  FLARE_TRY(check_sizes(B, H, N, M, D, dt));
  FLARE_TRY(check_scale(scale));
  FLARE_TRY(check_ptr(Q));
  FLARE_TRY(check_ptr(K));
  FLARE_TRY(check_ptr(V));
  FLARE_TRY(check_ptr(Z1));
  FLARE_TRY(check_ptr(lse1));
  FLARE_TRY(check_ptr(dQ_dyn));
  FLARE_TRY(check_ptr(dQ_part));
  FLARE_TRY(check_ptr(dK));
  FLARE_TRY(check_ptr(dV));
  const WsLayout L = ws_layout(FLARE_OP_PP_BWD, B, H, N, M, D, dt, current_sm_count());
  FLARE_TRY(check_ws(workspace, workspace_bytes, L.total));
  g_error_detail[0] = 0;
  FLARE_CUDA(launch_pp_bwd_tail(Q, K, V, Z1, lse1, dQ_dyn, nullptr, dK, dV, Dims{B, H, N, M, D}, dt,
                                scale, L, (char*)workspace, (cudaStream_t)stream, dQ_part,
                                add_dq_dyn != 0));
  return FLARE_OK;
}

flare_status_t flare_device_status(void* workspace, size_t workspace_bytes, uint32_t* detail,
                                   void* stream) {
  if (workspace == nullptr || workspace_bytes < 256 || ((uintptr_t)workspace & 255u) != 0)
    return FLARE_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return FLARE_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return FLARE_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, 4, st) != cudaSuccess) return FLARE_ERR_CUDA;
  if (detail) *detail = word;
  if (word == 0) return FLARE_OK;
  return word == kErrSeqLen ? FLARE_ERR_INVALID_ARG : FLARE_ERR_DEVICE_TIMEOUT;
}

}  // extern "C"
