// C ABI of the FlashLoop loop-r attention sublayer (see include/flashloop.h).
//
// Host side only: argument checks, workspace carving and kernel launches on
// the caller's stream.  Nothing here allocates or synchronises, apart from
// flashloop_check_error_word, whose job is to read the error word back.
#include <math.h>
#include <stdio.h>

#include <atomic>

#include "common.cuh"

namespace fl {
int launch_gate(const flashloop_params*, const uint16_t*, const uint16_t*, const int32_t*,
                const int32_t*, int, int32_t*, int32_t*, int32_t*, int, void*, int32_t*, cudaStream_t);
int launch_gate_topk(const flashloop_params*, const uint16_t*, const uint16_t*, const int32_t*, const int32_t*,
                     int, int, int32_t*, int32_t*, int32_t*, void*, int32_t*, cudaStream_t);
int launch_kv_quant(const flashloop_params*, int, const float*, const float*, const int32_t*,
                    const int32_t*, flashloop_state*, cudaStream_t);
int launch_selcol_dequant(const flashloop_params*, int, const int32_t*, int, int, flashloop_state*,
                          __half*, __half*, __half*, __half*, cudaStream_t);
int launch_topk(const flashloop_params*, const float*, const int32_t*, int, int, int32_t*, int32_t*,
                cudaStream_t, const float* row_m = nullptr, const float* row_z = nullptr,
                float* probs_out = nullptr, const int32_t* n_dev = nullptr, int32_t* k_out = nullptr,
                const int32_t* out_map = nullptr);
int launch_qkv_gemm(const flashloop_params*, const uint16_t*, const int32_t*, const int32_t*, int,
                    const uint16_t*, const float*, uint16_t*, float*, float*, int32_t*, cudaStream_t);
int launch_out_gemm(const flashloop_params*, const uint16_t*, const int32_t*, const int32_t*, int,
                    const uint16_t*, uint16_t*, int32_t*, cudaStream_t);
int launch_qkv_quant_gemm(const flashloop_params*, int, const uint16_t*, const int32_t*, const int32_t*, int,
                          const uint16_t*, flashloop_state*, uint16_t*, cudaStream_t);
}  // namespace fl

#include "attn_args.cuh"

namespace fl {
int launch_attn_tc(const flashloop_params*, const AttnArgs&, int, cudaStream_t);
int launch_attn_row_counts(const AttnArgs&, int32_t*, cudaStream_t);
DecodeLayout decode_layout(const flashloop_params*);
int launch_decode_attn(const flashloop_params*, int, const flashloop_state*, flashloop_decode_state*, cudaStream_t);
int launch_decode_select(const flashloop_params*, flashloop_decode_state*, cudaStream_t);
int launch_decode_qkv(const flashloop_params*, int, const uint16_t*, const uint16_t*, flashloop_decode_state*,
                      cudaStream_t);
int launch_decode_out(const flashloop_params*, const uint16_t*, flashloop_decode_state*, cudaStream_t);
int launch_colmass_tc(const flashloop_params*, const ColmassArgs&, void*, void*, cudaStream_t);
int launch_paper_quant(const flashloop_params*, int, const float*, const float*, const int32_t*, const int32_t*,
                       int, const flashloop_state*, cudaStream_t);
int launch_paper_selcol(const flashloop_params*, int, const int32_t*, int, int, const flashloop_state*, __half*,
                        __half*, __half*, __half*, cudaStream_t);

// ---------------------------------------------------------------------------
// checks
// ---------------------------------------------------------------------------
static int check_arch() {
  static std::atomic<int> cached[64];  // 0 = unknown, 1 = sm_100, -1 = other
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLASHLOOP_ERR_CUDA;
  if (dev < 0 || dev >= 64) return FLASHLOOP_ERR_CUDA;
  int c = cached[dev].load(std::memory_order_relaxed);
  if (c == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return FLASHLOOP_ERR_CUDA;
    c = (major == 10 && minor == 0) ? 1 : -1;
    cached[dev].store(c, std::memory_order_relaxed);
  }
  return c == 1 ? FLASHLOOP_OK : FLASHLOOP_ERR_ARCH;
}

static int check_params(const flashloop_params* p) {
  if (p == nullptr) return FLASHLOOP_ERR_INVALID_ARG;
  if (p->seq < 1 || p->n_heads < 1 || p->n_loops < 1 || p->n_loops > FLASHLOOP_MAX_LOOPS)
    return FLASHLOOP_ERR_INVALID_ARG;
  if (p->head_dim != 64 && p->head_dim != 128) return FLASHLOOP_ERR_UNSUPPORTED;
  if (p->d_model != p->n_heads * p->head_dim) return FLASHLOOP_ERR_INVALID_ARG;
  if (p->d_model % 128 != 0) return FLASHLOOP_ERR_UNSUPPORTED;
  if (!(p->tau >= 0.f) || !(p->rope_theta > 0.f)) return FLASHLOOP_ERR_INVALID_ARG;
  if (p->kv_scheme != 0 && p->kv_scheme != 1) return FLASHLOOP_ERR_UNSUPPORTED;
  if (p->attn_pairs != 0) return FLASHLOOP_ERR_UNSUPPORTED;  // reserved
  if (p->kv_scheme == 0 && p->bits[0] != 8) return FLASHLOOP_ERR_UNSUPPORTED;
  for (int r = 2; r <= p->n_loops; ++r) {
    const int b = p->bits[r - 1];
    if (p->kv_scheme == 0 && b != 8 && b != 4 && b != 2) return FLASHLOOP_ERR_UNSUPPORTED;
    const int k = p->topk[r - 1];
    if (k < 1 || k > p->seq) return FLASHLOOP_ERR_INVALID_ARG;
    if (r >= 3 && k > p->topk[r - 2]) return FLASHLOOP_ERR_INVALID_ARG;  // nested selection
    if (p->capacity[r - 1] < 1 || p->capacity[r - 1] > p->seq) return FLASHLOOP_ERR_INVALID_ARG;
  }
  return FLASHLOOP_OK;
}

static int check_common(const flashloop_params* p) {
  int rc = check_params(p);
  if (rc != FLASHLOOP_OK) return rc;
  return check_arch();
}

// The parameter and architecture checks of every entry point, for the entry
// points defined in other files.
int check_params_and_arch(const flashloop_params* p) { return check_common(p); }
int check_device_arch() { return check_arch(); }

static inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

static inline int capacity_of(const flashloop_params* p, int r) {
  return r == 1 ? p->seq : p->capacity[r - 1];
}

}  // namespace fl

using namespace fl;

// ---------------------------------------------------------------------------
// rope table
// ---------------------------------------------------------------------------
__global__ void rope_table_kernel(int n_pos, int half, double theta, float* cs) {
  const long long n = (long long)n_pos * half;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int t = static_cast<int>(i / half), e = static_cast<int>(i % half);
    const double inv = pow(theta, -(2.0 * e) / (2.0 * half));
    const double ang = static_cast<double>(t) * inv;
    double s, c;
    sincos(ang, &s, &c);
    cs[2 * i] = static_cast<float>(c);
    cs[2 * i + 1] = static_cast<float>(s);
  }
}

extern "C" {

size_t flashloop_workspace_bytes(const flashloop_params* p) {
  if (check_params(p) != FLASHLOOP_OK) return 0;
  return workspace_layout(p).total;
}

size_t flashloop_cache_bytes(const flashloop_params* p, const int32_t* n_per_loop) {
  if (check_params(p) != FLASHLOOP_OK || n_per_loop == nullptr) return 0;
  const size_t H = p->n_heads, dh = p->head_dim;
  const size_t scales = 2 * (dh / FLASHLOOP_GROUP);
  size_t total = 2 * (size_t)p->seq * H * (dh * p->bits[0] / 8 + scales);
  for (int r = 2; r <= p->n_loops; ++r)
    total += 2 * (size_t)n_per_loop[r - 1] * H * (dh * p->bits[r - 1] / 8 + scales);
  return total;
}

int flashloop_rope_table(const flashloop_params* p, int32_t n_pos, float* cs, void* stream) {
  int rc = check_common(p);
  if (rc != FLASHLOOP_OK) return rc;
  if (cs == nullptr || n_pos < 1) return FLASHLOOP_ERR_INVALID_ARG;
  const int half = p->head_dim / 2;
  long long n = (long long)n_pos * half;
  int grid = (int)((n + 255) / 256);
  if (grid > 148 * 8) grid = 148 * 8;
  rope_table_kernel<<<grid, 256, 0, as_stream(stream)>>>(n_pos, half, (double)p->rope_theta, cs);
  return launch_status();
}

int32_t flashloop_selection_loop(const flashloop_params* p, int32_t loop) {
  if (p == nullptr || loop < 2 || loop > p->n_loops) return -1;
  int sel = 2;
  for (int r = 3; r <= loop; ++r)
    if (p->topk[r - 1] < p->topk[r - 2]) sel = r;
  return sel;
}

int flashloop_gate(const flashloop_params* p, const uint16_t* x_cur, const uint16_t* x_prev,
                   const int32_t* prev_active, const int32_t* n_prev, int32_t prev_capacity,
                   int32_t* active_out, int32_t* slot_out, int32_t* n_active_out,
                   int32_t out_capacity, void* workspace, int32_t* err_word, void* stream) {
  int rc = check_common(p);
  if (rc != FLASHLOOP_OK) return rc;
  if (!x_cur || !x_prev || !active_out || !slot_out || !n_active_out || !workspace)
    return FLASHLOOP_ERR_INVALID_ARG;
  if (prev_active != nullptr && n_prev == nullptr) return FLASHLOOP_ERR_INVALID_ARG;
  if (prev_capacity < 1 || prev_capacity > p->seq || out_capacity < 1 || out_capacity > p->seq)
    return FLASHLOOP_ERR_INVALID_ARG;
  return launch_gate(p, x_cur, x_prev, prev_active, n_prev, prev_capacity, active_out, slot_out,
                     n_active_out, out_capacity, workspace, err_word, as_stream(stream));
}

int flashloop_gate_topk(const flashloop_params* p, const uint16_t* x_cur, const uint16_t* x_prev,
                        const int32_t* prev_active, const int32_t* n_prev, int32_t prev_capacity,
                        int32_t budget, int32_t* active_out, int32_t* slot_out, int32_t* n_active_out,
                        int32_t out_capacity, void* workspace, int32_t* err_word, void* stream) {
  int rc = check_common(p);
  if (rc != FLASHLOOP_OK) return rc;
  if (!x_cur || !x_prev || !active_out || !slot_out || !n_active_out || !workspace) return FLASHLOOP_ERR_INVALID_ARG;
  if (prev_active != nullptr && n_prev == nullptr) return FLASHLOOP_ERR_INVALID_ARG;
  if (prev_capacity < 1 || prev_capacity > p->seq || out_capacity < 1 || out_capacity > p->seq)
    return FLASHLOOP_ERR_INVALID_ARG;
  if (prev_active == nullptr && prev_capacity != p->seq) return FLASHLOOP_ERR_INVALID_ARG;
  if (budget < 0 || budget > out_capacity) return FLASHLOOP_ERR_INVALID_ARG;
  if (prev_capacity > 49152) return FLASHLOOP_ERR_UNSUPPORTED;
  return launch_gate_topk(p, x_cur, x_prev, prev_active, n_prev, prev_capacity, budget, active_out, slot_out,
                          n_active_out, workspace, err_word, as_stream(stream));
}

int flashloop_qkv_gathered(const flashloop_params* p, const uint16_t* x, const int32_t* active,
                           const int32_t* n_active, int32_t capacity, const uint16_t* w_qkv,
                           const float* rope_cs, uint16_t* q_out, float* k_out, float* v_out,
                           void* stream) {
  int rc = check_common(p);
  if (rc != FLASHLOOP_OK) return rc;
  if (!x || !w_qkv || !rope_cs || !q_out || !k_out || !v_out) return FLASHLOOP_ERR_INVALID_ARG;
  if (active != nullptr && n_active == nullptr) return FLASHLOOP_ERR_INVALID_ARG;
  if (capacity < 1 || capacity > p->seq) return FLASHLOOP_ERR_INVALID_ARG;
  return launch_qkv_gemm(p, x, active, n_active, capacity, w_qkv, rope_cs, q_out, k_out, v_out,
                         nullptr, as_stream(stream));
}

int flashloop_kv_quant_residual(const flashloop_params* p, int32_t loop, const float* k_new,
                                const float* v_new, const int32_t* active, const int32_t* n_active,
                                flashloop_state* st, void* stream) {
  int rc = check_common(p);
  if (rc != FLASHLOOP_OK) return rc;
  if (loop < 1 || loop > p->n_loops || !k_new || !v_new || !st) return FLASHLOOP_ERR_INVALID_ARG;
  if (p->kv_scheme != 0) return FLASHLOOP_ERR_UNSUPPORTED;  // see flashloop_paper_kv_quant
  if (!st->k.base_codes || !st->k.base_scales || !st->v.base_codes || !st->v.base_scales)
    return FLASHLOOP_ERR_INVALID_ARG;
  if (loop >= 2) {
    if (!active || !n_active) return FLASHLOOP_ERR_INVALID_ARG;
    for (int l = 2; l <= loop; ++l) {
      if (!st->k.res_codes[l - 1] || !st->k.res_scales[l - 1] || !st->v.res_codes[l - 1] ||
          !st->v.res_scales[l - 1])
        return FLASHLOOP_ERR_INVALID_ARG;
      if (l < loop && !st->slot[l - 1]) return FLASHLOOP_ERR_INVALID_ARG;
    }
  }
  return launch_kv_quant(p, loop, k_new, v_new, active, n_active, st, as_stream(stream));
}

int flashloop_qkv_quant(const flashloop_params* p, int32_t loop, const uint16_t* x, const int32_t* active,
                        const int32_t* n_active, const uint16_t* w_qkv, flashloop_state* st,
                        uint16_t* q_out, void* stream) {
  int rc = check_common(p);
  if (rc != FLASHLOOP_OK) return rc;
  if (loop < 1 || loop > p->n_loops || !x || !w_qkv || !st || !st->rope_cs)
    return FLASHLOOP_ERR_INVALID_ARG;
  if (p->kv_scheme != 0) return FLASHLOOP_ERR_UNSUPPORTED;  // the fused quantiser writes the INT8 / INT4 / INT2 streams
  if (!st->k.base_codes || !st->k.base_scales || !st->v.base_codes || !st->v.base_scales)
    return FLASHLOOP_ERR_INVALID_ARG;
  if (active != nullptr && n_active == nullptr) return FLASHLOOP_ERR_INVALID_ARG;
  if (loop >= 2) {
    if (!active) return FLASHLOOP_ERR_INVALID_ARG;
    for (int l = 2; l <= loop; ++l) {
      if (!st->k.res_codes[l - 1] || !st->k.res_scales[l - 1] || !st->v.res_codes[l - 1] ||
          !st->v.res_scales[l - 1] || !st->slot[l - 1])
        return FLASHLOOP_ERR_INVALID_ARG;
    }
  }
  return launch_qkv_quant_gemm(p, loop, x, active, active ? n_active : nullptr,
                               active ? capacity_of(p, loop) : p->seq, w_qkv, st, q_out, as_stream(stream));
}

int flashloop_topk_columns(const flashloop_params* p, const float* mass, const int32_t* candidates,
                           int32_t n_cand, int32_t k, int32_t* out, void* stream) {
  int rc = check_common(p);
  if (rc != FLASHLOOP_OK) return rc;
  if (!mass || !out) return FLASHLOOP_ERR_INVALID_ARG;
  const int n = candidates ? n_cand : p->seq;
  if (n < 1 || n > p->seq) return FLASHLOOP_ERR_INVALID_ARG;
  if (n > 49152) return FLASHLOOP_ERR_UNSUPPORTED;
  if (k < 1 || k > n) return FLASHLOOP_ERR_INVALID_ARG;
  return launch_topk(p, mass, candidates, n_cand, k, out, nullptr, as_stream(stream));
}

// The pages' streams of loops 1..loop are present (params.kv_scheme == 1).
static int check_paper_streams(const flashloop_params* p, const flashloop_state* st, int loop) {
  if (!st->paper_k || !st->paper_v) return FLASHLOOP_ERR_INVALID_ARG;
  for (const flashloop_paper_kv* kv : {st->paper_k, st->paper_v})
    for (int r = 1; r <= loop; ++r)
      if (!kv->codes[r - 1] || !kv->scale[r - 1] || !kv->minv[r - 1] || !kv->tail[r - 1])
        return FLASHLOOP_ERR_INVALID_ARG;
  (void)p;
  return FLASHLOOP_OK;
}

static int check_state(const flashloop_params* p, const flashloop_state* st, int loop) {
  if (!st || !st->n_active || !st->O || !st->err_word || !st->workspace) return FLASHLOOP_ERR_INVALID_ARG;
  if (st->workspace_bytes < workspace_layout(p).total) return FLASHLOOP_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (!st->q[i] || !st->m[i] || !st->Z[i] || !st->N[i]) return FLASHLOOP_ERR_INVALID_ARG;
  if (!st->colmass[0]) return FLASHLOOP_ERR_INVALID_ARG;
  if (p->fixed_mass)
    for (int i = 0; i < 3; ++i)
      if (!st->G[i]) return FLASHLOOP_ERR_INVALID_ARG;
  for (int r = 2; r <= loop; ++r)
    if (!st->active[r - 1] || !st->slot[r - 1]) return FLASHLOOP_ERR_INVALID_ARG;
  if (p->kv_scheme == 1) {
    if (check_paper_streams(p, st, loop) != FLASHLOOP_OK) return FLASHLOOP_ERR_INVALID_ARG;
  } else {
    if (!st->k.base_codes || !st->v.base_codes) return FLASHLOOP_ERR_INVALID_ARG;
    for (int r = 2; r <= loop; ++r)
      if (!st->k.res_codes[r - 1] || !st->v.res_codes[r - 1] || !st->k.res_scales[r - 1] ||
          !st->v.res_scales[r - 1])
        return FLASHLOOP_ERR_INVALID_ARG;
  }
  if (loop >= 2) {
    const int sel = flashloop_selection_loop(p, loop);
    if (!st->cols[sel - 1]) return FLASHLOOP_ERR_INVALID_ARG;
  }
  return FLASHLOOP_OK;
}

// Buffers of the rebuilt selected columns inside the workspace: K as
// [H, kcp, dh], V transposed as [H, dh, kcp] (kcp = kc rounded up to 8).
struct ColBuffers {
  int kc, kcp;
  const int32_t* cols;
  __half *k_new, *v_new, *k_old, *v_old;
};

static ColBuffers col_buffers(const flashloop_params* p, int loop, flashloop_state* st) {
  const Workspace w = workspace_layout(p);
  ColBuffers b{};
  const bool dense = loop == 1;
  const int sel = dense ? 1 : flashloop_selection_loop(p, loop);
  b.kc = dense ? p->seq : p->topk[sel - 1];
  b.kcp = pad8(b.kc);
  b.cols = dense ? nullptr : st->cols[sel - 1];
  __half* base = ws_ptr<__half>(st->workspace, w.cols_kv);
  const size_t one = (size_t)p->n_heads * b.kcp * p->head_dim;
  b.k_new = base;
  b.v_new = base + one;
  b.k_old = dense ? nullptr : base + 2 * one;
  b.v_old = dense ? nullptr : base + 3 * one;
  return b;
}

int flashloop_selcol_dequant(const flashloop_params* p, int32_t loop, flashloop_state* st,
                             void* stream) {
  int rc = check_common(p);
  if (rc != FLASHLOOP_OK) return rc;
  if (loop < 1 || loop > p->n_loops) return FLASHLOOP_ERR_INVALID_ARG;
  rc = check_state(p, st, loop);
  if (rc != FLASHLOOP_OK) return rc;
  const ColBuffers b = col_buffers(p, loop, st);
  if (p->kv_scheme == 1)
    return launch_paper_selcol(p, loop, b.cols, b.kc, b.kcp, st, b.k_old, b.k_new, b.v_old, b.v_new,
                               as_stream(stream));
  return launch_selcol_dequant(p, loop, b.cols, b.kc, b.kcp, st, b.k_old, b.k_new, b.v_old, b.v_new,
                               as_stream(stream));
}

int flashloop_paper_kv_quant(const flashloop_params* p, int32_t loop, const float* k_new, const float* v_new,
                             const int32_t* active, const int32_t* n_active, flashloop_state* st, void* stream) {
  int rc = check_common(p);
  if (rc != FLASHLOOP_OK) return rc;
  if (p->kv_scheme != 1) return FLASHLOOP_ERR_UNSUPPORTED;
  if (loop < 1 || loop > p->n_loops || !k_new || !v_new || !st || !st->err_word) return FLASHLOOP_ERR_INVALID_ARG;
  if (check_paper_streams(p, st, loop) != FLASHLOOP_OK) return FLASHLOOP_ERR_INVALID_ARG;
  if (loop >= 2) {
    if (!active || !n_active) return FLASHLOOP_ERR_INVALID_ARG;
    for (int l = 2; l <= loop; ++l)
      if (!st->slot[l - 1]) return FLASHLOOP_ERR_INVALID_ARG;
  }
  return launch_paper_quant(p, loop, k_new, v_new, loop == 1 ? nullptr : active, loop == 1 ? nullptr : n_active,
                            capacity_of(p, loop), st, as_stream(stream));
}

int flashloop_sparse_attn_update(const flashloop_params* p, int32_t loop, flashloop_state* st,
                                 int32_t want_colmass, void* stream) {
  int rc = check_common(p);
  if (rc != FLASHLOOP_OK) return rc;
  if (loop < 1 || loop > p->n_loops) return FLASHLOOP_ERR_INVALID_ARG;
  rc = check_state(p, st, loop);
  if (rc != FLASHLOOP_OK) return rc;
  if (want_colmass && loop >= 2 && !st->colmass[1]) return FLASHLOOP_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  const int dense = loop == 1;
  const ColBuffers b = col_buffers(p, loop, st);
  const int cur = slot_of_loop(loop), prev = dense ? 0 : slot_of_loop(loop - 1);
  AttnArgs a{};
  a.S = p->seq; a.H = p->n_heads; a.kc = b.kc; a.dense = dense;
  a.rows = dense ? nullptr : st->active[loop - 1];
  a.n_rows = dense ? nullptr : st->n_active + (loop - 1);
  a.row_cap = capacity_of(p, loop);
  a.cols = b.cols; a.k_new = b.k_new; a.v_new = b.v_new; a.k_old = b.k_old; a.v_old = b.v_old;
  a.q_new = st->q[cur]; a.q_old = st->q[prev];
  a.m_in = st->m[prev]; a.z_in = st->Z[prev]; a.n_in = st->N[prev];
  a.m_out = st->m[cur]; a.z_out = st->Z[cur]; a.n_out = st->N[cur];
  a.o = st->O;
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)p->head_dim);
  a.err = st->err_word;
  if (!dense) {
    // each active row's causal prefix of the selection, per head
    int32_t* cnt = ws_ptr<int32_t>(st->workspace, workspace_layout(p).row_cnt);
    rc = launch_attn_row_counts(a, cnt, s);
    if (rc != FLASHLOOP_OK) return rc;
    a.row_cnt = cnt;
  }
  if (p->fixed_mass && !dense) {
    // fixed-mass form: a statistics pass (frame m' and factor g per row), then the update
    a.g_in = st->G[prev];
    a.g_out = st->G[cur];
    a.mode = 1;
    rc = launch_attn_tc(p, a, b.kcp, s);
    if (rc != FLASHLOOP_OK) return rc;
    a.mode = 2;
  } else if (p->fixed_mass) {
    a.g_out = st->G[cur];  // the dense loop's distribution: g = 1
  }
  rc = launch_attn_tc(p, a, b.kcp, s);
  if (rc != FLASHLOOP_OK) return rc;
  if (dense || want_colmass) {
    ColmassArgs c{};
    c.S = p->seq; c.H = p->n_heads; c.kc = b.kc; c.kcp = b.kcp;
    c.rows = a.rows; c.n_rows = a.n_rows; c.row_cap = a.row_cap; c.cols = b.cols;
    c.k_new = b.k_new; c.q = st->q[cur]; c.m = st->m[cur]; c.z = st->Z[cur];
    c.out = dense ? st->colmass[0] : st->colmass[1];
    c.scale_log2 = 1.0f;  // the rebuilt keys already carry log2(e)/sqrt(dh)
    c.err = st->err_word;
    c.g = p->fixed_mass ? st->G[cur] : nullptr;
    const Workspace w = workspace_layout(p);
    rc = launch_colmass_tc(p, c, ws_ptr<void>(st->workspace, w.cm_q), ws_ptr<void>(st->workspace, w.cm_rows), s);
  }
  return rc;
}

int flashloop_out_proj(const flashloop_params* p, const uint16_t* o, const int32_t* active,
                       const int32_t* n_active, int32_t capacity, const uint16_t* w_o, uint16_t* y,
                       void* stream) {
  int rc = check_common(p);
  if (rc != FLASHLOOP_OK) return rc;
  if (!o || !w_o || !y) return FLASHLOOP_ERR_INVALID_ARG;
  if (active != nullptr && n_active == nullptr) return FLASHLOOP_ERR_INVALID_ARG;
  if (capacity < 1 || capacity > p->seq) return FLASHLOOP_ERR_INVALID_ARG;
  return launch_out_gemm(p, o, active, n_active, capacity, w_o, y, nullptr, as_stream(stream));
}

int flashloop_loop_step(const flashloop_params* p, int32_t loop, const uint16_t* x_cur,
                        const uint16_t* x_prev, const uint16_t* w_qkv, const uint16_t* w_o,
                        flashloop_state* st, void* stream) {
  int rc = check_common(p);
  if (rc != FLASHLOOP_OK) return rc;
  if (loop < 1 || loop > p->n_loops || !x_cur || !w_qkv || !w_o || !st || !st->Y || !st->rope_cs)
    return FLASHLOOP_ERR_INVALID_ARG;
  if (loop >= 2 && !x_prev) return FLASHLOOP_ERR_INVALID_ARG;
  if (loop >= 2 && p->gate_topk && p->seq > 49152) return FLASHLOOP_ERR_UNSUPPORTED;
  rc = check_state(p, st, loop);
  if (rc != FLASHLOOP_OK) return rc;
  cudaStream_t s = as_stream(stream);
  const int cur = slot_of_loop(loop);
  const int cap = capacity_of(p, loop);
  // the pages' cache setting: the projection writes float32 K / V of the active
  // rows to the workspace, then the asymmetric quantiser codes them
  float* kf = p->kv_scheme == 1 ? ws_ptr<float>(st->workspace, workspace_layout(p).kv_f32) : nullptr;
  float* vf = kf ? kf + (size_t)p->seq * p->d_model : nullptr;
  if (loop == 1) {
    if (p->kv_scheme == 1) {
      rc = launch_qkv_gemm(p, x_cur, nullptr, nullptr, p->seq, w_qkv, st->rope_cs, st->q[0], kf, vf, st->err_word, s);
      if (rc == FLASHLOOP_OK) rc = launch_paper_quant(p, 1, kf, vf, nullptr, nullptr, p->seq, st, s);
    } else {
      rc = launch_qkv_quant_gemm(p, 1, x_cur, nullptr, nullptr, p->seq, w_qkv, st, st->q[0], s);
    }
    if (rc != FLASHLOOP_OK) return rc;
    rc = flashloop_selcol_dequant(p, 1, st, stream);
    if (rc != FLASHLOOP_OK) return rc;
    rc = flashloop_sparse_attn_update(p, 1, st, 1, stream);
    if (rc != FLASHLOOP_OK) return rc;
    return launch_out_gemm(p, st->O, nullptr, nullptr, p->seq, w_o, st->Y, st->err_word, s);
  }
  int32_t* act = st->active[loop - 1];
  int32_t* n_act = st->n_active + (loop - 1);
  const int32_t* prev_act = loop == 2 ? nullptr : st->active[loop - 2];
  const int32_t* n_prev = loop == 2 ? nullptr : st->n_active + (loop - 2);
  if (p->gate_topk)
    rc = launch_gate_topk(p, x_cur, x_prev, prev_act, n_prev, capacity_of(p, loop - 1), cap, act,
                          st->slot[loop - 1], n_act, st->workspace, st->err_word, s);
  else
    rc = launch_gate(p, x_cur, x_prev, prev_act, n_prev, capacity_of(p, loop - 1), act,
                     st->slot[loop - 1], n_act, cap, st->workspace, st->err_word, s);
  if (rc != FLASHLOOP_OK) return rc;
  if (p->kv_scheme == 1) {
    rc = launch_qkv_gemm(p, x_cur, act, n_act, cap, w_qkv, st->rope_cs, st->q[cur], kf, vf, st->err_word, s);
    if (rc == FLASHLOOP_OK) rc = launch_paper_quant(p, loop, kf, vf, act, n_act, cap, st, s);
  } else {
    rc = launch_qkv_quant_gemm(p, loop, x_cur, act, n_act, cap, w_qkv, st, st->q[cur], s);
  }
  if (rc != FLASHLOOP_OK) return rc;
  const int sel = flashloop_selection_loop(p, loop);
  if (sel == loop && loop == 2 && p->seq > 49152) return FLASHLOOP_ERR_UNSUPPORTED;
  if (sel == loop) {
    const int k = p->topk[loop - 1];
    if (loop == 2) {
      rc = launch_topk(p, st->colmass[0], nullptr, 0, k, st->cols[loop - 1], st->err_word, s);
    } else {
      const int prev_sel = flashloop_selection_loop(p, loop - 1);
      rc = launch_topk(p, st->colmass[1], st->cols[prev_sel - 1], p->topk[prev_sel - 1], k,
                       st->cols[loop - 1], st->err_word, s);
    }
    if (rc != FLASHLOOP_OK) return rc;
  }
  const int want_cm = (loop < p->n_loops && p->topk[loop] < p->topk[loop - 1]) ? 1 : 0;
  rc = flashloop_selcol_dequant(p, loop, st, stream);
  if (rc != FLASHLOOP_OK) return rc;
  rc = flashloop_sparse_attn_update(p, loop, st, want_cm, stream);
  if (rc != FLASHLOOP_OK) return rc;
  return launch_out_gemm(p, st->O, act, n_act, cap, w_o, st->Y, st->err_word, s);
}

size_t flashloop_kv_workspace_bytes(const flashloop_params* p) {
  if (check_params(p) != FLASHLOOP_OK) return 0;
  return workspace_layout(p).keys + (size_t)p->seq * sizeof(float);
}

int flashloop_kv_step(const flashloop_params* p, int32_t loop, const uint16_t* x_cur, const uint16_t* x_prev,
                      const uint16_t* w_qkv, flashloop_state* st, void* stream) {
  int rc = check_common(p);
  if (rc != FLASHLOOP_OK) return rc;
  if (loop < 1 || loop > p->n_loops || !x_cur || !w_qkv || !st || !st->rope_cs || !st->err_word)
    return FLASHLOOP_ERR_INVALID_ARG;
  if (p->kv_scheme != 0) return FLASHLOOP_ERR_UNSUPPORTED;  // decode contexts keep the INT8 / INT4 / INT2 streams
  if (!st->k.base_codes || !st->k.base_scales || !st->v.base_codes || !st->v.base_scales)
    return FLASHLOOP_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  if (loop == 1) return launch_qkv_quant_gemm(p, 1, x_cur, nullptr, nullptr, p->seq, w_qkv, st, nullptr, s);
  if (!x_prev || !st->n_active || !st->workspace || st->workspace_bytes < flashloop_kv_workspace_bytes(p))
    return FLASHLOOP_ERR_INVALID_ARG;
  if (p->gate_topk && p->seq > 49152) return FLASHLOOP_ERR_UNSUPPORTED;
  for (int l = 2; l <= loop; ++l)
    if (!st->active[l - 1] || !st->slot[l - 1] || !st->k.res_codes[l - 1] || !st->k.res_scales[l - 1] ||
        !st->v.res_codes[l - 1] || !st->v.res_scales[l - 1])
      return FLASHLOOP_ERR_INVALID_ARG;
  int32_t* act = st->active[loop - 1];
  int32_t* n_act = st->n_active + (loop - 1);
  const int cap = capacity_of(p, loop);
  if (p->gate_topk)
    rc = launch_gate_topk(p, x_cur, x_prev, loop == 2 ? nullptr : st->active[loop - 2],
                          loop == 2 ? nullptr : st->n_active + (loop - 2), capacity_of(p, loop - 1), cap, act,
                          st->slot[loop - 1], n_act, st->workspace, st->err_word, s);
  else
    rc = launch_gate(p, x_cur, x_prev, loop == 2 ? nullptr : st->active[loop - 2],
                     loop == 2 ? nullptr : st->n_active + (loop - 2), capacity_of(p, loop - 1), act,
                     st->slot[loop - 1], n_act, cap, st->workspace, st->err_word, s);
  if (rc != FLASHLOOP_OK) return rc;
  return launch_qkv_quant_gemm(p, loop, x_cur, act, n_act, cap, w_qkv, st, nullptr, s);
}

// ---------------------------------------------------------------------------
// decode
// ---------------------------------------------------------------------------
static int check_decode_params(const flashloop_params* p) {
  int rc = check_params(p);
  if (rc != FLASHLOOP_OK) return rc;
  if (p->batch < 1 || p->batch > 64) return FLASHLOOP_ERR_INVALID_ARG;
  if (p->fixed_mass) return FLASHLOOP_ERR_UNSUPPORTED;  // decode keeps the running (m, N, Z) form
  if (p->kv_scheme != 0) return FLASHLOOP_ERR_UNSUPPORTED;  // decode reads the INT8 / INT4 / INT2 streams
  const int hd = p->n_heads * p->head_dim, hg = hd / 32;
  if (hd % 256 != 0 || 256 % hg != 0 || hg % 8 != 0) return FLASHLOOP_ERR_UNSUPPORTED;
  if (p->n_loops >= 2 && p->topk[1] > p->seq + 1) return FLASHLOOP_ERR_INVALID_ARG;
  return FLASHLOOP_OK;
}

static int check_decode_common(const flashloop_params* p, const flashloop_decode_state* ds) {
  int rc = check_decode_params(p);
  if (rc != FLASHLOOP_OK) return rc;
  rc = check_arch();
  if (rc != FLASHLOOP_OK) return rc;
  if (!ds || !ds->err_word || !ds->workspace || !ds->O) return FLASHLOOP_ERR_INVALID_ARG;
  if (ds->workspace_bytes < decode_layout(p).total) return FLASHLOOP_ERR_INVALID_ARG;
  return FLASHLOOP_OK;
}

static int check_decode_state(const flashloop_params* p, int loop, const flashloop_state* ctx,
                              const flashloop_decode_state* ds) {
  if (!ctx || !ds) return FLASHLOOP_ERR_INVALID_ARG;
  if (!ctx->k.base_codes || !ctx->k.base_scales || !ctx->v.base_codes || !ctx->v.base_scales ||
      !ds->k.base_codes || !ds->k.base_scales || !ds->v.base_codes || !ds->v.base_scales)
    return FLASHLOOP_ERR_INVALID_ARG;
  for (int l = 2; l <= loop; ++l)
    if (!ctx->slot[l - 1] || !ctx->k.res_codes[l - 1] || !ctx->k.res_scales[l - 1] || !ctx->v.res_codes[l - 1] ||
        !ctx->v.res_scales[l - 1] || !ds->k.res_codes[l - 1] || !ds->k.res_scales[l - 1] ||
        !ds->v.res_codes[l - 1] || !ds->v.res_scales[l - 1])
      return FLASHLOOP_ERR_INVALID_ARG;
  const int cur = slot_of_loop(loop);
  if (!ds->q[cur] || !ds->m[cur] || !ds->Z[cur] || !ds->N[cur]) return FLASHLOOP_ERR_INVALID_ARG;
  if (loop >= 2) {
    const int prev = slot_of_loop(loop - 1);
    if (!ds->q[prev] || !ds->m[prev] || !ds->Z[prev] || !ds->N[prev]) return FLASHLOOP_ERR_INVALID_ARG;
  }
  if (p->n_loops >= 2 && !ds->cols) return FLASHLOOP_ERR_INVALID_ARG;
  if (loop == 1 && !ds->probs) return FLASHLOOP_ERR_INVALID_ARG;
  return FLASHLOOP_OK;
}

size_t flashloop_decode_workspace_bytes(const flashloop_params* p) {
  if (check_decode_params(p) != FLASHLOOP_OK) return 0;
  return decode_layout(p).total;
}

int flashloop_decode_qkv(const flashloop_params* p, int32_t loop, const uint16_t* x_tok, const uint16_t* w_qkv,
                         flashloop_decode_state* ds, void* stream) {
  int rc = check_decode_common(p, ds);
  if (rc != FLASHLOOP_OK) return rc;
  if (loop < 1 || loop > p->n_loops || !x_tok || !w_qkv || !ds->rope_cs || !ds->q[slot_of_loop(loop)])
    return FLASHLOOP_ERR_INVALID_ARG;
  if (!ds->k.base_codes || !ds->k.base_scales || !ds->v.base_codes || !ds->v.base_scales)
    return FLASHLOOP_ERR_INVALID_ARG;
  for (int l = 2; l <= loop; ++l)
    if (!ds->k.res_codes[l - 1] || !ds->k.res_scales[l - 1] || !ds->v.res_codes[l - 1] || !ds->v.res_scales[l - 1])
      return FLASHLOOP_ERR_INVALID_ARG;
  return launch_decode_qkv(p, loop, x_tok, w_qkv, ds, as_stream(stream));
}

int flashloop_decode_attn(const flashloop_params* p, int32_t loop, const flashloop_state* ctx,
                          flashloop_decode_state* ds, void* stream) {
  int rc = check_decode_common(p, ds);
  if (rc != FLASHLOOP_OK) return rc;
  if (loop < 1 || loop > p->n_loops) return FLASHLOOP_ERR_INVALID_ARG;
  rc = check_decode_state(p, loop, ctx, ds);
  if (rc != FLASHLOOP_OK) return rc;
  return launch_decode_attn(p, loop, ctx, ds, as_stream(stream));
}

int flashloop_decode_select(const flashloop_params* p, flashloop_decode_state* ds, void* stream) {
  int rc = check_decode_common(p, ds);
  if (rc != FLASHLOOP_OK) return rc;
  if (p->n_loops < 2 || !ds->probs || !ds->cols) return FLASHLOOP_ERR_INVALID_ARG;
  if (p->seq + 1 > 49152) return FLASHLOOP_ERR_UNSUPPORTED;
  return launch_decode_select(p, ds, as_stream(stream));
}

int flashloop_decode_out(const flashloop_params* p, const uint16_t* w_o, flashloop_decode_state* ds,
                         void* stream) {
  int rc = check_decode_common(p, ds);
  if (rc != FLASHLOOP_OK) return rc;
  if (!w_o || !ds->Y) return FLASHLOOP_ERR_INVALID_ARG;
  return launch_decode_out(p, w_o, ds, as_stream(stream));
}

int flashloop_decode_step(const flashloop_params* p, int32_t loop, const uint16_t* x_tok,
                          const uint16_t* w_qkv, const uint16_t* w_o, const flashloop_state* ctx,
                          flashloop_decode_state* ds, void* stream) {
  int rc = check_decode_common(p, ds);
  if (rc != FLASHLOOP_OK) return rc;
  if (loop < 1 || loop > p->n_loops || !x_tok || !w_qkv || !w_o || !ds->rope_cs || !ds->Y)
    return FLASHLOOP_ERR_INVALID_ARG;
  rc = check_decode_state(p, loop, ctx, ds);
  if (rc != FLASHLOOP_OK) return rc;
  if (loop == 1 && p->n_loops >= 2 && p->seq + 1 > 49152) return FLASHLOOP_ERR_UNSUPPORTED;
  cudaStream_t s = as_stream(stream);
  rc = launch_decode_qkv(p, loop, x_tok, w_qkv, ds, s);
  if (rc != FLASHLOOP_OK) return rc;
  rc = launch_decode_attn(p, loop, ctx, ds, s);
  if (rc != FLASHLOOP_OK) return rc;
  if (loop == 1 && p->n_loops >= 2) {
    rc = launch_decode_select(p, ds, s);
    if (rc != FLASHLOOP_OK) return rc;
  }
  return launch_decode_out(p, w_o, ds, s);
}

int flashloop_check_error_word(const int32_t* err_word, int32_t* code, void* stream) {
  if (!err_word) return FLASHLOOP_ERR_INVALID_ARG;
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, err_word, sizeof(v), cudaMemcpyDeviceToHost, as_stream(stream)) != cudaSuccess)
    return FLASHLOOP_ERR_CUDA;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return FLASHLOOP_ERR_CUDA;
  if (code) *code = v;
  return v == 0 ? FLASHLOOP_OK : FLASHLOOP_ERR_DEVICE;
}

const char* flashloop_status_string(int status) {
  switch (status) {
    case FLASHLOOP_OK: return "ok";
    case FLASHLOOP_ERR_INVALID_ARG: return "invalid argument";
    case FLASHLOOP_ERR_UNSUPPORTED: return "unsupported shape or bit width";
    case FLASHLOOP_ERR_CUDA: return "CUDA runtime error";
    case FLASHLOOP_ERR_DEVICE: return "device-side check failed (see error word)";
    case FLASHLOOP_ERR_ARCH: return "device is not sm_100";
    default: return "unknown status";
  }
}

}  // extern "C"
