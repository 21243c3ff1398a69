// (f2) The pages' own cache setting [FlashLoop App. E "Quantization setting";
// the "Looping a Transformer Quadruples the Bill" page, §3]: INT4 asymmetric
// codes in groups of 64 (value = code * scale + minimum, codes 0..15, fp16
// scale and minimum per group), keys grouped per channel over 64 consecutive
// rows, values per row over 64 consecutive channels, the last 64 tokens kept
// in bf16.  Loop 1 codes the values of the body tokens; loop r >= 2 codes,
// for its active body tokens, the residual against the reconstruction of loop
// r-1 (row = the token's position in the loop's active list).
//
// Kernels:
//   paper_key_quant_kernel   one block per (64-row group, head), four threads per
//                            channel, 16 rows each: the residuals in registers,
//                            the group's minimum and maximum through shared
//                            memory, scale, minimum, codes (two channels share a
//                            byte: lanes pair up);
//   paper_value_quant_kernel one warp per (row, head, 64-channel group), two
//                            channels per lane, warp reductions;
//   paper_tail_kernel        bf16 copies of the tail tokens active at the loop;
//   paper_selcol_kernel      the selected columns' reconstructions of loops r-1
//                            and r (loop 1: every token), rebuilt as the fp16
//                            keys (scaled by log2(e)/sqrt(dh)) and transposed
//                            values the attention kernels read.
// Reconstruction follows the definition: the loop-1 codes dequantised, then in
// loop order the residual of every loop where the token was active, float32
// additions; a tail token's value is the bf16 value of the latest loop <= r
// that stored it.
#include "common.cuh"

namespace fl {

constexpr int kPaperGroup = FLASHLOOP_PAPER_GROUP;
constexpr float kPaperLevels = 15.f;
constexpr int kPaperKeyQ = 4;  // threads per channel in the key quantiser (16 of a group's 64 rows each)

struct PaperStreams {
  const uint8_t* codes[FLASHLOOP_MAX_LOOPS];
  const uint16_t* scale[FLASHLOOP_MAX_LOOPS];
  const uint16_t* minv[FLASHLOOP_MAX_LOOPS];
  const uint16_t* tail[FLASHLOOP_MAX_LOOPS];
};

struct PaperOut {  // the streams of the loop being written
  uint8_t* codes;
  uint16_t* scale;
  uint16_t* minv;
  uint16_t* tail;
};

inline PaperStreams paper_streams(const flashloop_paper_kv& kv) {
  PaperStreams s{};
  for (int i = 0; i < FLASHLOOP_MAX_LOOPS; ++i) {
    s.codes[i] = kv.codes[i];
    s.scale[i] = kv.scale[i];
    s.minv[i] = kv.minv[i];
    s.tail[i] = kv.tail[i];
  }
  return s;
}

__device__ __forceinline__ float half_bits_f(uint16_t b) { return __half2float(__ushort_as_half(b)); }

// code * scale + minimum of element c of stream row `row` (loop l): the product
// is exact (4-bit code, fp16 scale), so one fused rounding equals the product
// followed by the addition.
template <int DH, bool KEY>
__device__ __forceinline__ float paper_deq(const PaperStreams& ps, int l, int row, int h, int H, int c) {
  const uint8_t b = ps.codes[l - 1][((size_t)row * H + h) * (DH / 2) + (c >> 1)];
  const int code = (c & 1) ? (b >> 4) : (b & 15);
  const size_t gi = KEY ? ((size_t)(row / kPaperGroup) * H + h) * DH + c
                        : ((size_t)row * H + h) * (DH / kPaperGroup) + c / kPaperGroup;
  return fmaf(static_cast<float>(code), half_bits_f(ps.scale[l - 1][gi]), half_bits_f(ps.minv[l - 1][gi]));
}

// Reconstruction of element c of token t at loop `upto` (>= 1).
template <int DH, bool KEY>
__device__ __forceinline__ float paper_recon(const PaperStreams& ps, const LoopTables& lt, int body, int t, int h,
                                             int H, int c, int upto) {
  if (t >= body) {
    int l = upto;
    while (l > 1 && lt.slot[l - 1][t] < 0) --l;  // the latest loop <= upto that stored the token
    return bf16_bits_to_float(ps.tail[l - 1][((size_t)(t - body) * H + h) * DH + c]);
  }
  float acc = paper_deq<DH, KEY>(ps, 1, t, h, H, c);
  for (int l = 2; l <= upto; ++l) {
    const int sl = lt.slot[l - 1][t];
    if (sl >= 0) acc = acc + paper_deq<DH, KEY>(ps, l, sl, h, H, c);
  }
  return acc;
}

// Number of rows of this loop that are body tokens: loop 1 the body; loop r
// the active tokens below `body` (the active list ascends).
__device__ __forceinline__ int paper_body_rows(const int32_t* active, int n_rows, int body) {
  if (active == nullptr) return min(n_rows, body);
  int lo = 0, hi = n_rows;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(active + mid) < body) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// Scale, minimum and codes of one group from its minimum and maximum (float32,
// IEEE division, round-half-even, clamp to 0..15; a zero scale gives code 0).
__device__ __forceinline__ void paper_group_params(float mn, float mx, uint16_t& s16, uint16_t& lo16, float& s,
                                                   float& lo) {
  lo16 = __half_as_ushort(__float2half_rn(mn));
  s16 = __half_as_ushort(__float2half_rn(__fdiv_rn(mx - mn, kPaperLevels)));
  s = half_bits_f(s16);
  lo = half_bits_f(lo16);
}

__device__ __forceinline__ uint32_t paper_code(float x, float s, float lo) {
  if (!(s > 0.f)) return 0u;
  const float q = rintf(__fdiv_rn(__fsub_rn(x, lo), s));
  return static_cast<uint32_t>(fminf(fmaxf(q, 0.f), kPaperLevels));
}

template <int DH>
__global__ void __launch_bounds__(kPaperKeyQ * DH)
paper_key_quant_kernel(const float* __restrict__ x, const int32_t* __restrict__ active,
                       const int32_t* __restrict__ n_active, int n_cap, int S, int H, int body, int loop,
                       PaperStreams ps, LoopTables lt, PaperOut out, int32_t* err) {
  constexpr int kR = kPaperGroup / kPaperKeyQ;  // rows per thread
  __shared__ int s_rows;
  __shared__ float s_mn[kPaperKeyQ][DH], s_mx[kPaperKeyQ][DH];
  const int c = threadIdx.x % DH, q = threadIdx.x / DH;
  const int h = blockIdx.y, g = blockIdx.x;
  if (threadIdx.x == 0) {
    int n = active ? *n_active : S;
    if (n > n_cap) n = n_cap;
    s_rows = paper_body_rows(active, n < 0 ? 0 : n, body);
  }
  __syncthreads();
  const int rows = s_rows;
  const int r0 = g * kPaperGroup + q * kR;
  if (g * kPaperGroup >= rows) return;  // the whole block: no row of this group
  float rho[kR];
  float mn = INFINITY, mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < kR; ++i) {
    const int row = r0 + i;
    rho[i] = 0.f;
    if (row < rows) {
      const int t = active ? __ldg(active + row) : row;
      float v = x[((size_t)row * H + h) * DH + c];
      if (t < 0 || t >= S) {
        set_error(err, FLASHLOOP_DEVERR_INDEX);
      } else if (loop > 1) {
        v = __fsub_rn(v, paper_recon<DH, true>(ps, lt, body, t, h, H, c, loop - 1));
      }
      rho[i] = v;
      mn = fminf(mn, v);
      mx = fmaxf(mx, v);
    }
  }
  // the group's minimum and maximum over its 64 rows (kPaperKeyQ threads per channel)
  s_mn[q][c] = mn;
  s_mx[q][c] = mx;
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kPaperKeyQ; ++k) {
    mn = fminf(mn, s_mn[k][c]);
    mx = fmaxf(mx, s_mx[k][c]);
  }
  uint16_t s16, lo16;
  float s, lo;
  paper_group_params(mn, mx, s16, lo16, s, lo);
  if (q == 0) {
    const size_t gi = ((size_t)g * H + h) * DH + c;
    out.scale[gi] = s16;
    out.minv[gi] = lo16;
  }
#pragma unroll
  for (int i = 0; i < kR; ++i) {
    const int row = r0 + i;
    const uint32_t code = paper_code(rho[i], s, lo);
    const uint32_t other = __shfl_down_sync(0xffffffffu, code, 1);  // channel c + 1
    if (row < rows && (c & 1) == 0) out.codes[((size_t)row * H + h) * (DH / 2) + (c >> 1)] = (uint8_t)(code | (other << 4));
  }
}

template <int DH>
__global__ void __launch_bounds__(256)
paper_value_quant_kernel(const float* __restrict__ x, const int32_t* __restrict__ active,
                         const int32_t* __restrict__ n_active, int n_cap, int S, int H, int body, int loop,
                         PaperStreams ps, LoopTables lt, PaperOut out, int32_t* err) {
  constexpr int kGroups = DH / kPaperGroup;
  int n = active ? *n_active : S;
  if (n > n_cap) n = n_cap;
  if (n < 0) n = 0;
  const int rows = paper_body_rows(active, n, body);
  const int lane = threadIdx.x & 31;
  const long long items = (long long)rows * H * kGroups;
  for (long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); w < items; w += (long long)gridDim.x * 8) {
    const int gr = (int)(w % kGroups), h = (int)((w / kGroups) % H), row = (int)(w / ((long long)kGroups * H));
    const int t = active ? __ldg(active + row) : row;
    const int c0 = gr * kPaperGroup + 2 * lane;
    float v0 = x[((size_t)row * H + h) * DH + c0], v1 = x[((size_t)row * H + h) * DH + c0 + 1];
    if (t < 0 || t >= S) {
      if (lane == 0) set_error(err, FLASHLOOP_DEVERR_INDEX);
    } else if (loop > 1) {
      v0 = __fsub_rn(v0, paper_recon<DH, false>(ps, lt, body, t, h, H, c0, loop - 1));
      v1 = __fsub_rn(v1, paper_recon<DH, false>(ps, lt, body, t, h, H, c0 + 1, loop - 1));
    }
    float mn = fminf(v0, v1), mx = fmaxf(v0, v1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    uint16_t s16, lo16;
    float s, lo;
    paper_group_params(mn, mx, s16, lo16, s, lo);
    if (lane == 0) {
      const size_t gi = ((size_t)row * H + h) * kGroups + gr;
      out.scale[gi] = s16;
      out.minv[gi] = lo16;
    }
    out.codes[((size_t)row * H + h) * (DH / 2) + (c0 >> 1)] =
        (uint8_t)(paper_code(v0, s, lo) | (paper_code(v1, s, lo) << 4));
  }
}

// bf16 copies of the loop's active tail tokens (k and v, x rows as above).
template <int DH>
__global__ void __launch_bounds__(256)
paper_tail_kernel(const float* __restrict__ k, const float* __restrict__ v, const int32_t* __restrict__ active,
                  const int32_t* __restrict__ n_active, int n_cap, int S, int H, int body, uint16_t* k_tail,
                  uint16_t* v_tail) {
  int n = active ? *n_active : S;
  if (n > n_cap) n = n_cap;
  if (n < 0) n = 0;
  const int first = paper_body_rows(active, n, body);
  const long long per = (long long)H * DH;
  const long long items = (long long)(n - first) * per;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < items;
       i += (long long)gridDim.x * blockDim.x) {
    const int row = first + (int)(i / per);
    const int t = active ? __ldg(active + row) : row;
    if (t < body || t >= S) continue;
    const size_t e = (size_t)(i % per);
    const size_t dst = (size_t)(t - body) * per + e;
    k_tail[dst] = float_to_bf16_bits(k[(size_t)row * per + e]);
    v_tail[dst] = float_to_bf16_bits(v[(size_t)row * per + e]);
  }
}

// E consecutive elements c0.. of stream row `row` (loop l) dequantised: the
// same arithmetic as paper_deq, with the codes, scales and minima of the
// lane's slice loaded together.
template <int DH, bool KEY, int E>
__device__ __forceinline__ void paper_deq_vec(const PaperStreams& ps, int l, int row, int h, int H, int c0,
                                              float (&out)[E]) {
  const uint8_t* cp = ps.codes[l - 1] + ((size_t)row * H + h) * (DH / 2) + (c0 >> 1);
  uint32_t cw;
  if (E == 4) cw = *reinterpret_cast<const uint16_t*>(cp);
  else cw = *cp;
  if (KEY) {
    const size_t gi = ((size_t)(row / kPaperGroup) * H + h) * DH + c0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float code = static_cast<float>((cw >> (4 * e)) & 15u);
      out[e] = fmaf(code, half_bits_f(ps.scale[l - 1][gi + e]), half_bits_f(ps.minv[l - 1][gi + e]));
    }
  } else {
    const size_t gi = ((size_t)row * H + h) * (DH / kPaperGroup) + c0 / kPaperGroup;
    const float sc = half_bits_f(ps.scale[l - 1][gi]), mn = half_bits_f(ps.minv[l - 1][gi]);
#pragma unroll
    for (int e = 0; e < E; ++e) out[e] = fmaf(static_cast<float>((cw >> (4 * e)) & 15u), sc, mn);
  }
}

// (a5) in the pages' setting: the selected columns' reconstructions of loops
// r-1 and r (loop 1: of every token), as fp16 K [H, kcp, dh] scaled by kscale
// and transposed V [H, dh, kcp].  One block = 64 columns of one head; a warp
// takes one column at a time, each lane DH/32 consecutive elements; the sum
// over loops runs once, keeping loop r-1's value on the way; V rows are
// staged in shared memory and written transposed.
template <int DH>
__global__ void __launch_bounds__(256)
paper_selcol_kernel(const int32_t* __restrict__ cols, int kc, int kcp, int S, int H, int body, int loop,
                    float kscale, PaperStreams kps, PaperStreams vps, LoopTables lt, __half* k_old, __half* k_new,
                    __half* vt_old, __half* vt_new, int32_t* err) {
  constexpr int E = DH / 32;
  __shared__ __align__(16) __half sv[2][64][DH + 8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = blockIdx.y, j0 = blockIdx.x * 64;
  const bool has_old = loop > 1;
  const int c0 = lane * E;
  for (int cl = warp; cl < 64; cl += 8) {
    const int col = j0 + cl;
    int j = -1;
    if (col < kc) {
      j = cols ? cols[(size_t)h * kc + col] : col;
      if (j < 0 || j >= S) {
        if (lane == 0) set_error(err, FLASHLOOP_DEVERR_INDEX);
        j = -1;
      }
    }
    float kn[E], ko[E], vn[E], vo[E];
#pragma unroll
    for (int e = 0; e < E; ++e) kn[e] = ko[e] = vn[e] = vo[e] = 0.f;
    if (j >= body) {
      // a tail token: the bf16 value of the latest loop <= r (and <= r-1) that stored it
      int ln = loop;
      while (ln > 1 && lt.slot[ln - 1][j] < 0) --ln;
      int lo = has_old ? loop - 1 : 1;
      while (lo > 1 && lt.slot[lo - 1][j] < 0) --lo;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const size_t ti = ((size_t)(j - body) * H + h) * DH + c0 + e;
        kn[e] = bf16_bits_to_float(kps.tail[ln - 1][ti]);
        vn[e] = bf16_bits_to_float(vps.tail[ln - 1][ti]);
        if (has_old) {
          ko[e] = bf16_bits_to_float(kps.tail[lo - 1][ti]);
          vo[e] = bf16_bits_to_float(vps.tail[lo - 1][ti]);
        }
      }
    } else if (j >= 0) {
      // body: the loop-1 codes, then in loop order the residual of every loop
      // where the token was active (float32 additions, as paper_recon)
      paper_deq_vec<DH, true, E>(kps, 1, j, h, H, c0, kn);
      paper_deq_vec<DH, false, E>(vps, 1, j, h, H, c0, vn);
      if (loop == 2) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          ko[e] = kn[e];
          vo[e] = vn[e];
        }
      }
      for (int l = 2; l <= loop; ++l) {
        const int sl = lt.slot[l - 1][j];
        if (sl >= 0) {
          float dk[E], dv[E];
          paper_deq_vec<DH, true, E>(kps, l, sl, h, H, c0, dk);
          paper_deq_vec<DH, false, E>(vps, l, sl, h, H, c0, dv);
#pragma unroll
          for (int e = 0; e < E; ++e) {
            kn[e] = kn[e] + dk[e];
            vn[e] = vn[e] + dv[e];
          }
        }
        if (l == loop - 1) {
#pragma unroll
          for (int e = 0; e < E; ++e) {
            ko[e] = kn[e];
            vo[e] = vn[e];
          }
        }
      }
    }
    bool ok = true;
#pragma unroll
    for (int e = 0; e < E; ++e)
      ok = ok && half_range_ok(kn[e] * kscale) && half_range_ok(ko[e] * kscale) && half_range_ok(vn[e]) &&
           half_range_ok(vo[e]);
    if (!ok) set_error(err, FLASHLOOP_DEVERR_RANGE);
    if (col < kcp) {
      const size_t off = ((size_t)h * kcp + col) * DH + c0;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        k_new[off + e] = __float2half_rn(kn[e] * kscale);
        if (has_old) k_old[off + e] = __float2half_rn(ko[e] * kscale);
      }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
      sv[1][cl][c0 + e] = __float2half_rn(vn[e]);
      sv[0][cl][c0 + e] = __float2half_rn(vo[e]);
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < 2 * DH * 32; idx += 256) {
    const int which = idx / (DH * 32);
    if (which == 0 && !has_old) continue;
    const int rem = idx % (DH * 32);
    const int d = rem / 32, jp = (rem % 32) * 2;
    if (j0 + jp >= kcp) continue;
    __half* dst = (which == 0 ? vt_old : vt_new) + ((size_t)h * DH + d) * kcp + j0 + jp;
    *reinterpret_cast<__half2*>(dst) = __halves2half2(sv[which][jp][d], sv[which][jp + 1][d]);
  }
}

static int paper_tail_of(int S) { return S < FLASHLOOP_PAPER_TAIL ? S : FLASHLOOP_PAPER_TAIL; }

static PaperOut paper_out(const flashloop_paper_kv& kv, int loop) {
  PaperOut o{};
  o.codes = kv.codes[loop - 1];
  o.scale = kv.scale[loop - 1];
  o.minv = kv.minv[loop - 1];
  o.tail = kv.tail[loop - 1];
  return o;
}

int launch_paper_quant(const flashloop_params* p, int loop, const float* k, const float* v, const int32_t* active,
                       const int32_t* n_active, int n_cap, const flashloop_state* st, cudaStream_t stream) {
  const int S = p->seq, H = p->n_heads, dh = p->head_dim;
  const int body = S - paper_tail_of(S);
  const LoopTables lt = loop_tables(p, st);
  const PaperStreams kps = paper_streams(*st->paper_k), vps = paper_streams(*st->paper_v);
  const PaperOut ko = paper_out(*st->paper_k, loop), vo = paper_out(*st->paper_v, loop);
  const int rows_cap = loop == 1 ? body : n_cap;
  const dim3 kgrid((rows_cap + kPaperGroup - 1) / kPaperGroup > 0 ? (rows_cap + kPaperGroup - 1) / kPaperGroup : 1, H);
  long long vitems = (long long)rows_cap * H * (dh / kPaperGroup);
  int vgrid = (int)((vitems + 7) / 8);
  if (vgrid > 148 * 16) vgrid = 148 * 16;
  if (vgrid < 1) vgrid = 1;
  long long titems = (long long)paper_tail_of(S) * H * dh;
  int tgrid = (int)((titems + 255) / 256);
  if (tgrid < 1) tgrid = 1;
  if (dh == 128) {
    paper_key_quant_kernel<128><<<kgrid, kPaperKeyQ * 128, 0, stream>>>(k, active, n_active, n_cap, S, H, body, loop, kps, lt, ko,
                                                           st->err_word);
    paper_value_quant_kernel<128><<<vgrid, 256, 0, stream>>>(v, active, n_active, n_cap, S, H, body, loop, vps, lt,
                                                             vo, st->err_word);
    paper_tail_kernel<128><<<tgrid, 256, 0, stream>>>(k, v, active, n_active, n_cap, S, H, body, ko.tail, vo.tail);
  } else {
    paper_key_quant_kernel<64><<<kgrid, kPaperKeyQ * 64, 0, stream>>>(k, active, n_active, n_cap, S, H, body, loop, kps, lt, ko,
                                                         st->err_word);
    paper_value_quant_kernel<64><<<vgrid, 256, 0, stream>>>(v, active, n_active, n_cap, S, H, body, loop, vps, lt,
                                                            vo, st->err_word);
    paper_tail_kernel<64><<<tgrid, 256, 0, stream>>>(k, v, active, n_active, n_cap, S, H, body, ko.tail, vo.tail);
  }
  return launch_status();
}

int launch_paper_selcol(const flashloop_params* p, int loop, const int32_t* cols, int kc, int kcp,
                        const flashloop_state* st, __half* k_old, __half* k_new, __half* vt_old, __half* vt_new,
                        cudaStream_t stream) {
  const int S = p->seq, H = p->n_heads;
  const int body = S - paper_tail_of(S);
  const dim3 grid((kcp + 63) / 64, H);
  const LoopTables lt = loop_tables(p, st);
  const PaperStreams kps = paper_streams(*st->paper_k), vps = paper_streams(*st->paper_v);
  const float kscale = 1.4426950408889634f / sqrtf(static_cast<float>(p->head_dim));
  if (p->head_dim == 128)
    paper_selcol_kernel<128><<<grid, 256, 0, stream>>>(cols, kc, kcp, S, H, body, loop, kscale, kps, vps, lt, k_old,
                                                       k_new, vt_old, vt_new, st->err_word);
  else
    paper_selcol_kernel<64><<<grid, 256, 0, stream>>>(cols, kc, kcp, S, H, body, loop, kscale, kps, vps, lt, k_old,
                                                      k_new, vt_old, vt_new, st->err_word);
  return launch_status();
}

}  // namespace fl
