// (a3) Cross-loop KV residual quantisation and (a5) selected-column
// reconstruction.
//
// [FlashLoop §3.3, §4.3, App. D.3]: a quantised first-loop base plus, per
// later loop, a quantised residual against the reconstructed previous loop,
// stored for active tokens only.  Groups of 32 head_dim elements, symmetric
// codes, fp16 scales.  One warp handles one (token, head) vector of K or V:
// each lane owns E = dh/32 consecutive elements, a group is 32/E lanes, and
// the group maximum is a shuffle reduction.  Every decision uses IEEE
// float32 division and round-half-even, so codes are reproducible bit for
// bit from the same float32 input.
#include "common.cuh"

namespace fl {

constexpr int kQuantThreads = 256;

// fp16 scale of a group: fp16_rn(amax / qmax), clamped to the largest finite fp16.
__device__ __forceinline__ uint16_t group_scale(float amax, int qmax) {
  __half h = __float2half_rn(__fdiv_rn(amax, static_cast<float>(qmax)));
  uint16_t bits = __half_as_ushort(h);
  if ((bits & 0x7FFFu) == 0x7C00u) bits = (bits & 0x8000u) | 0x7BFFu;  // inf -> 65504
  return bits;
}

__device__ __forceinline__ float half_bits_to_float(uint16_t b) {
  return __half2float(__ushort_as_half(b));
}

// Rebuild Xhat^(upto) of one (token, head) for this lane's E elements:
// base, then the residual of every loop 2..upto where the token is present,
// added in loop order in float32.
template <int E, int DH>
__device__ __forceinline__ void reconstruct_lane(const KVStreams& kv, const LoopTables& lt, int t,
                                                 int h, int H, int upto, int lane, float (&acc)[E]) {
  const int e0 = lane * E;
  const int g = e0 / FLASHLOOP_GROUP;
  {
    const int8_t* row = kv.base_codes + ((size_t)t * H + h) * DH;
    const float s = half_bits_to_float(kv.base_scales[((size_t)t * H + h) * (DH / 32) + g]);
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = static_cast<float>(row[e0 + e]) * s;
  }
  for (int l = 2; l <= upto; ++l) {
    const int sl = lt.slot[l - 1] ? lt.slot[l - 1][t] : t;  // no slot map: every row present at its own index
    if (sl < 0) continue;
    const int b = lt.bits[l - 1];
    const uint8_t* row = kv.res_codes[l - 1] + ((size_t)sl * H + h) * (DH * b / 8);
    const float s = half_bits_to_float(kv.res_scales[l - 1][((size_t)sl * H + h) * (DH / 32) + g]);
    int c[E];
    unpack_codes<E>(row, e0, b, c);
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = acc[e] + static_cast<float>(c[e]) * s;
  }
}

// Quantise this lane's E values (one group spans 32/E lanes) and store the
// packed codes and the group scale at row `dst_row` of the given stream.
template <int E, int DH>
__device__ __forceinline__ void quantize_store(const float (&x)[E], int bits, int lane,
                                               uint8_t* codes_row, uint16_t* scales_row) {
  constexpr int kLanesPerGroup = 32 / E;
  const int qmax = (1 << (bits - 1)) - 1;
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
  for (int o = 1; o < kLanesPerGroup; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const uint16_t sbits = group_scale(amax, qmax);
  const float s = half_bits_to_float(sbits);
  uint32_t packed = 0;
  const uint32_t mask = (1u << bits) - 1u;
  const float rs = s > 0.f ? approx_rcp(s) : 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int c = s > 0.f ? static_cast<int>(quant_code(x[e], s, rs, qmax)) : 0;
    packed |= (static_cast<uint32_t>(c) & mask) << (e * bits);
  }
  const int lane_bits = E * bits;
  if (lane_bits >= 8) {
    uint8_t* dst = codes_row + (lane * lane_bits) / 8;
    if (lane_bits == 32) *reinterpret_cast<uint32_t*>(dst) = packed;
    else if (lane_bits == 16) *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(packed);
    else *dst = static_cast<uint8_t>(packed);
  } else {
    // 4 bits per lane: even lanes combine with their odd neighbour.
    const uint32_t other = __shfl_down_sync(0xffffffffu, packed, 1);
    if ((lane & 1) == 0) codes_row[lane / 2] = static_cast<uint8_t>(packed | (other << 4));
  }
  if ((lane % kLanesPerGroup) == 0) scales_row[(lane * E) / FLASHLOOP_GROUP] = sbits;
}

// loop == 1: INT8 base of every token.  loop >= 2: residual of the active rows.
template <int DH>
__global__ void __launch_bounds__(kQuantThreads)
kv_quant_kernel(const float* __restrict__ k_new, const float* __restrict__ v_new,
                const int32_t* __restrict__ active, const int32_t* __restrict__ n_ptr, int cap,
                int S, int H, int loop, KVStreams Ks, KVStreams Vs, LoopTables lt,
                uint8_t* k_codes_out, uint16_t* k_scales_out, uint8_t* v_codes_out,
                uint16_t* v_scales_out, int32_t* err) {
  constexpr int E = DH / 32;
  int n = (loop == 1 || active == nullptr) ? S : *n_ptr;
  if (n > cap) n = cap;
  const int lane = threadIdx.x & 31;
  const long long total = (long long)n * H * 2;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  const int bits = lt.bits[loop - 1];
  const int row_bytes = DH * bits / 8;
  for (long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < total;
       w += warps) {
    const int which = static_cast<int>(w & 1);  // 0 = K, 1 = V
    const int h = static_cast<int>((w >> 1) % H);
    const int a = static_cast<int>((w >> 1) / H);
    const int t = (loop == 1 || active == nullptr) ? a : active[a];
    if (t < 0 || t >= S) {
      if (lane == 0) set_error(err, FLASHLOOP_DEVERR_INDEX);
      continue;
    }
    const float* src = (which == 0 ? k_new : v_new) + ((size_t)a * H + h) * DH + lane * E;
    float x[E];
    if constexpr (E == 4) {
      const float4 v4 = *reinterpret_cast<const float4*>(src);
      x[0] = v4.x; x[1] = v4.y; x[2] = v4.z; x[3] = v4.w;
    } else {
      const float2 v2 = *reinterpret_cast<const float2*>(src);
      x[0] = v2.x; x[1] = v2.y;
    }
    if (loop >= 2) {
      float prev[E];
      reconstruct_lane<E, DH>(which == 0 ? Ks : Vs, lt, t, h, H, loop - 1, lane, prev);
#pragma unroll
      for (int e = 0; e < E; ++e) x[e] = x[e] - prev[e];
    }
    uint8_t* codes = (which == 0 ? k_codes_out : v_codes_out) + ((size_t)a * H + h) * row_bytes;
    uint16_t* scales = (which == 0 ? k_scales_out : v_scales_out) + ((size_t)a * H + h) * (DH / 32);
    quantize_store<E, DH>(x, bits, lane, codes, scales);
  }
}

int launch_kv_quant(const flashloop_params* p, int loop, const float* k_new, const float* v_new,
                    const int32_t* active, const int32_t* n_active, flashloop_state* st,
                    cudaStream_t stream) {
  const int cap = loop == 1 ? p->seq : p->capacity[loop - 1];
  const int H = p->n_heads;
  const long long items = (long long)cap * H * 2;
  long long grid = (items + (kQuantThreads / 32) - 1) / (kQuantThreads / 32);
  if (grid > 148 * 16) grid = 148 * 16;
  if (grid < 1) grid = 1;
  const KVStreams Ks = kv_streams(st->k), Vs = kv_streams(st->v);
  const LoopTables lt = loop_tables(p, st);
  uint8_t *kc, *vc;
  uint16_t *ks, *vs;
  if (loop == 1) {
    kc = reinterpret_cast<uint8_t*>(st->k.base_codes);
    vc = reinterpret_cast<uint8_t*>(st->v.base_codes);
    ks = st->k.base_scales;
    vs = st->v.base_scales;
  } else {
    kc = st->k.res_codes[loop - 1];
    vc = st->v.res_codes[loop - 1];
    ks = st->k.res_scales[loop - 1];
    vs = st->v.res_scales[loop - 1];
  }
  if (p->head_dim == 128) {
    kv_quant_kernel<128><<<(int)grid, kQuantThreads, 0, stream>>>(
        k_new, v_new, active, n_active, cap, p->seq, H, loop, Ks, Vs, lt, kc, ks, vc, vs, st->err_word);
  } else {
    kv_quant_kernel<64><<<(int)grid, kQuantThreads, 0, stream>>>(
        k_new, v_new, active, n_active, cap, p->seq, H, loop, Ks, Vs, lt, kc, ks, vc, vs, st->err_word);
  }
  return launch_status();
}

// The same quantisation for n_rows rows that are present at every loop (the
// decode tokens): row a of k_new / v_new goes to row a of the base (loop 1)
// or of the loop's residual stream, and reconstruction reads row a of every
// earlier stream.
int launch_kv_quant_rows(int dh, int loop, int n_rows, int H, const int* bits, const float* k_new,
                         const float* v_new, const flashloop_kv& k, const flashloop_kv& v, int32_t* err,
                         cudaStream_t stream) {
  const long long items = (long long)n_rows * H * 2;
  const int grid = (int)((items + (kQuantThreads / 32) - 1) / (kQuantThreads / 32));
  const KVStreams Ks = kv_streams(k), Vs = kv_streams(v);
  LoopTables lt{};
  for (int i = 0; i < FLASHLOOP_MAX_LOOPS; ++i) {
    lt.slot[i] = nullptr;
    lt.bits[i] = bits[i];
  }
  uint8_t* kc = loop == 1 ? reinterpret_cast<uint8_t*>(k.base_codes) : k.res_codes[loop - 1];
  uint8_t* vc = loop == 1 ? reinterpret_cast<uint8_t*>(v.base_codes) : v.res_codes[loop - 1];
  uint16_t* ks = loop == 1 ? k.base_scales : k.res_scales[loop - 1];
  uint16_t* vs = loop == 1 ? v.base_scales : v.res_scales[loop - 1];
  if (dh == 128)
    kv_quant_kernel<128><<<grid, kQuantThreads, 0, stream>>>(k_new, v_new, nullptr, nullptr, n_rows, n_rows, H,
                                                              loop, Ks, Vs, lt, kc, ks, vc, vs, err);
  else
    kv_quant_kernel<64><<<grid, kQuantThreads, 0, stream>>>(k_new, v_new, nullptr, nullptr, n_rows, n_rows, H,
                                                             loop, Ks, Vs, lt, kc, ks, vc, vs, err);
  return launch_status();
}

// (a5) Rebuild Khat^(r-1), Khat^(r), Vhat^(r-1), Vhat^(r) of the selected
// columns (loop 1 / dense: Khat^(1), Vhat^(1) of every token) as fp16:
// K as [H, kcp, dh] rows scaled by `kscale` (log2(e)/sqrt(dh), so that q.k
// comes out in log2 units; one fp16 rounding either way), V transposed as
// [H, dh, kcp], so that both feed the attention MMAs as K-major tiles.  [FlashLoop App. G]: only the selected
// columns are rebuilt, never the full cache.  One block = 64 columns of one
// head; V rows are staged in shared memory and written transposed.
template <int DH>
__global__ void __launch_bounds__(kQuantThreads)
selcol_dequant_kernel(const int32_t* __restrict__ cols, int kc, int kcp, int S, int H, int loop,
                      float kscale, KVStreams Ks, KVStreams Vs, LoopTables lt, __half* k_old, __half* k_new,
                      __half* vt_old, __half* vt_new, int32_t* err) {
  constexpr int E = DH / 32;
  __shared__ __align__(16) __half sv[2][64][DH + 8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = blockIdx.y, j0 = blockIdx.x * 64;
  const bool has_old = loop > 1;
  for (int c = warp; c < 64; c += kQuantThreads / 32) {
    const int col = j0 + c;
    int j = -1;
    if (col < kc) {
      j = cols ? cols[(size_t)h * kc + col] : col;
      if (j < 0 || j >= S) {
        if (lane == 0) set_error(err, FLASHLOOP_DEVERR_INDEX);
        j = -1;
      }
    }
    for (int which = 0; which < 2; ++which) {
      const KVStreams& kv = which == 0 ? Ks : Vs;
      float acc[E], oldv[E];
      if (j >= 0) {
        reconstruct_lane<E, DH>(kv, lt, j, h, H, has_old ? loop - 1 : 1, lane, acc);
#pragma unroll
        for (int e = 0; e < E; ++e) oldv[e] = acc[e];
        if (has_old) {
          const int sl = lt.slot[loop - 1][j];
          if (sl >= 0) {
            const int b = lt.bits[loop - 1];
            const int g = (lane * E) / FLASHLOOP_GROUP;
            const uint8_t* row = kv.res_codes[loop - 1] + ((size_t)sl * H + h) * (DH * b / 8);
            const float sc = half_bits_to_float(kv.res_scales[loop - 1][((size_t)sl * H + h) * (DH / 32) + g]);
            int cc[E];
            unpack_codes<E>(row, lane * E, b, cc);
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] = acc[e] + static_cast<float>(cc[e]) * sc;
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = oldv[e] = 0.f;
      }
      {
        // the attention MMAs take fp16 operands: flag a value that does not fit
        const float sc = which == 0 ? kscale : 1.f;
        bool ok = true;
#pragma unroll
        for (int e = 0; e < E; ++e) ok = ok && half_range_ok(acc[e] * sc) && half_range_ok(oldv[e] * sc);
        if (!ok) set_error(err, FLASHLOOP_DEVERR_RANGE);
      }
      if (which == 0) {
        if (col < kcp) {
          const size_t off = ((size_t)h * kcp + col) * DH + lane * E;
#pragma unroll
          for (int e = 0; e < E; ++e) k_new[off + e] = __float2half_rn(acc[e] * kscale);
          if (has_old) {
#pragma unroll
            for (int e = 0; e < E; ++e) k_old[off + e] = __float2half_rn(oldv[e] * kscale);
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          sv[1][c][lane * E + e] = __float2half_rn(acc[e]);
          sv[0][c][lane * E + e] = __float2half_rn(oldv[e]);
        }
      }
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < 2 * DH * 32; idx += kQuantThreads) {
    const int which = idx / (DH * 32);
    if (which == 0 && !has_old) continue;
    const int rem = idx % (DH * 32);
    const int d = rem / 32, jp = (rem % 32) * 2;
    if (j0 + jp >= kcp) continue;
    __half* dst = (which == 0 ? vt_old : vt_new) + ((size_t)h * DH + d) * kcp + j0 + jp;
    *reinterpret_cast<__half2*>(dst) = __halves2half2(sv[which][jp][d], sv[which][jp + 1][d]);
  }
}

int launch_selcol_dequant(const flashloop_params* p, int loop, const int32_t* cols, int kc, int kcp,
                          flashloop_state* st, __half* k_old, __half* k_new, __half* vt_old,
                          __half* vt_new, cudaStream_t stream) {
  const int H = p->n_heads;
  dim3 grid((kcp + 63) / 64, H);
  const KVStreams Ks = kv_streams(st->k), Vs = kv_streams(st->v);
  const LoopTables lt = loop_tables(p, st);
  const float kscale = 1.4426950408889634f / sqrtf(static_cast<float>(p->head_dim));
  if (p->head_dim == 128) {
    selcol_dequant_kernel<128><<<grid, kQuantThreads, 0, stream>>>(
        cols, kc, kcp, p->seq, H, loop, kscale, Ks, Vs, lt, k_old, k_new, vt_old, vt_new, st->err_word);
  } else {
    selcol_dequant_kernel<64><<<grid, kQuantThreads, 0, stream>>>(
        cols, kc, kcp, p->seq, H, loop, kscale, Ks, Vs, lt, k_old, k_new, vt_old, vt_new, st->err_word);
  }
  return launch_status();
}

}  // namespace fl
