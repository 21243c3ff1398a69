// Shared device helpers of the FlashLoop sm_100a library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "flashloop.h"

namespace fl {

#define FL_TRY(expr)                                        \
  do {                                                      \
    cudaError_t fl_err_ = (expr);                           \
    if (fl_err_ != cudaSuccess) return FLASHLOOP_ERR_CUDA; \
  } while (0)

// Launch-error check after a kernel launch.
inline int launch_status() {
  return cudaGetLastError() == cudaSuccess ? FLASHLOOP_OK : FLASHLOOP_ERR_CUDA;
}

// Query-slot of loop r: loop 1 owns slot 0, loops >= 2 alternate 1, 2.
inline int slot_of_loop(int r) { return r == 1 ? 0 : 1 + (r % 2); }

// Record the first device-side error code; never traps.
__device__ __forceinline__ void set_error(int32_t* err, int code) {
  if (err != nullptr) atomicCAS(err, 0, code);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Two bf16 packed in a 32-bit word -> two floats (low half first).
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Largest finite fp16: the range of every tensor-core operand of the library.
constexpr float kHalfMax = 65504.f;

// |x| <= 65504 (false for NaN): x converts to fp16 without overflow.
__device__ __forceinline__ bool half_range_ok(float x) { return fabsf(x) <= kHalfMax; }

// bf16 pair -> fp16 pair (exact for |x| in fp16's normal range).
__device__ __forceinline__ uint32_t bf16x2_to_half2_bits(uint32_t w) {
  float2 f = bf16x2_to_float2(w);
  __half2 h = __floats2half2_rn(f.x, f.y);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------------------------------
// Workspace layout (host).  Offsets are 256-byte aligned.
// ---------------------------------------------------------------------------
struct Workspace {
  size_t ticket;    // uint32 counter of the last-block compaction (gate)
  size_t flags;     // uint8 [S] per-candidate gate decisions
  size_t keys;      // float [S] per-candidate change ratios (top-k retention)
  size_t cm_q;      // column-mass scratch: fp16 q of the rows [H, S, dh] (room for float [S, H, dh])
  size_t cm_rows;   // column-mass scratch: row max (log2), 1/Z [H, S] each, row tokens [S]
  size_t cols_kv;   // fp16 dequantised selected columns: 4 x [H, kmax, dh] or 2 x [H, S, dh]
  size_t row_cnt;   // int32 [H, S]: per head and active row, the selected columns at or before its token
  size_t kv_f32;    // float32 K and V of the loop's active rows, 2 x [S, H, dh] (kv_scheme 1 only)
  size_t total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline int pad8(int x) { return (x + 7) & ~7; }

inline int max_topk(const flashloop_params* p) {
  int k = 0;
  for (int r = 2; r <= p->n_loops; ++r) k = p->topk[r - 1] > k ? p->topk[r - 1] : k;
  return k;
}

inline Workspace workspace_layout(const flashloop_params* p) {
  Workspace w{};
  const size_t S = (size_t)p->seq, H = (size_t)p->n_heads, dh = (size_t)p->head_dim;
  size_t off = 0;
  w.ticket = off; off = align256(off + 16);
  w.flags = off; off = align256(off + S);
  w.keys = off; off = align256(off + S * sizeof(float));
  const size_t S128 = (S + 127) / 128 * 128;  // the column mass pads its rows to whole 128-row tiles
  const size_t cmq = S * H * dh * sizeof(float) > S128 * H * dh * 2 ? S * H * dh * sizeof(float) : S128 * H * dh * 2;
  const size_t cmr = S * H * dh * sizeof(float) > S128 * (8 * H + 4) ? S * H * dh * sizeof(float) : S128 * (8 * H + 4);
  w.cm_q = off; off = align256(off + cmq);
  w.cm_rows = off; off = align256(off + cmr);
  size_t sel = 4 * H * (size_t)pad8(max_topk(p)) * dh;
  size_t dense = 2 * H * (size_t)pad8(p->seq) * dh;
  w.cols_kv = off; off = align256(off + (sel > dense ? sel : dense) * sizeof(__half));
  w.row_cnt = off; off = align256(off + H * S * sizeof(int32_t));
  w.kv_f32 = off; off = align256(off + (p->kv_scheme == 1 ? 2 * S * H * dh * sizeof(float) : 0));
  w.total = off;
  return w;
}

// Decode scratch layout (offsets into flashloop_decode_state::workspace) and
// the split of the dense loop-1 pass (nsplit column ranges of `range`
// columns per sequence) and of the sparse loops (nblk ranges per head).
struct DecodeLayout {
  size_t k_new, v_new, scores, part_m, part_mu, part_Z, part_N, kv_part, total;
  int nsplit, range, nblk;
};

template <typename T>
inline T* ws_ptr(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(base) + off);
}

// ---------------------------------------------------------------------------
// Block-wide exclusive scan of one int per thread (blockDim.x <= 1024).
// `warp_sums` must hold 32 ints of shared memory.  Returns the exclusive
// prefix; *total receives the block total (valid in every thread).
// ---------------------------------------------------------------------------
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = (blockDim.x + 31) >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nwarps ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;  // inclusive prefix of warp totals
  }
  __syncthreads();
  int warp_prefix = warp > 0 ? warp_sums[warp - 1] : 0;
  *total = warp_sums[nwarps - 1];
  __syncthreads();
  return warp_prefix + x - v;
}

// Aggregate of the per-loop pointers a quantisation or reconstruction kernel
// reads (passed by value as a kernel parameter).
struct KVStreams {
  const int8_t* base_codes;
  const uint16_t* base_scales;
  const uint8_t* res_codes[FLASHLOOP_MAX_LOOPS];
  const uint16_t* res_scales[FLASHLOOP_MAX_LOOPS];
};

struct LoopTables {
  const int32_t* slot[FLASHLOOP_MAX_LOOPS];
  int bits[FLASHLOOP_MAX_LOOPS];
};

inline KVStreams kv_streams(const flashloop_kv& kv) {
  KVStreams s{};
  s.base_codes = kv.base_codes;
  s.base_scales = kv.base_scales;
  for (int i = 0; i < FLASHLOOP_MAX_LOOPS; ++i) {
    s.res_codes[i] = kv.res_codes[i];
    s.res_scales[i] = kv.res_scales[i];
  }
  return s;
}

inline LoopTables loop_tables(const flashloop_params* p, const flashloop_state* st) {
  LoopTables t{};
  for (int i = 0; i < FLASHLOOP_MAX_LOOPS; ++i) {
    t.slot[i] = st->slot[i];
    t.bits[i] = p->bits[i];
  }
  return t;
}

// Read E consecutive b-bit two's-complement codes of one packed row starting
// at element e0 (E * b <= 32; the fields never straddle a 32-bit word here
// because e0 * b is a multiple of E * b).
template <int E>
__device__ __forceinline__ void unpack_codes(const uint8_t* row, int e0, int bits, int (&c)[E]) {
  const int bit0 = e0 * bits;
  uint32_t word;
  const int nbytes = (E * bits) >> 3;
  const uint8_t* src = row + (bit0 >> 3);
  if (nbytes >= 4) {
    word = *reinterpret_cast<const uint32_t*>(src);
  } else if (nbytes == 2) {
    word = *reinterpret_cast<const uint16_t*>(src);
  } else {
    word = *src;
  }
  const int shift0 = (E * bits >= 8) ? 0 : (bit0 & 7);
  const uint32_t mask = (1u << bits) - 1u;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    uint32_t f = (word >> (shift0 + e * bits)) & mask;
    int v = static_cast<int>(f);
    if (v >= (1 << (bits - 1))) v -= (1 << bits);
    c[e] = v;
  }
}

// Quantiser code of x with stored scale s > 0: clamp(rint(fl(x / s)), -qmax, qmax)
// where fl is the IEEE round-to-nearest float32 quotient.  The quotient is
// taken from an approximate reciprocal (a few ulps off, i.e. < 2^-16 for
// |x/s| <= 128); only when it falls within 2^-12 of a half-integer, where the
// two could round differently, is the exact IEEE quotient computed.  The
// result is therefore identical to the definition for every input.
__device__ __forceinline__ float quant_code(float x, float s, float rs, int qmax) {
  const float q = x * rs;
  float c = rintf(q);
  if (fabsf(q - c) > 0.5f - 2.44140625e-4f) c = rintf(__fdiv_rn(x, s));
  return fminf(fmaxf(c, static_cast<float>(-qmax)), static_cast<float>(qmax));
}

__device__ __forceinline__ float approx_rcp(float s) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;\n" : "=f"(r) : "f"(s));
  return r;
}

}  // namespace fl
