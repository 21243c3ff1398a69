// (a2)+(a3) Gathered Q/K/V projection with RoPE and fused residual
// quantisation, and (a7) the gathered output projection, on the sm_100a
// tensor cores (tcgen05.mma, accumulators in TMEM).
//
// [FlashLoop §4.1, App. G]: only the active rows are projected ("active-token
// execution", "fused projections"); [FlashLoop §4.3, §4.4]: the new K/V of
// the active tokens are quantised as residuals against the reconstructed
// previous loop in the same pass that produces them.
//
// Persistent, warp-specialised kernel: tile 128 rows x 256 columns, K step 64,
// 4-stage shared-memory ring, two TMEM accumulators (512 columns) so the
// epilogue of one tile overlaps the main loop of the next.
//   warps 0-1   gather the A rows (active tokens) with 16-byte cp.async into
//               the 128-byte-swizzled layout and arrive when their copies land
//               (a TMA tile::gather4 of four 128-byte rows per request was
//               measured 2.8x slower on this shape);
//   warp 2      allocates TMEM; lane 0 streams the weight tiles by TMA;
//   warp 3      lane 0 issues tcgen05.mma (M128 N256 K16, bf16 -> f32);
//   warps 4-11  epilogue, two warps per TMEM lane quarter (one per 128-column
//               half of the tile), one row per thread:
//               OUT  -> bf16 Y at the token's row;
//               QKV  -> RoPE (table computed in double) on q and k, bf16 q at
//                       the token's row, and either float32 k/v at the row's
//                       compact position or, fused, the loop's INT8 base /
//                       INT4 / INT2 residual codes and fp16 scales.
// Every wait is bounded; a wait that gives up records FLASHLOOP error 3 and
// the block unwinds, releasing its TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tc_util.cuh"

namespace fl {

constexpr int kTcBM = 128, kTcBN = 256, kTcBK = 64, kTcStages = 4, kTcThreads = 384;
constexpr int kTcEpiThreads = 256, kTcProdThreads = 64;
constexpr int kTcABytes = kTcBM * kTcBK * 2;  // 16 KiB
constexpr int kTcBBytes = kTcBN * kTcBK * 2;  // 32 KiB
constexpr int kTcSmem = 1024 + kTcStages * (kTcABytes + kTcBBytes) + 256;
constexpr uint32_t kTcIdesc = f16_idesc(kTcBM, kTcBN, 1);

enum TcMode { kTcQkvF32 = 0, kTcQkvQuant = 1, kTcOut = 2 };

struct TcGemmArgs {
  const uint16_t* A;      // [S, K] bf16, rows gathered through `rows`
  const int32_t* rows;    // active tokens (NULL: identity)
  const int32_t* n_rows;  // device count (NULL: S)
  int S, K, N, cap;
  int d_model, head_dim, loop;
  const float* rope_cs;   // [S, dh/2] (cos, sin)
  uint16_t* q_out;        // bf16 [S, d], row = token
  float* k_out;           // float32 [cap, d], row = compact position (mode QKV f32)
  float* v_out;
  uint16_t* y_out;        // bf16 [S, N], row = token (mode OUT)
  KVStreams Ks, Vs;       // caches read for the previous reconstruction (mode QKV quant)
  LoopTables lt;
  uint8_t* k_codes;       // this loop's stream: base (loop 1) or residual, row = compact position
  uint16_t* k_scales;
  uint8_t* v_codes;
  uint16_t* v_scales;
  int32_t* err;
};

__device__ __forceinline__ void rope_rot(float& x1, float& x2, float c, float s) {
  // explicit roundings: the same float32 result in every kernel that rotates
  const float y1 = __fsub_rn(__fmul_rn(x1, c), __fmul_rn(x2, s));
  const float y2 = __fadd_rn(__fmul_rn(x2, c), __fmul_rn(x1, s));
  x1 = y1;
  x2 = y2;
}

// acc += code * s for the 32 BITS-bit two's-complement codes of one group
// (packed words w); BITS is a template constant so that every field index is
// a constant and the words stay in registers.
template <int BITS>
__device__ __forceinline__ void add_codes(const uint32_t (&w)[8], float s, float (&acc)[32]) {
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    constexpr uint32_t kMask = (1u << BITS) - 1u;
    const int bit = e * BITS;
    int c = static_cast<int>((w[bit >> 5] >> (bit & 31)) & kMask);
    if (c >= (1 << (BITS - 1))) c -= (1 << BITS);
    acc[e] = acc[e] + static_cast<float>(c) * s;
  }
}

// Rebuild Xhat^(upto) of 32 consecutive elements (group g) of one (token, head).
template <int DH>
__device__ __forceinline__ void recon_group(const KVStreams& kv, const LoopTables& lt, int t, int h, int H,
                                            int g, int upto, float (&acc)[32]) {
  {
    const int8_t* src = kv.base_codes + ((size_t)t * H + h) * DH + g * 32;
    const float s = __half2float(__ushort_as_half(kv.base_scales[((size_t)t * H + h) * (DH / 32) + g]));
    const uint4 w0 = *reinterpret_cast<const uint4*>(src);
    const uint4 w1 = *reinterpret_cast<const uint4*>(src + 16);
    const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int c = static_cast<int8_t>((w[e >> 2] >> ((e & 3) * 8)) & 0xFF);
      acc[e] = static_cast<float>(c) * s;
    }
  }
  for (int l = 2; l <= upto; ++l) {
    const int sl = lt.slot[l - 1][t];
    if (sl < 0) continue;
    const int b = lt.bits[l - 1];
    const uint8_t* row = kv.res_codes[l - 1] + ((size_t)sl * H + h) * (DH * b / 8) + g * 4 * b;
    const float s = __half2float(__ushort_as_half(kv.res_scales[l - 1][((size_t)sl * H + h) * (DH / 32) + g]));
    uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (b == 8) {
      const uint4 a0 = *reinterpret_cast<const uint4*>(row);
      const uint4 a1 = *reinterpret_cast<const uint4*>(row + 16);
      w[0] = a0.x; w[1] = a0.y; w[2] = a0.z; w[3] = a0.w; w[4] = a1.x; w[5] = a1.y; w[6] = a1.z; w[7] = a1.w;
      add_codes<8>(w, s, acc);
    } else if (b == 4) {
      const uint4 a0 = *reinterpret_cast<const uint4*>(row);
      w[0] = a0.x; w[1] = a0.y; w[2] = a0.z; w[3] = a0.w;
      add_codes<4>(w, s, acc);
    } else {
      const uint2 a0 = *reinterpret_cast<const uint2*>(row);
      w[0] = a0.x; w[1] = a0.y;
      add_codes<2>(w, s, acc);
    }
  }
}

// Quantise 32 values and store their packed codes (32*BITS/8 bytes) and
// scale; BITS is a template constant so that the packed words stay in
// registers.
template <int BITS>
__device__ __forceinline__ void quant_store_group_b(const float (&x)[32], uint8_t* codes, uint16_t* scale) {
  constexpr int qmax = (1 << (BITS - 1)) - 1;
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(x[e]));
  __half hs = __float2half_rn(__fdiv_rn(amax, static_cast<float>(qmax)));
  uint16_t sbits = __half_as_ushort(hs);
  if ((sbits & 0x7FFFu) == 0x7C00u) sbits = (sbits & 0x8000u) | 0x7BFFu;
  const float s = __half2float(__ushort_as_half(sbits));
  const float rs = s > 0.f ? approx_rcp(s) : 0.f;
  uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const int c = s > 0.f ? static_cast<int>(quant_code(x[e], s, rs, qmax)) : 0;
    const int bit = e * BITS;
    w[bit >> 5] |= (static_cast<uint32_t>(c) & ((1u << BITS) - 1u)) << (bit & 31);
  }
  if (BITS == 8) {
    *reinterpret_cast<uint4*>(codes) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4*>(codes + 16) = make_uint4(w[4], w[5], w[6], w[7]);
  } else if (BITS == 4) {
    *reinterpret_cast<uint4*>(codes) = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    *reinterpret_cast<uint2*>(codes) = make_uint2(w[0], w[1]);
  }
  *scale = sbits;
}

__device__ __forceinline__ void quant_store_group(const float (&x)[32], int bits, uint8_t* codes,
                                                  uint16_t* scale) {
  if (bits == 8) quant_store_group_b<8>(x, codes, scale);
  else if (bits == 4) quant_store_group_b<4>(x, codes, scale);
  else quant_store_group_b<2>(x, codes, scale);
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];\n" ::"l"(p));
}

// The cache lines the fused quantiser will read for one row of a K or V tile
// (the previous loops' reconstruction of the heads in this thread's half:
// base codes and scales, then each earlier residual row present and its
// scales), requested into L2 while the thread waits for the tile's
// accumulator, so that the epilogue's loads need not go to DRAM.
template <int DH>
__device__ __forceinline__ void prefetch_recon_row(const TcGemmArgs& g, const KVStreams& kv, int t, int h0,
                                                   int heads) {
  const int H = g.d_model / DH;
  for (int k = 0; k < heads; ++k) {
    const size_t th = (size_t)t * H + h0 + k;
#pragma unroll
    for (int c = 0; c < DH; c += 128) prefetch_l2(kv.base_codes + th * DH + c);
  }
  prefetch_l2(kv.base_scales + ((size_t)t * H + h0) * (DH / 32));
  for (int l = 2; l < g.loop; ++l) {
    const int sl = g.lt.slot[l - 1][t];
    if (sl < 0) continue;
    const int rb = DH * g.lt.bits[l - 1] / 8;
    for (int k = 0; k < heads; ++k) prefetch_l2(kv.res_codes[l - 1] + ((size_t)sl * H + h0 + k) * rb);
    prefetch_l2(kv.res_scales[l - 1] + ((size_t)sl * H + h0) * (DH / 32));
  }
}

template <int DH>
__device__ __forceinline__ void epilogue_tile(const TcGemmArgs& g, int mode, int m0, int n0, int row,
                                              int n_rows, uint32_t tbase, int half) {
  const int a = m0 + row;
  int t = -1;
  if (a < n_rows) {
    t = g.rows ? g.rows[a] : a;
    if (t < 0 || t >= g.S) t = -1;
  }
  if (mode == kTcOut) {
#pragma unroll 1
    for (int c0 = half * 128; c0 < half * 128 + 128; c0 += 32) {
      uint32_t r[32];
      __syncwarp();
      tmem_ld32(tbase + c0, r);
      tmem_wait_ld();
      if (t >= 0) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = (uint32_t)float_to_bf16_bits(__uint_as_float(r[2 * e])) |
                  ((uint32_t)float_to_bf16_bits(__uint_as_float(r[2 * e + 1])) << 16);
        uint4* dst = reinterpret_cast<uint4*>(g.y_out + (size_t)t * g.N + n0 + c0);
#pragma unroll
        for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
      }
    }
    return;
  }
  const int d = g.d_model, H = d / DH;
  constexpr int kHalf = DH / 2;
  constexpr int kChunksPerHalf = kHalf / 32;
  const int section = n0 / d;  // 0 = q, 1 = k, 2 = v
  const int c_base = n0 - section * d;
#pragma unroll 1
  for (int hl = 0; hl < 128 / DH; ++hl) {
    const int hcol = half * 128 + hl * DH;  // first tile column of this head
    const int h = (c_base + hcol) / DH;
#pragma unroll 1
    for (int j = 0; j < kChunksPerHalf; ++j) {
      const int lo = hcol + j * 32, hi = lo + kHalf;
      uint32_t rl[32], rh[32];
      __syncwarp();
      tmem_ld32(tbase + lo, rl);
      tmem_ld32(tbase + hi, rh);
      tmem_wait_ld();
      if (t < 0) continue;
      float xl[32], xh[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        xl[e] = __uint_as_float(rl[e]);
        xh[e] = __uint_as_float(rh[e]);
      }
      if (section < 2) {
        const float4* cs = reinterpret_cast<const float4*>(g.rope_cs + ((size_t)t * kHalf + j * 32) * 2);
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) {
          const float4 v = cs[e2];
          rope_rot(xl[2 * e2], xh[2 * e2], v.x, v.y);
          rope_rot(xl[2 * e2 + 1], xh[2 * e2 + 1], v.z, v.w);
        }
      }
      const int col_lo = c_base + lo, col_hi = c_base + hi;
      if (section == 0) {
        if (g.q_out == nullptr) continue;  // a decode context stores only its K/V
        uint16_t* dst_l = g.q_out + (size_t)t * d + col_lo;
        uint16_t* dst_h = g.q_out + (size_t)t * d + col_hi;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint32_t pl[4], ph[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int e = v * 8 + 2 * u;
            pl[u] = (uint32_t)float_to_bf16_bits(xl[e]) | ((uint32_t)float_to_bf16_bits(xl[e + 1]) << 16);
            ph[u] = (uint32_t)float_to_bf16_bits(xh[e]) | ((uint32_t)float_to_bf16_bits(xh[e + 1]) << 16);
          }
          reinterpret_cast<uint4*>(dst_l)[v] = make_uint4(pl[0], pl[1], pl[2], pl[3]);
          reinterpret_cast<uint4*>(dst_h)[v] = make_uint4(ph[0], ph[1], ph[2], ph[3]);
        }
      } else if (mode == kTcQkvF32) {
        float* dst = (section == 1 ? g.k_out : g.v_out) + (size_t)a * d;
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          reinterpret_cast<float4*>(dst + col_lo)[v] = make_float4(xl[4 * v], xl[4 * v + 1], xl[4 * v + 2], xl[4 * v + 3]);
          reinterpret_cast<float4*>(dst + col_hi)[v] = make_float4(xh[4 * v], xh[4 * v + 1], xh[4 * v + 2], xh[4 * v + 3]);
        }
      } else {
        const KVStreams& kv = section == 1 ? g.Ks : g.Vs;
        uint8_t* codes = section == 1 ? g.k_codes : g.v_codes;
        uint16_t* scales = section == 1 ? g.k_scales : g.v_scales;
        const int bits = g.lt.bits[g.loop - 1];
        const int row_bytes = DH * bits / 8;
        const int g_lo = j, g_hi = j + kChunksPerHalf;
        if (g.loop >= 2) {
          float prev[32];
          recon_group<DH>(kv, g.lt, t, h, H, g_lo, g.loop - 1, prev);
#pragma unroll
          for (int e = 0; e < 32; ++e) xl[e] = xl[e] - prev[e];
          recon_group<DH>(kv, g.lt, t, h, H, g_hi, g.loop - 1, prev);
#pragma unroll
          for (int e = 0; e < 32; ++e) xh[e] = xh[e] - prev[e];
        }
        // the base is indexed by token, a residual by the token's slot in this loop's active list
        const int dst_row = g.loop == 1 ? t : g.lt.slot[g.loop - 1][t];
        uint8_t* crow = codes + ((size_t)dst_row * H + h) * row_bytes;
        uint16_t* srow = scales + ((size_t)dst_row * H + h) * (DH / 32);
        quant_store_group(xl, bits, crow + g_lo * 4 * bits, srow + g_lo);
        quant_store_group(xh, bits, crow + g_hi * 4 * bits, srow + g_hi);
      }
    }
  }
}

template <int DH>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmap_b, TcGemmArgs g, int mode) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kTcStages * kTcABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + kTcStages * kTcBBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kTcStages;
  uint64_t* acc_full = bars + 2 * kTcStages;
  uint64_t* acc_empty = bars + 2 * kTcStages + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kTcStages + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int n_rows = g.n_rows ? *g.n_rows : g.S;
  if (n_rows > g.cap) n_rows = g.cap;
  if (n_rows < 0) n_rows = 0;
  const int m_tiles = (n_rows + kTcBM - 1) / kTcBM;
  const int n_tiles = g.N / kTcBN;
  const int total = m_tiles * n_tiles;
  const int KT = g.K / kTcBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full[s], kTcProdThreads + 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kTcEpiThreads);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 2) {
    // ---- A producers: gather the active rows (16 rows x 8 chunks per pass)
    const int tid = threadIdx.x;
    const int chunk = tid & 7;
    int stage = 0;
    uint32_t phase = 0;
    for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
      const int m0 = (tile / n_tiles) * kTcBM;
      const uint16_t* src[16];
      int ok[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = (tid >> 3) + 8 * i;
        const int a = m0 + r;
        int t = -1;
        if (a < n_rows) {
          t = g.rows ? g.rows[a] : a;
          if (t < 0 || t >= g.S) {
            set_error(g.err, FLASHLOOP_DEVERR_INDEX);
            t = -1;
          }
        }
        ok[i] = t >= 0;
        src[i] = g.A + (size_t)(t >= 0 ? t : 0) * g.K + chunk * 8;
      }
      for (int kt = 0; kt < KT; ++kt) {
        if (!mbar_wait(&empty[stage], phase ^ 1)) {
          set_error(g.err, kDevErrTimeout);
          *abort_flag = 1;
          break;
        }
        uint8_t* dst = sA + stage * kTcABytes;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int r = (tid >> 3) + 8 * i;
          cp_async16(dst + sw128_offset(r, chunk), src[i] + kt * kTcBK, ok[i] ? 16 : 0);
        }
        cp_async_mbar_arrive_noinc(&full[stage]);
        if (++stage == kTcStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    cp_async_wait_all();
  } else if (warp == 2) {
    // ---- weight tiles by TMA
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued[kTcStages];
      for (int s2 = 0; s2 < kTcStages; ++s2) issued[s2] = -1;
      for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
        const int n0 = (tile % n_tiles) * kTcBN;
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) {
            set_error(g.err, kDevErrTimeout);
            *abort_flag = 1;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], kTcBBytes);
          tma_load_2d(sB + stage * kTcBBytes, &tmap_b, kt * kTcBK, n0, &full[stage]);
          issued[stage] = phase;
          if (++stage == kTcStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // never leave with a copy in flight: the full barrier of each stage's last
      // load completes once its bytes (and the A rows) have landed (bounded wait)
      for (int s2 = 0; s2 < kTcStages; ++s2)
        if (issued[s2] >= 0) (void)mbar_wait(&full[s2], (uint32_t)issued[s2]);
    }
  } else if (warp == 3) {
    // ---- MMA issue
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x, ++it) {
        const int buf = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&acc_empty[buf], acc_phase ^ 1)) {
          set_error(g.err, kDevErrTimeout);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * kTcBN;
        bool ok = true;
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(&full[stage], phase)) {
            set_error(g.err, kDevErrTimeout);
            *abort_flag = 1;
            ok = false;
            break;
          }
          fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * kTcABytes);
          const uint32_t b_addr = smem_u32(sB + stage * kTcBBytes);
#pragma unroll
          for (int k = 0; k < kTcBK / 16; ++k) {
            umma_f16(d_tmem, sw128_kmajor_desc(a_addr + k * 32), sw128_kmajor_desc(b_addr + k * 32), kTcIdesc,
                     (kt > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == kTcStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[buf]);
      }
    }
  } else {
    // ---- epilogue: warps 4-11, two per TMEM lane quarter, one row per thread
    const int lane_grp = warp & 3;
    const int half = (warp - 4) >> 2;
    const int row = lane_grp * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x, ++it) {
      const int buf = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (mode == kTcQkvQuant && g.loop >= 2) {
        // while the accumulator is computed: this row's earlier codes into L2
        const int n0p = (tile % n_tiles) * kTcBN, section = n0p / g.d_model;
        const int a = (tile / n_tiles) * kTcBM + row;
        if (section >= 1 && a < n_rows) {
          const int t = g.rows ? g.rows[a] : a;
          if (t >= 0 && t < g.S) {
            prefetch_recon_row<DH>(g, section == 1 ? g.Ks : g.Vs, t,
                                   (n0p - section * g.d_model + half * 128) / DH, 128 / DH);
            if (section == 1) {  // the row's RoPE table entries (keys are rotated)
              const float* cs = g.rope_cs + (size_t)t * DH;
#pragma unroll
              for (int c = 0; c < DH; c += 32) prefetch_l2(cs + c);
            }
          }
        }
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[buf], acc_phase))) {
        set_error(g.err, kDevErrTimeout);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int m0 = (tile / n_tiles) * kTcBM;
      const int n0 = (tile % n_tiles) * kTcBN;
      const uint32_t tbase = tmem_base + ((uint32_t)(lane_grp * 32) << 16) + buf * kTcBN;
      epilogue_tile<DH>(g, mode, m0, n0, row, n_rows, tbase, half);
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// The driver's cuTensorMapEncodeTiled, looked up once (a function-local
// static: its initialisation is thread-safe).
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return nullptr;
  }();
  return fn;
}

// Tensor map of a row-major bf16 matrix [rows, cols] read in 64 x box_rows tiles, 128-byte swizzle.
static int make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return FLASHLOOP_ERR_CUDA;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0 || (cols * 2) % 16 != 0) return FLASHLOOP_ERR_INVALID_ARG;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FLASHLOOP_OK : FLASHLOOP_ERR_CUDA;
}

static int sm_count() {
  static int cached[128];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

static int launch_tc(const flashloop_params* p, const TcGemmArgs& g, const uint16_t* w, int mode,
                     cudaStream_t stream) {
  if (g.K % kTcBK != 0 || g.N % kTcBN != 0) return FLASHLOOP_ERR_UNSUPPORTED;
  CUtensorMap tmap;
  int rc = make_tmap_bf16(&tmap, w, (uint64_t)g.N, (uint64_t)g.K, kTcBN);
  if (rc != FLASHLOOP_OK) return rc;
  const int max_tiles = ((g.cap + kTcBM - 1) / kTcBM) * (g.N / kTcBN);
  int grid = sm_count();
  if (grid > max_tiles) grid = max_tiles;
  if (grid < 1) grid = 1;
  if (p->head_dim == 128) {
    FL_TRY(cudaFuncSetAttribute(tc_gemm_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmem));
    tc_gemm_kernel<128><<<grid, kTcThreads, kTcSmem, stream>>>(tmap, g, mode);
  } else {
    FL_TRY(cudaFuncSetAttribute(tc_gemm_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmem));
    tc_gemm_kernel<64><<<grid, kTcThreads, kTcSmem, stream>>>(tmap, g, mode);
  }
  return launch_status();
}

int launch_qkv_gemm(const flashloop_params* p, const uint16_t* x, const int32_t* active,
                    const int32_t* n_active, int cap, const uint16_t* w_qkv, const float* rope_cs,
                    uint16_t* q_out, float* k_out, float* v_out, int32_t* err, cudaStream_t stream) {
  TcGemmArgs g{};
  g.A = x; g.rows = active; g.n_rows = n_active; g.S = p->seq; g.K = p->d_model; g.N = 3 * p->d_model;
  g.cap = cap; g.d_model = p->d_model; g.head_dim = p->head_dim; g.loop = 1; g.rope_cs = rope_cs;
  g.q_out = q_out; g.k_out = k_out; g.v_out = v_out; g.err = err;
  return launch_tc(p, g, w_qkv, kTcQkvF32, stream);
}

int launch_qkv_quant_gemm(const flashloop_params* p, int loop, const uint16_t* x, const int32_t* active,
                          const int32_t* n_active, int cap, const uint16_t* w_qkv, flashloop_state* st,
                          uint16_t* q_out, cudaStream_t stream) {
  TcGemmArgs g{};
  g.A = x; g.rows = active; g.n_rows = n_active; g.S = p->seq; g.K = p->d_model; g.N = 3 * p->d_model;
  g.cap = cap; g.d_model = p->d_model; g.head_dim = p->head_dim; g.loop = loop; g.rope_cs = st->rope_cs;
  g.q_out = q_out; g.err = st->err_word;
  g.Ks = kv_streams(st->k);
  g.Vs = kv_streams(st->v);
  g.lt = loop_tables(p, st);
  if (loop == 1) {
    g.k_codes = reinterpret_cast<uint8_t*>(st->k.base_codes); g.k_scales = st->k.base_scales;
    g.v_codes = reinterpret_cast<uint8_t*>(st->v.base_codes); g.v_scales = st->v.base_scales;
  } else {
    g.k_codes = st->k.res_codes[loop - 1]; g.k_scales = st->k.res_scales[loop - 1];
    g.v_codes = st->v.res_codes[loop - 1]; g.v_scales = st->v.res_scales[loop - 1];
  }
  return launch_tc(p, g, w_qkv, kTcQkvQuant, stream);
}

int launch_out_gemm(const flashloop_params* p, const uint16_t* o, const int32_t* active,
                    const int32_t* n_active, int cap, const uint16_t* w_o, uint16_t* y,
                    int32_t* err, cudaStream_t stream) {
  TcGemmArgs g{};
  g.A = o; g.rows = active; g.n_rows = n_active; g.S = p->seq; g.K = p->d_model; g.N = p->d_model;
  g.cap = cap; g.y_out = y; g.err = err;
  return launch_tc(p, g, w_o, kTcOut, stream);
}

}  // namespace fl
