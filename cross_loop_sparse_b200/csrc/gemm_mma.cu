// (a2) Gathered Q/K/V projection with RoPE and (a7) gathered output
// projection -- warp-level tensor-core path (mma.sync m16n8k16, bf16 in,
// float32 accumulate).
//
// [FlashLoop §4.1, App. G]: only the active rows are projected ("active-token
// execution", "fused projections").  A rows are gathered through the active
// list by 16-byte cp.async into a 3-stage shared-memory ring; B = W is [N, K]
// row-major.  The epilogue stages the float32 tile in shared memory, then
//   QKV: applies rotate-half RoPE (table in float32, computed in double) to
//        q and k, stores q as bf16 at the token's row and k, v as float32
//        at the row's compact position;
//   OUT: stores bf16 Y at the token's row.
#include "common.cuh"
#include "mma_util.cuh"

namespace fl {

constexpr int kBM = 128, kBN = 128, kBK = 32, kStages = 3, kGemmThreads = 256;
constexpr int kLdA = kBK + 8;       // padded row (halves): conflict-free ldmatrix
constexpr int kLdC = kBN + 4;       // padded epilogue row (floats)
constexpr int kGemmSmem =
    (kStages * (kBM + kBN) * kLdA * 2) > (kBM * kLdC * 4) ? (kStages * (kBM + kBN) * kLdA * 2)
                                                           : (kBM * kLdC * 4);

enum GemmMode { kModeQKV = 0, kModeOut = 1 };

struct GemmArgs {
  const uint16_t* A;       // [S, K] bf16 (rows gathered)
  const int32_t* rows;     // active tokens (NULL: identity)
  const int32_t* n_rows;   // device count (NULL: S)
  int S, K, N, cap;
  const uint16_t* B;       // [N, K] bf16
  // QKV epilogue
  int d_model, head_dim;
  const float* rope_cs;    // [S, dh/2] float2
  uint16_t* q_out;         // [S, d] bf16, row = token
  float* k_out;            // [cap, d] float32, row = compact position
  float* v_out;
  // OUT epilogue
  uint16_t* y_out;         // [S, N] bf16, row = token
  int32_t* err;
};

template <int MODE>
__global__ void __launch_bounds__(kGemmThreads)
gemm_gathered_kernel(GemmArgs g) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ int s_tok[kBM];
  uint16_t* sA = reinterpret_cast<uint16_t*>(smem_raw);
  uint16_t* sB = sA + kStages * kBM * kLdA;

  int n_rows = g.n_rows ? *g.n_rows : g.S;
  if (n_rows > g.cap) n_rows = g.cap;
  const int m0 = blockIdx.x * kBM;
  const int n0 = blockIdx.y * kBN;
  if (m0 >= n_rows) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wm = warp >> 2, wn = warp & 3;  // 2 x 4 warps, warp tile 64 x 32

  for (int i = tid; i < kBM; i += kGemmThreads) {
    const int a = m0 + i;
    int t = -1;
    if (a < n_rows) {
      t = g.rows ? g.rows[a] : a;
      if (t < 0 || t >= g.S) {
        set_error(g.err, FLASHLOOP_DEVERR_INDEX);
        t = -1;
      }
    }
    s_tok[i] = t;
  }
  __syncthreads();

  auto load_stage = [&](int stage, int k0) {
    uint16_t* a_dst = sA + stage * kBM * kLdA;
    uint16_t* b_dst = sB + stage * kBN * kLdA;
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int c = tid + it * kGemmThreads;  // 512 chunks of 16 B per operand
      const int r = c >> 2, q = c & 3;
      const int t = s_tok[r];
      const uint16_t* src = g.A + (size_t)(t < 0 ? 0 : t) * g.K + k0 + q * 8;
      cp_async16(a_dst + r * kLdA + q * 8, src, t < 0 ? 0 : 16);
      const int nrow = n0 + r;
      const uint16_t* bsrc = g.B + (size_t)(nrow < g.N ? nrow : 0) * g.K + k0 + q * 8;
      cp_async16(b_dst + r * kLdA + q * 8, bsrc, nrow < g.N ? 16 : 0);
    }
  };

  float acc[4][4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

  const int ktiles = g.K / kBK;
#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < ktiles) load_stage(s, s * kBK);
    cp_async_commit();
  }
  for (int kt = 0; kt < ktiles; ++kt) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    const int nk = kt + kStages - 1;
    if (nk < ktiles) load_stage(nk % kStages, nk * kBK);
    cp_async_commit();
    const uint16_t* a_s = sA + (kt % kStages) * kBM * kLdA;
    const uint16_t* b_s = sB + (kt % kStages) * kBN * kLdA;
#pragma unroll
    for (int ks = 0; ks < kBK / 16; ++ks) {
      uint32_t af[4][4];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        const int row = wm * 64 + mt * 16 + (lane & 15);
        const int col = ks * 16 + (lane >> 4) * 8;
        ldmatrix_x4(af[mt], a_s + row * kLdA + col);
      }
      uint32_t bf[4][2];
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        uint32_t r[4];
        const int row = wn * 32 + np * 16 + (lane & 7) + (lane >> 4) * 8;
        const int col = ks * 16 + ((lane >> 3) & 1) * 8;
        ldmatrix_x4(r, b_s + row * kLdA + col);
        bf[np * 2][0] = r[0];
        bf[np * 2][1] = r[1];
        bf[np * 2 + 1][0] = r[2];
        bf[np * 2 + 1][1] = r[3];
      }
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) mma_bf16(acc[mt][nt], af[mt], bf[nt][0], bf[nt][1]);
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // Stage the float32 tile.
  float* sC = reinterpret_cast<float*>(smem_raw);
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int r = wm * 64 + mt * 16 + (lane >> 2);
      const int c = wn * 32 + nt * 8 + (lane & 3) * 2;
      sC[r * kLdC + c] = acc[mt][nt][0];
      sC[r * kLdC + c + 1] = acc[mt][nt][1];
      sC[(r + 8) * kLdC + c] = acc[mt][nt][2];
      sC[(r + 8) * kLdC + c + 1] = acc[mt][nt][3];
    }
  __syncthreads();

  if constexpr (MODE == kModeOut) {
    for (int i = tid; i < kBM * (kBN / 2); i += kGemmThreads) {
      const int r = i / (kBN / 2), c = (i % (kBN / 2)) * 2;
      const int t = s_tok[r];
      if (t < 0 || n0 + c >= g.N) continue;
      const uint32_t lo = float_to_bf16_bits(sC[r * kLdC + c]);
      const uint32_t hi = float_to_bf16_bits(sC[r * kLdC + c + 1]);
      *reinterpret_cast<uint32_t*>(g.y_out + (size_t)t * g.N + n0 + c) = lo | (hi << 16);
    }
  } else {
    const int d = g.d_model, dh = g.head_dim, half = dh / 2;
    const int section = n0 / d;  // 0 = q, 1 = k, 2 = v
    const int c_base = n0 - section * d;
    // One item = one (row, rotation pair) of the tile.
    for (int i = tid; i < kBM * (kBN / 2); i += kGemmThreads) {
      const int r = i / (kBN / 2), pidx = i % (kBN / 2);
      const int t = s_tok[r];
      if (t < 0) continue;
      const int hl = pidx / half, e = pidx % half;    // head within the tile, pair index
      const int c1 = hl * dh + e, c2 = c1 + half;      // tile columns of the pair
      float x1 = sC[r * kLdC + c1], x2 = sC[r * kLdC + c2];
      if (section < 2) {
        const float2 cs = reinterpret_cast<const float2*>(g.rope_cs)[(size_t)t * half + e];
        const float y1 = x1 * cs.x - x2 * cs.y;
        const float y2 = x2 * cs.x + x1 * cs.y;
        x1 = y1;
        x2 = y2;
      }
      const int col1 = c_base + c1, col2 = c_base + c2;
      if (section == 0) {
        g.q_out[(size_t)t * d + col1] = float_to_bf16_bits(x1);
        g.q_out[(size_t)t * d + col2] = float_to_bf16_bits(x2);
      } else {
        float* dst = (section == 1 ? g.k_out : g.v_out) + (size_t)(m0 + r) * d;
        dst[col1] = x1;
        dst[col2] = x2;
      }
    }
  }
}

static int set_gemm_smem() {
  FL_TRY(cudaFuncSetAttribute(gemm_gathered_kernel<kModeQKV>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem));
  FL_TRY(cudaFuncSetAttribute(gemm_gathered_kernel<kModeOut>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem));
  return FLASHLOOP_OK;
}

int launch_qkv_gemm(const flashloop_params* p, const uint16_t* x, const int32_t* active,
                    const int32_t* n_active, int cap, const uint16_t* w_qkv, const float* rope_cs,
                    uint16_t* q_out, float* k_out, float* v_out, int32_t* err, cudaStream_t stream) {
  int rc = set_gemm_smem();
  if (rc != FLASHLOOP_OK) return rc;
  GemmArgs g{};
  g.A = x; g.rows = active; g.n_rows = n_active; g.S = p->seq; g.K = p->d_model;
  g.N = 3 * p->d_model; g.cap = cap; g.B = w_qkv; g.d_model = p->d_model; g.head_dim = p->head_dim;
  g.rope_cs = rope_cs; g.q_out = q_out; g.k_out = k_out; g.v_out = v_out; g.err = err;
  dim3 grid((cap + kBM - 1) / kBM, g.N / kBN);
  gemm_gathered_kernel<kModeQKV><<<grid, kGemmThreads, kGemmSmem, stream>>>(g);
  return launch_status();
}

int launch_out_gemm(const flashloop_params* p, const uint16_t* o, const int32_t* active,
                    const int32_t* n_active, int cap, const uint16_t* w_o, uint16_t* y,
                    int32_t* err, cudaStream_t stream) {
  int rc = set_gemm_smem();
  if (rc != FLASHLOOP_OK) return rc;
  GemmArgs g{};
  g.A = o; g.rows = active; g.n_rows = n_active; g.S = p->seq; g.K = p->d_model;
  g.N = p->d_model; g.cap = cap; g.B = w_o; g.y_out = y; g.err = err;
  dim3 grid((cap + kBM - 1) / kBM, g.N / kBN);
  gemm_gathered_kernel<kModeOut><<<grid, kGemmThreads, kGemmSmem, stream>>>(g);
  return launch_status();
}

}  // namespace fl
