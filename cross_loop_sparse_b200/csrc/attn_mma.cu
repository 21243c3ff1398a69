// Column-mass pass (warp-level tensor-core path, mma.sync m16n8k16, fp16
// operands, float32 accumulators): the loop-1 dense column sums of the
// softmax that rank the columns at loop 2, and the sums over active rows for
// the selected columns when a later loop shrinks its budget.
#include <math.h>

#include "common.cuh"
#include "mma_util.cuh"
#include "attn_args.cuh"

namespace fl {

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// Column mass c[j] = sum_{i >= j, i active} e^(s_ij - m_i) / Z_i over the
// given columns ([FlashLoop App. D.2]: the updated probabilities prepare the
// next selection).  One block owns 64 columns (4 warps x 16) of one head and
// walks the active rows from the first one whose token reaches its columns.
// ---------------------------------------------------------------------------
constexpr int kCmCols = 64, kCmRows = 64, kCmThreads = 128;



template <int DH>
__global__ void __launch_bounds__(kCmThreads)
colmass_kernel(ColmassArgs g) {
  constexpr int kLd = DH + 8;
  constexpr int KS = DH / 16;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __half* sK = reinterpret_cast<__half*>(smem_raw);       // [64][kLd]
  __half* sQ = sK + kCmCols * kLd;                         // [64][kLd]
  __shared__ int s_ctok[kCmCols];
  __shared__ int s_rtok[kCmRows];
  __shared__ float s_m[kCmRows], s_iz[kCmRows];
  __shared__ int s_first;

  const int h = blockIdx.y;
  const int c0 = blockIdx.x * kCmCols;
  if (c0 >= g.kc) return;
  int n_rows = g.n_rows ? *g.n_rows : g.S;
  if (n_rows > g.row_cap) n_rows = g.row_cap;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t* hcols = g.cols ? g.cols + (size_t)h * g.kc : nullptr;
  const int HD = g.H * DH;

  for (int c = tid; c < kCmCols; c += kCmThreads) {
    const int col = c0 + c;
    s_ctok[c] = col < g.kc ? (hcols ? hcols[col] : col) : 0x7fffffff;
  }
  for (int c = tid; c < kCmCols * (DH / 8); c += kCmThreads) {
    const int r = c / (DH / 8), q8 = (c % (DH / 8)) * 8;
    const int col = c0 + r;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (col < g.kc) v = *reinterpret_cast<const uint4*>(g.k_new + ((size_t)h * g.kcp + col) * DH + q8);
    *reinterpret_cast<uint4*>(sK + r * kLd + q8) = v;
  }
  __syncthreads();
  if (tid == 0) {
    // first active row whose token is >= the smallest column token
    const int tmin = s_ctok[0];
    int lo = 0, hi = n_rows;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      const int t = g.rows ? g.rows[mid] : mid;
      if (t < tmin) lo = mid + 1;
      else hi = mid;
    }
    s_first = lo;
  }
  uint32_t kf[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int row = warp * 16 + (lane & 15);
    const int col = ks * 16 + (lane >> 4) * 8;
    ldmatrix_x4(kf[ks], sK + row * kLd + col);
  }
  __syncthreads();
  const int cj0 = warp * 16 + (lane >> 2), cj1 = cj0 + 8;
  const int ct0 = s_ctok[cj0], ct1 = s_ctok[cj1];
  float sum0 = 0.f, sum1 = 0.f;
  for (int a0 = (s_first / kCmRows) * kCmRows; a0 < n_rows; a0 += kCmRows) {
    for (int i = tid; i < kCmRows; i += kCmThreads) {
      const int a = a0 + i;
      int t = -1;
      if (a < n_rows) {
        t = g.rows ? g.rows[a] : a;
        if (t < 0 || t >= g.S) t = -1;
      }
      s_rtok[i] = t;
      s_m[i] = t >= 0 ? g.m[(size_t)h * g.S + t] * kLog2e : 0.f;
      s_iz[i] = t >= 0 ? 1.f / g.z[(size_t)h * g.S + t] : 0.f;
    }
    __syncthreads();
    for (int c = tid; c < kCmRows * (DH / 8); c += kCmThreads) {
      const int r = c / (DH / 8), q8 = (c % (DH / 8)) * 8;
      const int t = s_rtok[r];
      uint4 v = make_uint4(0, 0, 0, 0);
      if (t >= 0) {
        const uint4 b = *reinterpret_cast<const uint4*>(g.q + (size_t)t * HD + (size_t)h * DH + q8);
        v = make_uint4(bf16x2_to_half2_bits(b.x), bf16x2_to_half2_bits(b.y),
                       bf16x2_to_half2_bits(b.z), bf16x2_to_half2_bits(b.w));
      }
      *reinterpret_cast<uint4*>(sQ + r * kLd + q8) = v;
    }
    __syncthreads();
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t r[4];
        const int row = np * 16 + (lane & 7) + (lane >> 4) * 8;
        const int col = ks * 16 + ((lane >> 3) & 1) * 8;
        ldmatrix_x4(r, sQ + row * kLd + col);
        mma_f16(s[2 * np], kf[ks], r[0], r[1]);
        mma_f16(s[2 * np + 1], kf[ks], r[2], r[3]);
      }
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int ri = nt * 8 + (lane & 3) * 2 + (e & 1);
        const int rt = s_rtok[ri];
        const int ct = (e >> 1) ? ct1 : ct0;
        if (rt >= 0 && ct <= rt) {
          const float pv = ex2(s[nt][e] * g.scale_log2 - s_m[ri]) * s_iz[ri];
          if (e >> 1) sum1 += pv; else sum0 += pv;
        }
      }
    __syncthreads();
  }
  sum0 += __shfl_xor_sync(0xffffffffu, sum0, 1);
  sum0 += __shfl_xor_sync(0xffffffffu, sum0, 2);
  sum1 += __shfl_xor_sync(0xffffffffu, sum1, 1);
  sum1 += __shfl_xor_sync(0xffffffffu, sum1, 2);
  if ((lane & 3) == 0) {
    if (c0 + cj0 < g.kc && ct0 >= 0 && ct0 < g.S) g.out[(size_t)h * g.S + ct0] = sum0;
    if (c0 + cj1 < g.kc && ct1 >= 0 && ct1 < g.S) g.out[(size_t)h * g.S + ct1] = sum1;
  }
}

int launch_colmass(const flashloop_params* p, const ColmassArgs& c, cudaStream_t stream) {
  dim3 grid((c.kc + kCmCols - 1) / kCmCols, p->n_heads);
  const int smem = 2 * kCmCols * (p->head_dim + 8) * 2;
  if (p->head_dim == 128) {
    FL_TRY(cudaFuncSetAttribute(colmass_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    colmass_kernel<128><<<grid, kCmThreads, smem, stream>>>(c);
  } else {
    FL_TRY(cudaFuncSetAttribute(colmass_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    colmass_kernel<64><<<grid, kCmThreads, smem, stream>>>(c);
  }
  return launch_status();
}

}  // namespace fl
