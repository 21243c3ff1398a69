// (a6) Sparse attention update and the loop-1 dense attention, plus the
// column-mass pass -- warp-level tensor-core path (mma.sync m16n8k16, fp16
// operands, float32 accumulators).
//
// [FlashLoop §3.2, §4.2, App. D.2]: for the active rows of loop r and the
// selected key columns j <= i, the loop r-1 contribution of (i, j) is
// removed and the loop-r one added to the running (m, N, Z) of the row:
//   S_old = Q^(r-1) Khat^(r-1)^T, S_new = Q^(r) Khat^(r)^T (scaled by 1/sqrt(dh)),
//   m' = max(m, max S_new), Z' = a Z - sum e^(S_old - m') + sum e^(S_new - m'),
//   N' = a N + [e^(S_new - m') | -e^(S_old - m')] [Vhat^(r); Vhat^(r-1)].
// The running maximum is updated tile by tile (rescaling N and Z when it
// grows), which gives the same m', Z', N' as the closed form.  One block
// holds 128 active rows (8 warps x 16 rows) of one head and walks the
// ascending selected columns in tiles of 64 up to its largest row token;
// K/V tiles come from the compact fp16 buffers the selected-column pass
// wrote.  Loop 1 runs the same kernel over every column with no removal.
#include <math.h>

#include "common.cuh"
#include "mma_util.cuh"
#include "attn_args.cuh"

namespace fl {

constexpr int kAttnRows = 128, kAttnCols = 64, kAttnThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;

template <int DH>
struct AttnSmem {
  static constexpr int kLd = DH + 8;  // padded fp16 row
  static constexpr int kQ = kAttnRows * kLd;
  static constexpr int kT = kAttnCols * kLd;
  // q_new, q_old, then 2 stages x {k_new, v_new, k_old, v_old}
  static constexpr int kHalves = 2 * kQ + 2 * 4 * kT;
  static constexpr int kBytes = kHalves * 2;
};



// Number of ascending columns <= tok (binary search).
__device__ __forceinline__ int count_le(const int32_t* cols, int n, int tok) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (cols[mid] <= tok) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

template <int DH>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_update_kernel(AttnArgs g) {
  using L = AttnSmem<DH>;
  constexpr int kLd = L::kLd;
  constexpr int KS = DH / 16;   // k-steps over head_dim
  constexpr int NT = DH / 8;    // n-tiles over head_dim
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __half* sQn = reinterpret_cast<__half*>(smem_raw);
  __half* sQo = sQn + L::kQ;
  __half* sKV = sQo + L::kQ;
  __shared__ int s_rtok[kAttnRows];
  __shared__ int s_ctok[2][kAttnCols];
  __shared__ int s_ncols;

  const int h = blockIdx.y;
  int n_rows = g.n_rows ? *g.n_rows : g.S;
  if (n_rows > g.row_cap) n_rows = g.row_cap;
  const int r0 = blockIdx.x * kAttnRows;
  if (r0 >= n_rows) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool has_old = !g.dense;
  const int32_t* hcols = g.cols ? g.cols + (size_t)h * g.kc : nullptr;
  const int HD = g.H * DH;

  for (int i = tid; i < kAttnRows; i += kAttnThreads) {
    const int a = r0 + i;
    int t = -1;
    if (a < n_rows) {
      t = g.rows ? g.rows[a] : a;
      if (t < 0 || t >= g.S) {
        set_error(g.err, FLASHLOOP_DEVERR_INDEX);
        t = -1;
      }
    }
    s_rtok[i] = t;
  }
  __syncthreads();
  if (tid == 0) {
    int maxtok = -1;
    for (int i = kAttnRows - 1; i >= 0; --i)
      if (s_rtok[i] >= 0) { maxtok = s_rtok[i]; break; }
    s_ncols = hcols ? count_le(hcols, g.kc, maxtok) : (maxtok + 1 < g.kc ? maxtok + 1 : g.kc);
  }
  // Gather q rows (bf16 -> fp16) into shared memory.
  for (int c = tid; c < kAttnRows * (DH / 8); c += kAttnThreads) {
    const int r = c / (DH / 8), q8 = (c % (DH / 8)) * 8;
    const int t = s_rtok[r];
    uint4 vn = make_uint4(0, 0, 0, 0), vo = make_uint4(0, 0, 0, 0);
    if (t >= 0) {
      const size_t off = (size_t)t * HD + (size_t)h * DH + q8;
      const uint4 bn = *reinterpret_cast<const uint4*>(g.q_new + off);
      vn = make_uint4(bf16x2_to_half2_bits(bn.x), bf16x2_to_half2_bits(bn.y),
                      bf16x2_to_half2_bits(bn.z), bf16x2_to_half2_bits(bn.w));
      if (has_old) {
        const uint4 bo = *reinterpret_cast<const uint4*>(g.q_old + off);
        vo = make_uint4(bf16x2_to_half2_bits(bo.x), bf16x2_to_half2_bits(bo.y),
                        bf16x2_to_half2_bits(bo.z), bf16x2_to_half2_bits(bo.w));
      }
    }
    *reinterpret_cast<uint4*>(sQn + r * kLd + q8) = vn;
    *reinterpret_cast<uint4*>(sQo + r * kLd + q8) = vo;
  }
  __syncthreads();
  const int ncols = s_ncols;
  const int ntiles = (ncols + kAttnCols - 1) / kAttnCols;

  auto load_tile = [&](int stage, int tile) {
    const int c0 = tile * kAttnCols;
    __half* base = sKV + stage * 4 * L::kT;
    const __half* srcs[4] = {g.k_new, g.v_new, g.k_old, g.v_old};
    const int nsrc = has_old ? 4 : 2;
    for (int c = tid; c < nsrc * kAttnCols * (DH / 8); c += kAttnThreads) {
      const int which = c / (kAttnCols * (DH / 8));
      const int rem = c % (kAttnCols * (DH / 8));
      const int r = rem / (DH / 8), q8 = (rem % (DH / 8)) * 8;
      const int col = c0 + r;
      const bool ok = col < ncols;
      const __half* src = srcs[which] + ((size_t)h * g.kc + (ok ? col : 0)) * DH + q8;
      cp_async16(base + which * L::kT + r * kLd + q8, src, ok ? 16 : 0);
    }
    for (int c = tid; c < kAttnCols; c += kAttnThreads) {
      const int col = c0 + c;
      s_ctok[stage][c] = col < ncols ? (hcols ? hcols[col] : col) : 0x7fffffff;
    }
  };

  // Per-warp q fragments (16 rows x DH).
  uint32_t qn[KS][4], qo[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int row = warp * 16 + (lane & 15);
    const int col = ks * 16 + (lane >> 4) * 8;
    ldmatrix_x4(qn[ks], sQn + row * kLd + col);
    if (has_old) ldmatrix_x4(qo[ks], sQo + row * kLd + col);
  }

  // Row state of this lane: rows lr0 = lane/4 and lr1 = lane/4 + 8 of the warp.
  const int lr0 = warp * 16 + (lane >> 2), lr1 = lr0 + 8;
  const int tok0 = s_rtok[lr0], tok1 = s_rtok[lr1];
  float m_run[2], z_run[2];
  float acc[NT][4];
  if (g.dense) {
    m_run[0] = m_run[1] = -INFINITY;
    z_run[0] = z_run[1] = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  } else {
    const int toks[2] = {tok0, tok1};
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int t = toks[rr];
      if (t >= 0) {
        m_run[rr] = g.m_in[(size_t)h * g.S + t] * kLog2e;
        z_run[rr] = (lane & 3) == 0 ? g.z_in[(size_t)h * g.S + t] : 0.f;
      } else {
        m_run[rr] = -INFINITY;
        z_run[rr] = 0.f;
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int c = nt * 8 + (lane & 3) * 2;
      float2 a = make_float2(0.f, 0.f), b = make_float2(0.f, 0.f);
      if (tok0 >= 0) a = *reinterpret_cast<const float2*>(g.n_in + ((size_t)h * g.S + tok0) * DH + c);
      if (tok1 >= 0) b = *reinterpret_cast<const float2*>(g.n_in + ((size_t)h * g.S + tok1) * DH + c);
      acc[nt][0] = a.x; acc[nt][1] = a.y; acc[nt][2] = b.x; acc[nt][3] = b.y;
    }
  }
  // Largest and smallest row tokens of this warp (warp-uniform skip tests).
  int wmax = max(tok0, tok1), wmin = (tok0 < 0 ? 0x7fffffff : tok0);
  if (tok1 >= 0) wmin = min(wmin, tok1);
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    wmax = max(wmax, __shfl_xor_sync(0xffffffffu, wmax, o));
    wmin = min(wmin, __shfl_xor_sync(0xffffffffu, wmin, o));
  }

  if (ntiles > 0) load_tile(0, 0);
  cp_async_commit();
  for (int tile = 0; tile < ntiles; ++tile) {
    const int stage = tile & 1;
    if (tile + 1 < ntiles) load_tile(stage ^ 1, tile + 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const __half* sKn = sKV + stage * 4 * L::kT;
    const __half* sVn = sKn + L::kT;
    const __half* sKo = sVn + L::kT;
    const __half* sVo = sKo + L::kT;
    const int* ctok = s_ctok[stage];
    const int first_tok = ctok[0];
    if (wmax >= 0 && first_tok <= wmax) {
      float sn[8][4], so[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) { sn[nt][e] = 0.f; so[nt][e] = 0.f; }
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t r[4];
          const int row = np * 16 + (lane & 7) + (lane >> 4) * 8;
          const int col = ks * 16 + ((lane >> 3) & 1) * 8;
          ldmatrix_x4(r, sKn + row * kLd + col);
          mma_f16(sn[2 * np], qn[ks], r[0], r[1]);
          mma_f16(sn[2 * np + 1], qn[ks], r[2], r[3]);
          if (has_old) {
            ldmatrix_x4(r, sKo + row * kLd + col);
            mma_f16(so[2 * np], qo[ks], r[0], r[1]);
            mma_f16(so[2 * np + 1], qo[ks], r[2], r[3]);
          }
        }
      }
      // Mask (j <= i, padding) and scale to the log2 domain.
      const bool need_mask = (ctok[kAttnCols - 1] > wmin);
      float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int rr = e >> 1;
          const int cj = nt * 8 + (lane & 3) * 2 + (e & 1);
          const int rt = rr ? tok1 : tok0;
          const bool valid = !need_mask || (ctok[cj] <= rt);
          const float vn = valid && rt >= 0 ? sn[nt][e] * g.scale_log2 : -INFINITY;
          const float vo = valid && rt >= 0 ? so[nt][e] * g.scale_log2 : -INFINITY;
          sn[nt][e] = vn;
          so[nt][e] = vo;
          tmax[rr] = fmaxf(tmax[rr], vn);
        }
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        tmax[rr] = fmaxf(tmax[rr], __shfl_xor_sync(0xffffffffu, tmax[rr], 1));
        tmax[rr] = fmaxf(tmax[rr], __shfl_xor_sync(0xffffffffu, tmax[rr], 2));
      }
      float mnew[2], alpha[2];
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        mnew[rr] = fmaxf(m_run[rr], tmax[rr]);
        alpha[rr] = (mnew[rr] == m_run[rr] || mnew[rr] == -INFINITY) ? 1.f : ex2(m_run[rr] - mnew[rr]);
        m_run[rr] = mnew[rr];
        z_run[rr] *= alpha[rr];
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        acc[nt][0] *= alpha[0]; acc[nt][1] *= alpha[0];
        acc[nt][2] *= alpha[1]; acc[nt][3] *= alpha[1];
      }
      // Probabilities (relative to m'), their row sums, fp16 A fragments.
      uint32_t pn[4][4], po[4][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        float en[4], eo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int rr = e >> 1;
          en[e] = sn[nt][e] == -INFINITY ? 0.f : ex2(sn[nt][e] - mnew[rr]);
          eo[e] = (!has_old || so[nt][e] == -INFINITY) ? 0.f : ex2(so[nt][e] - mnew[rr]);
          z_run[rr] += en[e] - eo[e];
        }
        const int kk = nt >> 1, hi = nt & 1;
        pn[kk][hi * 2 + 0] = pack_half2(en[0], en[1]);
        pn[kk][hi * 2 + 1] = pack_half2(en[2], en[3]);
        po[kk][hi * 2 + 0] = pack_half2(-eo[0], -eo[1]);
        po[kk][hi * 2 + 1] = pack_half2(-eo[2], -eo[3]);
      }
      // A fragment order is {rows 0-7 k0-7, rows 8-15 k0-7, rows 0-7 k8-15, rows 8-15 k8-15}.
      uint32_t an[4][4], ao[4][4];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        an[kk][0] = pn[kk][0]; an[kk][1] = pn[kk][1]; an[kk][2] = pn[kk][2]; an[kk][3] = pn[kk][3];
        ao[kk][0] = po[kk][0]; ao[kk][1] = po[kk][1]; ao[kk][2] = po[kk][2]; ao[kk][3] = po[kk][3];
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          uint32_t r[4];
          const int row = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int col = np * 16 + (lane >> 4) * 8;
          ldmatrix_x4_trans(r, sVn + row * kLd + col);
          mma_f16(acc[2 * np], an[kk], r[0], r[1]);
          mma_f16(acc[2 * np + 1], an[kk], r[2], r[3]);
          if (has_old) {
            ldmatrix_x4_trans(r, sVo + row * kLd + col);
            mma_f16(acc[2 * np], ao[kk], r[0], r[1]);
            mma_f16(acc[2 * np + 1], ao[kk], r[2], r[3]);
          }
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // Row totals of Z, then the new state and O = N / Z.
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    z_run[rr] += __shfl_xor_sync(0xffffffffu, z_run[rr], 1);
    z_run[rr] += __shfl_xor_sync(0xffffffffu, z_run[rr], 2);
  }
  const int toks[2] = {tok0, tok1};
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int t = toks[rr];
    if (t < 0) continue;
    if ((lane & 3) == 0) {
      g.m_out[(size_t)h * g.S + t] = m_run[rr] / kLog2e;
      g.z_out[(size_t)h * g.S + t] = z_run[rr];
    }
    const float inv = 1.f / z_run[rr];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int c = nt * 8 + (lane & 3) * 2;
      const float n0 = acc[nt][rr * 2], n1 = acc[nt][rr * 2 + 1];
      *reinterpret_cast<float2*>(g.n_out + ((size_t)h * g.S + t) * DH + c) = make_float2(n0, n1);
      const uint32_t packed = float_to_bf16_bits(n0 * inv) | (static_cast<uint32_t>(float_to_bf16_bits(n1 * inv)) << 16);
      *reinterpret_cast<uint32_t*>(g.o + (size_t)t * HD + (size_t)h * DH + c) = packed;
    }
  }
}

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
    if (col < g.kc) v = *reinterpret_cast<const uint4*>(g.k_new + ((size_t)h * g.kc + col) * DH + q8);
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

int launch_attn_update(const flashloop_params* p, const AttnArgs& a, cudaStream_t stream) {
  dim3 grid((a.row_cap + kAttnRows - 1) / kAttnRows, p->n_heads);
  if (p->head_dim == 128) {
    FL_TRY(cudaFuncSetAttribute(attn_update_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                AttnSmem<128>::kBytes));
    attn_update_kernel<128><<<grid, kAttnThreads, AttnSmem<128>::kBytes, stream>>>(a);
  } else {
    FL_TRY(cudaFuncSetAttribute(attn_update_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                AttnSmem<64>::kBytes));
    attn_update_kernel<64><<<grid, kAttnThreads, AttnSmem<64>::kBytes, stream>>>(a);
  }
  return launch_status();
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
