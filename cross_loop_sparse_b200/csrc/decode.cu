// (a8) Decode: B sequences, one new token each at position S (the context
// length), against that sequence's quantised context caches.
//
// [FL App. G]: the attention kernels read the packed base and residual
// streams directly, never a full-precision copy of the cache, and the decode
// token's column selection is fused behind its loop-1 pass.  [FZ §1]: a
// decode step is bound by the bytes of cache it has to read, so every kernel
// here is an HBM kernel on the CUDA cores (one query row per head leaves
// nothing for the tensor cores):
//   decode_gemv_kernel          x W^T for the B token rows, W streamed once;
//                               RoPE at the token position in the epilogue
//   decode_dense_kernel         loop 1: dense attention over the context's
//                               INT8 base and the token itself, split over
//                               column ranges; whole [columns, H, dh] code
//                               rows arrive by bulk copies; raw scores kept
//   decode_dense_merge_kernel   combine the ranges, O, loop-1 probabilities
//   decode_sparse_kernel        loop r >= 2: remove/add over the selected
//                               columns, split over column ranges
//   decode_sparse_merge_kernel  fold the ranges into the running state
//
// Context rows: token j < S of sequence b is row b*S + j of the context
// streams; its loop-l residual row is ctx slot[l-1][b*S + j] (-1: none).
// Token rows: the decode token of sequence b is row b of the token streams,
// residual rows b at every loop (it is always active).
// Scores are kept in log2 units (q.k * log2(e)/sqrt(dh)); m follows them.
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "tc_util.cuh"

namespace fl {

int launch_kv_quant_rows(int dh, int loop, int n_rows, int H, const int* bits, const float* k_new,
                         const float* v_new, const flashloop_kv& k, const flashloop_kv& v, int32_t* err,
                         cudaStream_t stream);
int launch_topk(const flashloop_params* p, const float* mass, const int32_t* cand, int n_cand, int k,
                int32_t* out, int32_t* err, cudaStream_t stream);

namespace {

constexpr int kThreads = 256;
constexpr int kGemvRows = 8;      // x rows staged per pass of the GEMV
constexpr int kStageCols = 8;     // columns per bulk-copy stage (all heads)
constexpr int kStages = 4;        // ring depth
constexpr int kChunkCols = 128;   // columns per online-softmax chunk
constexpr int kSparseThreads = 128;
constexpr int kSparseCols = 256;  // selected columns per sparse block

struct DecodeArgs {
  int S, H, B, P1, k, loop;
  float kscale;  // log2(e) / sqrt(dh)
  KVStreams ck, cv;  // context streams
  const int32_t* cslot[FLASHLOOP_MAX_LOOPS];
  KVStreams tk, tv;  // token streams
  int bits[FLASHLOOP_MAX_LOOPS];
  const uint16_t* q_old;  // [B, d] bf16
  const uint16_t* q_new;
  const int32_t* cols;  // [B*H, k]
  float* scores;        // [B*H, P1]
  float* part_m;        // dense: [B, nsplit, H];  sparse: [B*H, nblk] (max of s_new)
  float* part_mu;       // sparse: [B*H, nblk] block reference
  float* part_Z;        // dense: [B, nsplit, H];  sparse: [B*H, nblk] (sum e_new - sum e_old)
  float* part_N;        // dense: [B, nsplit, H*dh]; sparse: [B*H, nblk, dh]
  int nsplit;           // dense: column ranges per sequence
  int range;            // dense: columns per range (multiple of kChunkCols)
  int32_t* err;
};

__device__ __forceinline__ float half_bits_f(uint16_t b) { return __half2float(__ushort_as_half(b)); }

// int8 code e (0..3) of word u = w ^ 0x80808080 as float: the byte lands in
// the mantissa of 2^23, and 2^23 + 128 comes off again (exact).
__device__ __forceinline__ float i8_at(uint32_t u, int e) {
  return __int_as_float(static_cast<int>(__byte_perm(u, 0x4B000000u, 0x7540u + e))) - 8388736.0f;
}

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// One-dimensional bulk copy global -> shared (no multicast), completion
// counted in bytes on `bar`.  Both addresses 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------------------
// y[b, n] = sum_k x[b, k] W[n, k] for the B token rows.  One warp owns the
// output pair (n, n + dh/2) of one head block, so that the rotate-half RoPE
// partners meet in one warp.  mode 0: N = 3d (q | k | v): RoPE on q and k at
// the token position, q -> bf16 q_out [B, d], k, v -> f32 k_out, v_out
// [B, d].  mode 1: N = d, y -> bf16 y_out [B, d].
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads)
decode_gemv_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ w, int B, int K, int N,
                   int dh, int H, int mode, const float* __restrict__ rope_cs, uint16_t* q_out,
                   float* k_out, float* v_out, uint16_t* y_out) {
  extern __shared__ __align__(16) float xs[];  // [kGemvRows][K]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int half = dh >> 1;
  const int pair = blockIdx.x * (kThreads / 32) + warp;
  const bool live = pair < (N >> 1);
  const int hb = pair / half, i = pair % half;
  const int n0 = hb * dh + i, n1 = n0 + half;
  const int kc = K >> 3;  // 16-byte chunks per row
  for (int b0 = 0; b0 < B; b0 += kGemvRows) {
    const int nb = min(kGemvRows, B - b0);
    __syncthreads();
    for (int idx = threadIdx.x; idx < nb * kc; idx += kThreads) {
      const int b = idx / kc, c = idx - b * kc;
      const uint4 v = *reinterpret_cast<const uint4*>(x + (size_t)(b0 + b) * K + c * 8);
      const float2 f0 = bf16x2_to_float2(v.x), f1 = bf16x2_to_float2(v.y);
      const float2 f2 = bf16x2_to_float2(v.z), f3 = bf16x2_to_float2(v.w);
      float4* d = reinterpret_cast<float4*>(xs + (size_t)b * K + c * 8);
      d[0] = make_float4(f0.x, f0.y, f1.x, f1.y);
      d[1] = make_float4(f2.x, f2.y, f3.x, f3.y);
    }
    __syncthreads();
    if (!live) continue;
    float a0[kGemvRows], a1[kGemvRows];
#pragma unroll
    for (int b = 0; b < kGemvRows; ++b) a0[b] = a1[b] = 0.f;
    const uint16_t* w0 = w + (size_t)n0 * K;
    const uint16_t* w1 = w + (size_t)n1 * K;
#pragma unroll 2
    for (int c = lane; c < kc; c += 32) {
      const uint4 u0 = ld_stream(w0 + c * 8), u1 = ld_stream(w1 + c * 8);
      float wa[8], wb[8];
      {
        const uint32_t ua[4] = {u0.x, u0.y, u0.z, u0.w}, ub[4] = {u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 fa = bf16x2_to_float2(ua[e]), fb = bf16x2_to_float2(ub[e]);
          wa[2 * e] = fa.x; wa[2 * e + 1] = fa.y;
          wb[2 * e] = fb.x; wb[2 * e + 1] = fb.y;
        }
      }
#pragma unroll
      for (int b = 0; b < kGemvRows; ++b) {
        if (b < nb) {
          const float4* xp = reinterpret_cast<const float4*>(xs + (size_t)b * K + c * 8);
          const float4 x0 = xp[0], x1 = xp[1];
          const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            a0[b] = fmaf(wa[e], xv[e], a0[b]);
            a1[b] = fmaf(wb[e], xv[e], a1[b]);
          }
        }
      }
    }
#pragma unroll
    for (int b = 0; b < kGemvRows; ++b) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        a0[b] += __shfl_xor_sync(0xffffffffu, a0[b], o);
        a1[b] += __shfl_xor_sync(0xffffffffu, a1[b], o);
      }
    }
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int b = 0; b < kGemvRows; ++b)
      if (b == lane) { s0 = a0[b]; s1 = a1[b]; }
    if (lane >= nb) continue;
    const int row = b0 + lane;
    if (mode == 1) {
      y_out[(size_t)row * N + n0] = float_to_bf16_bits(s0);
      y_out[(size_t)row * N + n1] = float_to_bf16_bits(s1);
      continue;
    }
    const int d = H * dh;
    const int section = hb / H, h = hb - section * H;
    const size_t o0 = (size_t)row * d + h * dh + i, o1 = o0 + half;
    if (section < 2) {
      // rotate-half RoPE with explicit roundings (the same float32 result as
      // the prefill projection's epilogue)
      const float c = rope_cs[2 * i], sn = rope_cs[2 * i + 1];
      const float y1 = __fsub_rn(__fmul_rn(s0, c), __fmul_rn(s1, sn));
      const float y2 = __fadd_rn(__fmul_rn(s1, c), __fmul_rn(s0, sn));
      s0 = y1;
      s1 = y2;
    }
    if (section == 0) {
      q_out[o0] = float_to_bf16_bits(s0);
      q_out[o1] = float_to_bf16_bits(s1);
    } else {
      float* dst = section == 1 ? k_out : v_out;
      dst[o0] = s0;
      dst[o1] = s1;
    }
  }
}

// ---------------------------------------------------------------------------
// Loop 1, dense: block (range, b) walks columns [range*R, ...) of sequence b
// for all heads, in chunks of kChunkCols columns, keeping an online softmax
// per head (running max and sum in shared memory, N in registers).  Every
// chunk streams its K stages (scores), then its V stages (weighted sums);
// stages are [kStageCols, H*dh] code rows plus [kStageCols, H*dh/32] scales,
// brought in by bulk copies into a kStages-deep ring.
// Thread roles: scores — thread (column, head, group of 32) with the group's
// 32 q values in registers; weighted sums — thread owns EPT consecutive
// outputs of N (EPT = H*dh/256).
// ---------------------------------------------------------------------------
template <int DH, int EPT>
__global__ void __launch_bounds__(kThreads, 2) decode_dense_kernel(DecodeArgs a) {
  constexpr int G = DH / 32;
  const int H = a.H, HG = H * G;
  const int RB = H * DH;      // code bytes per column
  const int SB = HG * 2;      // scale bytes per column
  const int stage_bytes = kStageCols * (RB + SB);
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);  // [kStages]
  uint8_t* ring = smem + 128;
  float* sc = reinterpret_cast<float*>(ring + (size_t)kStages * stage_bytes);  // [H][kChunkCols]
  float* run_m = sc + H * kChunkCols;   // [H]
  float* run_z = run_m + H;             // [H]
  float* alpha = run_z + H;             // [H]
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.y;
  const int c_begin = blockIdx.x * a.range;
  const int c_end = min(a.P1, c_begin + a.range);
  const int ncols = max(0, c_end - c_begin);
  const int nchunks = (ncols + kChunkCols - 1) / kChunkCols;
  // stage s: chunk s / (2*spc), K if (s % (2*spc)) < spc, else V
  const int spc = kChunkCols / kStageCols;
  int total = 0;
  for (int ch = 0; ch < nchunks; ++ch) {
    const int n = min(kChunkCols, ncols - ch * kChunkCols);
    total += 2 * ((n + kStageCols - 1) / kStageCols);
  }

  if (tid == 0) {
    s_abort = 0;
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  for (int h = tid; h < H; h += kThreads) {
    run_m[h] = -INFINITY;
    run_z[h] = 0.f;
  }
  __syncthreads();

  // map stage sequence number -> (chunk, is_v, stage-in-chunk)
  auto stage_of = [&](int s, int& ch, int& isv, int& st) {
    int rem = s;
    for (ch = 0; ch < nchunks; ++ch) {
      const int n = min(kChunkCols, ncols - ch * kChunkCols);
      const int ns = (n + kStageCols - 1) / kStageCols;
      if (rem < 2 * ns) break;
      rem -= 2 * ns;
    }
    const int n = min(kChunkCols, ncols - ch * kChunkCols);
    const int ns = (n + kStageCols - 1) / kStageCols;
    isv = rem >= ns;
    st = isv ? rem - ns : rem;
  };
  auto issue = [&](int s) {
    int ch, isv, st;
    stage_of(s, ch, isv, st);
    const int col0 = c_begin + ch * kChunkCols + st * kStageCols;
    const int n = min(kStageCols, min(c_begin + (ch + 1) * kChunkCols, c_end) - col0);
    const int n_ctx = max(0, min(n, a.S - col0));
    const bool has_tok = col0 + n > a.S;
    uint8_t* buf = ring + (size_t)(s % kStages) * stage_bytes;
    uint64_t* bar = &full[s % kStages];
    const KVStreams& cs = isv ? a.cv : a.ck;
    const KVStreams& ts = isv ? a.tv : a.tk;
    const uint32_t bytes = (uint32_t)(n_ctx + (has_tok ? 1 : 0)) * (RB + SB);
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, bytes);
    if (n_ctx > 0) {
      const size_t row = (size_t)b * a.S + col0;
      bulk_load(buf, cs.base_codes + row * RB, (uint32_t)(n_ctx * RB), bar);
      bulk_load(buf + kStageCols * RB, reinterpret_cast<const uint8_t*>(cs.base_scales) + row * SB,
                (uint32_t)(n_ctx * SB), bar);
    }
    if (has_tok) {
      const int jt = a.S - col0;
      bulk_load(buf + (size_t)jt * RB, ts.base_codes + (size_t)b * RB, (uint32_t)RB, bar);
      bulk_load(buf + kStageCols * RB + (size_t)jt * SB,
                reinterpret_cast<const uint8_t*>(ts.base_scales) + (size_t)b * SB, (uint32_t)SB, bar);
    }
  };

  // score role: (column-in-pass, head, group)
  const int hg = tid % HG, jsub = tid / HG;
  const int cpp = kThreads / HG;  // columns per pass
  const int sh = hg / G;
  float q[32];
  {
    const uint16_t* qp = a.q_new + (size_t)b * RB + hg * 32;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint4 u = *reinterpret_cast<const uint4*>(qp + v * 8);
      const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = bf16x2_to_float2(uu[e]);
        q[v * 8 + 2 * e] = f.x;
        q[v * 8 + 2 * e + 1] = f.y;
      }
    }
  }
  // weighted-sum role: outputs [o, o + EPT) of head oh
  const int o = tid * EPT, oh = o / DH;
  float acc[EPT];
#pragma unroll
  for (int e = 0; e < EPT; ++e) acc[e] = 0.f;

  int issued = 0;  // thread 0 only
  if (tid == 0)
    for (; issued < kStages - 1 && issued < total; ++issued) issue(issued);

  bool ok = true;
  int s = 0;  // stage sequence number
  for (int ch = 0; ch < nchunks; ++ch) {
    const int chunk0 = c_begin + ch * kChunkCols;
    const int n = min(kChunkCols, ncols - ch * kChunkCols);
    const int ns = (n + kStageCols - 1) / kStageCols;
    for (int phase = 0; phase < 2; ++phase) {
      for (int st = 0; st < ns; ++st, ++s) {
        if (tid == 0 && !s_abort && s + kStages - 1 < total) issue(issued++);
        if (ok && !s_abort) {
          if (!mbar_wait(&full[s % kStages], (s / kStages) & 1)) {
            set_error(a.err, kDevErrTimeout);
            s_abort = 1;
            ok = false;
          }
        }
        const uint8_t* buf = ring + (size_t)(s % kStages) * stage_bytes;
        const int nv = min(kStageCols, n - st * kStageCols);
        // one decision per warp: the shuffles below need every lane
        if (__all_sync(0xffffffffu, ok && !s_abort)) {
          if (phase == 0) {
            for (int p0 = 0; p0 < kStageCols; p0 += cpp) {
              const int jj = p0 + jsub;
              float part = 0.f;
              if (jj < nv) {
                const uint8_t* row = buf + (size_t)jj * RB + hg * 32;
                // odd lanes read the second 16 bytes first: the two loads of
                // a warp then spread over all banks
                const bool odd = lane & 1;
                const uint4 ca = *reinterpret_cast<const uint4*>(row + (odd ? 16 : 0));
                const uint4 cb = *reinterpret_cast<const uint4*>(row + (odd ? 0 : 16));
                const uint4 c0 = odd ? cb : ca, c1 = odd ? ca : cb;
                const uint32_t w0[4] = {c0.x ^ 0x80808080u, c0.y ^ 0x80808080u, c0.z ^ 0x80808080u,
                                        c0.w ^ 0x80808080u};
                const uint32_t w1[4] = {c1.x ^ 0x80808080u, c1.y ^ 0x80808080u, c1.z ^ 0x80808080u,
                                        c1.w ^ 0x80808080u};
                float d0 = 0.f, d1 = 0.f;
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                  d0 = fmaf(q[e], i8_at(w0[e >> 2], e & 3), d0);
                  d1 = fmaf(q[16 + e], i8_at(w1[e >> 2], e & 3), d1);
                }
                const uint16_t* scl = reinterpret_cast<const uint16_t*>(buf + kStageCols * RB);
                part = (d0 + d1) * half_bits_f(scl[jj * HG + hg]);
              }
#pragma unroll
              for (int off = 1; off < G; off <<= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
              if (jj < nv && (hg % G) == 0) sc[sh * kChunkCols + st * kStageCols + jj] = part * a.kscale;
            }
          } else {
            const uint16_t* scl = reinterpret_cast<const uint16_t*>(buf + kStageCols * RB);
            for (int jj = 0; jj < nv; ++jj) {
              const float f = sc[oh * kChunkCols + st * kStageCols + jj] * half_bits_f(scl[jj * HG + o / 32]);
              const uint8_t* src = buf + (size_t)jj * RB + o;
              if constexpr (EPT >= 4) {
#pragma unroll
                for (int v = 0; v < EPT / 4; ++v) {
                  const uint32_t u = reinterpret_cast<const uint32_t*>(src)[v] ^ 0x80808080u;
#pragma unroll
                  for (int e = 0; e < 4; ++e) acc[4 * v + e] = fmaf(f, i8_at(u, e), acc[4 * v + e]);
                }
              } else {
#pragma unroll
                for (int e = 0; e < EPT; ++e)
                  acc[e] = fmaf(f, static_cast<float>(reinterpret_cast<const int8_t*>(src)[e]), acc[e]);
              }
            }
          }
        }
        __syncthreads();
      }
      if (phase == 0) {
        // online softmax over this chunk: new running max, rescale factor,
        // weights in place of the scores, raw scores kept for the selection
        for (int h = warp; h < H; h += kThreads / 32) {
          float mx = -INFINITY;
          for (int jc = lane; jc < n; jc += 32) mx = fmaxf(mx, sc[h * kChunkCols + jc]);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
          const float m_new = fmaxf(run_m[h], mx);
          float z = 0.f;
          float* srow = a.scores + ((size_t)b * H + h) * a.P1 + chunk0;
          for (int jc = lane; jc < n; jc += 32) {
            const float sv = sc[h * kChunkCols + jc];
            srow[jc] = sv;
            const float e = ex2(sv - m_new);
            sc[h * kChunkCols + jc] = e;
            z += e;
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
          if (lane == 0) {
            const float al = ex2(run_m[h] - m_new);  // 0 while run_m is -inf
            alpha[h] = al;
            run_z[h] = run_z[h] * al + z;
            run_m[h] = m_new;
          }
        }
        __syncthreads();
        const float al = alpha[oh];
#pragma unroll
        for (int e = 0; e < EPT; ++e) acc[e] *= al;
      }
    }
  }
  // partials of this range
  const size_t pr = (size_t)b * a.nsplit + blockIdx.x;
  for (int h = tid; h < H; h += kThreads) {
    a.part_m[pr * H + h] = run_m[h];
    a.part_Z[pr * H + h] = run_z[h];
  }
#pragma unroll
  for (int e = 0; e < EPT; ++e) a.part_N[pr * RB + o + e] = acc[e];
  // a wait that gave up may leave a copy in flight: let it land first
  if (tid == 0 && s_abort) {
    for (int t = max(0, issued - kStages); t < issued; ++t) mbar_wait(&full[t % kStages], (t / kStages) & 1);
  }
}

// Combine the ranges of each (sequence, head): state slot 0, O, and the
// loop-1 probabilities of every column 0..S.
template <int DH>
__global__ void __launch_bounds__(kThreads) decode_dense_merge_kernel(DecodeArgs a, float* m_out, float* z_out,
                                                                      float* n_out, uint16_t* o_out,
                                                                      float* probs) {
  const int bh = blockIdx.x, b = bh / a.H, h = bh - b * a.H;
  __shared__ float s_m, s_z;
  __shared__ float red[kThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float mx = -INFINITY;
  for (int r = tid; r < a.nsplit; r += kThreads) mx = fmaxf(mx, a.part_m[((size_t)b * a.nsplit + r) * a.H + h]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  if (tid == 0) {
    float m = red[0];
    for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, red[w]);
    float z = 0.f;
    for (int r = 0; r < a.nsplit; ++r) {
      const size_t i = ((size_t)b * a.nsplit + r) * a.H + h;
      z += ex2(a.part_m[i] - m) * a.part_Z[i];
    }
    s_m = m;
    s_z = z;
  }
  __syncthreads();
  const float m = s_m, z = s_z;
  for (int e = tid; e < DH; e += kThreads) {
    float n = 0.f;
    for (int r = 0; r < a.nsplit; ++r) {
      const size_t i = (size_t)b * a.nsplit + r;
      n += ex2(a.part_m[i * a.H + h] - m) * a.part_N[i * a.H * DH + h * DH + e];
    }
    n_out[(size_t)bh * DH + e] = n;
    o_out[(size_t)b * a.H * DH + h * DH + e] = float_to_bf16_bits(n / z);
  }
  if (tid == 0) {
    m_out[bh] = m;
    z_out[bh] = z;
  }
  const float rz = 1.f / z;
  const float* srow = a.scores + (size_t)bh * a.P1;
  float* prow = probs + (size_t)bh * a.P1;
  for (int j = tid; j < a.P1; j += kThreads) prow[j] = ex2(srow[j] - m) * rz;
}

// ---------------------------------------------------------------------------
// Loop r >= 2, sparse: block (range, b*H + h) takes kSparseCols of the
// selected columns.  8 lanes per column (each lane DH/8 elements), 16
// columns per block step.  Pass 1 rebuilds K^(r-1) and K^(r) of each column
// from the packed streams and keeps both scores; pass 2 rebuilds V^(r-1),
// V^(r) and sums e_new V^(r) - e_old V^(r-1) against the block's own
// reference max.
// ---------------------------------------------------------------------------
// acc[e] += code(e) * s for E8 consecutive BITS-bit two's-complement codes
// starting at src (E8 * BITS / 8 bytes, aligned to their size).
template <int E8, int BITS>
__device__ __forceinline__ void add_res(const uint8_t* src, float s, float (&acc)[E8]) {
  constexpr int NB = E8 * BITS / 8;
  constexpr int PW = 32 / BITS;
  uint32_t words[(NB + 3) / 4];
  if constexpr (NB >= 4) {
#pragma unroll
    for (int v = 0; v < NB / 4; ++v) words[v] = reinterpret_cast<const uint32_t*>(src)[v];
  } else if constexpr (NB == 2) {
    words[0] = *reinterpret_cast<const uint16_t*>(src);
  } else {
    words[0] = *src;
  }
#pragma unroll
  for (int e = 0; e < E8; ++e) {
    int c = static_cast<int>((words[e / PW] >> ((e % PW) * BITS)) & ((1u << BITS) - 1u));
    if (c >= (1 << (BITS - 1))) c -= (1 << BITS);
    acc[e] = acc[e] + static_cast<float>(c) * s;
  }
}

// Rows: a token column reads row b of every token stream; a context column
// reads base row t and residual rows cslot[l-1][t].
template <int E8>
__device__ __forceinline__ void rebuild(const KVStreams& kv, const DecodeArgs& a, bool tok, int b, size_t t,
                                        int h, int DH, int e0, float (&old_v)[E8], float (&new_v)[E8]) {
  const int H = a.H, loop = a.loop;
  const size_t base_row = tok ? (size_t)b : t;
  {
    const int8_t* src = kv.base_codes + (base_row * H + h) * DH + e0;
    const float s = half_bits_f(kv.base_scales[(base_row * H + h) * (DH / 32) + e0 / 32]);
#pragma unroll
    for (int v = 0; v < E8 / 4; ++v) {
      const uint32_t u = reinterpret_cast<const uint32_t*>(src)[v] ^ 0x80808080u;
#pragma unroll
      for (int e = 0; e < 4; ++e) old_v[4 * v + e] = i8_at(u, e) * s;
    }
  }
  for (int l = 2; l <= loop; ++l) {
    const int sl = tok ? b : a.cslot[l - 1][t];
    if (l == loop) {
#pragma unroll
      for (int e = 0; e < E8; ++e) new_v[e] = old_v[e];
    }
    if (sl < 0) continue;
    const int bb = a.bits[l - 1];
    const uint8_t* row = kv.res_codes[l - 1] + ((size_t)sl * H + h) * (DH * bb / 8);
    const float s = half_bits_f(kv.res_scales[l - 1][((size_t)sl * H + h) * (DH / 32) + e0 / 32]);
    const uint8_t* src = row + (e0 * bb) / 8;
    if (l < loop) {
      if (bb == 2) add_res<E8, 2>(src, s, old_v);
      else if (bb == 4) add_res<E8, 4>(src, s, old_v);
      else add_res<E8, 8>(src, s, old_v);
    } else {
      if (bb == 2) add_res<E8, 2>(src, s, new_v);
      else if (bb == 4) add_res<E8, 4>(src, s, new_v);
      else add_res<E8, 8>(src, s, new_v);
    }
  }
  if (loop == 1) {
#pragma unroll
    for (int e = 0; e < E8; ++e) new_v[e] = old_v[e];
  }
}

template <int DH>
__global__ void __launch_bounds__(kSparseThreads) decode_sparse_kernel(DecodeArgs a) {
  constexpr int E8 = DH / 8;
  __shared__ float s_old[kSparseCols], s_new[kSparseCols];
  __shared__ float red[3][kSparseThreads / 32];
  __shared__ float nred[kSparseThreads / 32][DH];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int u = lane & 7, grp = warp * 4 + (lane >> 3);
  const int bh = blockIdx.y, b = bh / a.H, h = bh - b * a.H;
  const int c_begin = blockIdx.x * kSparseCols;
  const int n = max(0, min(kSparseCols, a.k - c_begin));
  const int e0 = u * E8;
  const int d = a.H * DH;
  float qo[E8], qn[E8];
  {
    const uint16_t* po = a.q_old + (size_t)b * d + h * DH + e0;
    const uint16_t* pn = a.q_new + (size_t)b * d + h * DH + e0;
#pragma unroll
    for (int v = 0; v < E8 / 2; ++v) {
      const float2 fo = bf16x2_to_float2(reinterpret_cast<const uint32_t*>(po)[v]);
      const float2 fn = bf16x2_to_float2(reinterpret_cast<const uint32_t*>(pn)[v]);
      qo[2 * v] = fo.x; qo[2 * v + 1] = fo.y;
      qn[2 * v] = fn.x; qn[2 * v + 1] = fn.y;
    }
  }
  const int32_t* cols = a.cols + (size_t)bh * a.k + c_begin;
  auto column = [&](int jl, bool& tok) -> size_t {
    int j = cols[jl];
    if (j < 0 || j > a.S) {
      set_error(a.err, FLASHLOOP_DEVERR_INDEX);
      j = a.S;
    }
    tok = j == a.S;
    return (size_t)b * a.S + j;
  };
  const int steps = (n + 15) / 16;
  float mu = -INFINITY, mxn = -INFINITY;
  for (int it = 0; it < steps; ++it) {
    const int jl = it * 16 + grp;
    float dol = 0.f, dnw = 0.f;
    if (jl < n) {
      bool tok;
      const size_t t = column(jl, tok);
      float ko[E8], kn[E8];
      rebuild<E8>(tok ? a.tk : a.ck, a, tok, b, t, h, DH, e0, ko, kn);
#pragma unroll
      for (int e = 0; e < E8; ++e) {
        dol = fmaf(qo[e], ko[e], dol);
        dnw = fmaf(qn[e], kn[e], dnw);
      }
    }
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
      dol += __shfl_xor_sync(0xffffffffu, dol, off);
      dnw += __shfl_xor_sync(0xffffffffu, dnw, off);
    }
    if (jl < n) {
      dol *= a.kscale;
      dnw *= a.kscale;
      if (u == 0) {
        s_old[jl] = dol;
        s_new[jl] = dnw;
      }
      mu = fmaxf(mu, fmaxf(dol, dnw));
      mxn = fmaxf(mxn, dnw);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    mu = fmaxf(mu, __shfl_xor_sync(0xffffffffu, mu, off));
    mxn = fmaxf(mxn, __shfl_xor_sync(0xffffffffu, mxn, off));
  }
  if (lane == 0) {
    red[0][warp] = mu;
    red[1][warp] = mxn;
  }
  __syncthreads();
  mu = red[0][0];
  mxn = red[1][0];
#pragma unroll
  for (int w = 1; w < kSparseThreads / 32; ++w) {
    mu = fmaxf(mu, red[0][w]);
    mxn = fmaxf(mxn, red[1][w]);
  }
  float acc[E8];
#pragma unroll
  for (int e = 0; e < E8; ++e) acc[e] = 0.f;
  float zn = 0.f, zo = 0.f;
  for (int it = 0; it < steps; ++it) {
    const int jl = it * 16 + grp;
    if (jl < n) {
      bool tok;
      const size_t t = column(jl, tok);
      float vo[E8], vn[E8];
      rebuild<E8>(tok ? a.tv : a.cv, a, tok, b, t, h, DH, e0, vo, vn);
      const float en = ex2(s_new[jl] - mu), eo = ex2(s_old[jl] - mu);
#pragma unroll
      for (int e = 0; e < E8; ++e) acc[e] = fmaf(en, vn[e], fmaf(-eo, vo[e], acc[e]));
      zn += en;
      zo += eo;
    }
  }
  // reduce the 4 column groups of each warp, then the warps
#pragma unroll
  for (int e = 0; e < E8; ++e) {
    acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 8);
    acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
  }
  zn += __shfl_xor_sync(0xffffffffu, zn, 8);
  zn += __shfl_xor_sync(0xffffffffu, zn, 16);
  zo += __shfl_xor_sync(0xffffffffu, zo, 8);
  zo += __shfl_xor_sync(0xffffffffu, zo, 16);
  if (lane < 8) {
#pragma unroll
    for (int e = 0; e < E8; ++e) nred[warp][e0 + e] = acc[e];
  }
  if (lane == 0) {
    red[0][warp] = zn;
    red[1][warp] = zo;
  }
  __syncthreads();
  const size_t pi = (size_t)bh * gridDim.x + blockIdx.x;
  for (int e = tid; e < DH; e += kSparseThreads) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kSparseThreads / 32; ++w) v += nred[w][e];
    a.part_N[pi * DH + e] = v;
  }
  if (tid == 0) {
    float zsn = 0.f, zso = 0.f;
#pragma unroll
    for (int w = 0; w < kSparseThreads / 32; ++w) {
      zsn += red[0][w];
      zso += red[1][w];
    }
    a.part_m[pi] = mxn;
    a.part_mu[pi] = mu;
    a.part_Z[pi] = zsn - zso;
  }
}

// Fold the ranges into the running state: m' = max(m, max s_new),
// Z' = e^(m-m') Z + sum_ranges e^(mu-m') (sum e_new - sum e_old), and the
// same for N; O = N'/Z'.
template <int DH>
__global__ void __launch_bounds__(DH) decode_sparse_merge_kernel(DecodeArgs a, int nblk, const float* m_in,
                                                                 const float* z_in, const float* n_in,
                                                                 float* m_out, float* z_out, float* n_out,
                                                                 uint16_t* o_out) {
  const int bh = blockIdx.x, b = bh / a.H, h = bh - b * a.H;
  const int e = threadIdx.x;
  const float m = m_in[bh];
  float mn = m;
  for (int r = 0; r < nblk; ++r) mn = fmaxf(mn, a.part_m[(size_t)bh * nblk + r]);
  const float al = ex2(m - mn);
  float z = al * z_in[bh];
  float nv = al * n_in[(size_t)bh * DH + e];
  for (int r = 0; r < nblk; ++r) {
    const size_t i = (size_t)bh * nblk + r;
    const float f = ex2(a.part_mu[i] - mn);  // 0 for an empty range (mu = -inf)
    z = fmaf(f, a.part_Z[i], z);
    nv = fmaf(f, a.part_N[i * DH + e], nv);
  }
  n_out[(size_t)bh * DH + e] = nv;
  o_out[(size_t)b * a.H * DH + h * DH + e] = float_to_bf16_bits(nv / z);
  if (e == 0) {
    m_out[bh] = mn;
    z_out[bh] = z;
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
inline int dense_nsplit(int B, int P1) {
  // two resident blocks per SM over the whole batch, at least one chunk each
  int ns = (2 * 148 + B - 1) / B;
  const int max_ns = (P1 + kChunkCols - 1) / kChunkCols;
  return ns < max_ns ? ns : max_ns;
}

DecodeLayout decode_layout(const flashloop_params* p) {
  DecodeLayout L{};
  const size_t B = p->batch, H = p->n_heads, dh = p->head_dim, d = p->d_model;
  const int P1 = p->seq + 1;
  L.nsplit = dense_nsplit((int)B, P1);
  const int chunks = (P1 + kChunkCols - 1) / kChunkCols;
  L.range = ((chunks + L.nsplit - 1) / L.nsplit) * kChunkCols;
  L.nsplit = (P1 + L.range - 1) / L.range;
  const int k = p->n_loops >= 2 ? p->topk[1] : 1;
  L.nblk = (k + kSparseCols - 1) / kSparseCols;
  size_t off = 0;
  L.k_new = off; off = align256(off + B * d * sizeof(float));
  L.v_new = off; off = align256(off + B * d * sizeof(float));
  L.scores = off; off = align256(off + B * H * (size_t)P1 * sizeof(float));
  const size_t np = std::max(B * (size_t)L.nsplit * H, B * H * (size_t)L.nblk);
  L.part_m = off; off = align256(off + np * sizeof(float));
  L.part_mu = off; off = align256(off + np * sizeof(float));
  L.part_Z = off; off = align256(off + np * sizeof(float));
  const size_t nn = std::max(B * (size_t)L.nsplit * H * dh, B * H * (size_t)L.nblk * dh);
  L.part_N = off; off = align256(off + nn * sizeof(float));
  L.total = off;
  return L;
}

size_t decode_dense_smem(const flashloop_params* p) {
  const int H = p->n_heads, RB = H * p->head_dim, SB = H * (p->head_dim / 32) * 2;
  return 128 + (size_t)kStages * kStageCols * (RB + SB) + ((size_t)H * kChunkCols + 3 * H) * sizeof(float);
}

static DecodeArgs make_args(const flashloop_params* p, int loop, const flashloop_state* ctx,
                            const flashloop_decode_state* ds, const DecodeLayout& L) {
  DecodeArgs a{};
  a.S = p->seq;
  a.H = p->n_heads;
  a.B = p->batch;
  a.P1 = p->seq + 1;
  a.k = p->n_loops >= 2 ? p->topk[1] : 1;
  a.loop = loop;
  a.kscale = (float)(1.4426950408889634 / std::sqrt((double)p->head_dim));
  a.ck = kv_streams(ctx->k);
  a.cv = kv_streams(ctx->v);
  a.tk = kv_streams(ds->k);
  a.tv = kv_streams(ds->v);
  for (int i = 0; i < FLASHLOOP_MAX_LOOPS; ++i) {
    a.cslot[i] = ctx->slot[i];
    a.bits[i] = p->bits[i];
  }
  a.q_new = reinterpret_cast<const uint16_t*>(ds->q[slot_of_loop(loop)]);
  a.q_old = loop >= 2 ? reinterpret_cast<const uint16_t*>(ds->q[slot_of_loop(loop - 1)]) : nullptr;
  a.cols = ds->cols;
  a.scores = ws_ptr<float>(ds->workspace, L.scores);
  a.part_m = ws_ptr<float>(ds->workspace, L.part_m);
  a.part_mu = ws_ptr<float>(ds->workspace, L.part_mu);
  a.part_Z = ws_ptr<float>(ds->workspace, L.part_Z);
  a.part_N = ws_ptr<float>(ds->workspace, L.part_N);
  a.nsplit = L.nsplit;
  a.range = L.range;
  a.err = ds->err_word;
  return a;
}

template <int DH, int EPT>
static int launch_dense_t(const DecodeArgs& a, size_t smem, cudaStream_t stream) {
  static bool attr = false;
  if (!attr) {
    FL_TRY(cudaFuncSetAttribute(decode_dense_kernel<DH, EPT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem));
    attr = true;
  }
  decode_dense_kernel<DH, EPT><<<dim3(a.nsplit, a.B), kThreads, smem, stream>>>(a);
  return launch_status();
}

int launch_decode_attn(const flashloop_params* p, int loop, const flashloop_state* ctx,
                       flashloop_decode_state* ds, cudaStream_t stream) {
  const DecodeLayout L = decode_layout(p);
  const DecodeArgs a = make_args(p, loop, ctx, ds, L);
  const int dh = p->head_dim, H = p->n_heads, B = p->batch;
  if (loop == 1) {
    const size_t smem = decode_dense_smem(p);
    const int ept = H * dh / kThreads;
    int rc = FLASHLOOP_ERR_UNSUPPORTED;
#define FL_DENSE(D, E) \
  if (dh == D && ept == E) rc = launch_dense_t<D, E>(a, smem, stream);
    FL_DENSE(64, 1) FL_DENSE(64, 2) FL_DENSE(64, 4) FL_DENSE(64, 8)
    FL_DENSE(128, 1) FL_DENSE(128, 2) FL_DENSE(128, 4) FL_DENSE(128, 8) FL_DENSE(128, 16)
#undef FL_DENSE
    if (rc != FLASHLOOP_OK) return rc;
    if (dh == 128)
      decode_dense_merge_kernel<128><<<B * H, kThreads, 0, stream>>>(a, ds->m[0], ds->Z[0], ds->N[0],
                                                                     reinterpret_cast<uint16_t*>(ds->O), ds->probs);
    else
      decode_dense_merge_kernel<64><<<B * H, kThreads, 0, stream>>>(a, ds->m[0], ds->Z[0], ds->N[0],
                                                                    reinterpret_cast<uint16_t*>(ds->O), ds->probs);
    rc = launch_status();
    if (rc != FLASHLOOP_OK || p->n_loops < 2) return rc;
    // fused selection: top-k of each (sequence, head) row of probabilities
    flashloop_params ps = *p;
    ps.n_heads = B * H;
    ps.seq = p->seq + 1;
    return launch_topk(&ps, ds->probs, nullptr, 0, a.k, ds->cols, ds->err_word, stream);
  }
  const int si = slot_of_loop(loop - 1), so = slot_of_loop(loop);
  if (dh == 128) {
    decode_sparse_kernel<128><<<dim3(L.nblk, B * H), kSparseThreads, 0, stream>>>(a);
    decode_sparse_merge_kernel<128><<<B * H, 128, 0, stream>>>(a, L.nblk, ds->m[si], ds->Z[si], ds->N[si], ds->m[so],
                                                               ds->Z[so], ds->N[so], reinterpret_cast<uint16_t*>(ds->O));
  } else {
    decode_sparse_kernel<64><<<dim3(L.nblk, B * H), kSparseThreads, 0, stream>>>(a);
    decode_sparse_merge_kernel<64><<<B * H, 64, 0, stream>>>(a, L.nblk, ds->m[si], ds->Z[si], ds->N[si], ds->m[so],
                                                             ds->Z[so], ds->N[so], reinterpret_cast<uint16_t*>(ds->O));
  }
  return launch_status();
}

int launch_decode_gemv(const flashloop_params* p, const uint16_t* x, const uint16_t* w, int mode,
                       const float* rope_cs, uint16_t* q_out, float* k_out, float* v_out, uint16_t* y_out,
                       cudaStream_t stream) {
  const int d = p->d_model, N = mode == 0 ? 3 * d : d;
  const size_t smem = (size_t)kGemvRows * d * sizeof(float);
  static size_t attr = 0;
  if (smem > attr) {
    FL_TRY(cudaFuncSetAttribute(decode_gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    attr = smem;
  }
  const int pairs = N / 2, warps = kThreads / 32;
  decode_gemv_kernel<<<(pairs + warps - 1) / warps, kThreads, smem, stream>>>(
      x, w, p->batch, d, N, p->head_dim, p->n_heads, mode, rope_cs, q_out, k_out, v_out, y_out);
  return launch_status();
}

int launch_decode_step(const flashloop_params* p, int loop, const uint16_t* x_tok, const uint16_t* w_qkv,
                       const uint16_t* w_o, const flashloop_state* ctx, flashloop_decode_state* ds,
                       cudaStream_t stream) {
  const DecodeLayout L = decode_layout(p);
  float* k_new = ws_ptr<float>(ds->workspace, L.k_new);
  float* v_new = ws_ptr<float>(ds->workspace, L.v_new);
  int rc = launch_decode_gemv(p, x_tok, w_qkv, 0, ds->rope_cs,
                              reinterpret_cast<uint16_t*>(ds->q[slot_of_loop(loop)]), k_new, v_new, nullptr, stream);
  if (rc != FLASHLOOP_OK) return rc;
  rc = launch_kv_quant_rows(p->head_dim, loop, p->batch, p->n_heads, p->bits, k_new, v_new, ds->k, ds->v,
                            ds->err_word, stream);
  if (rc != FLASHLOOP_OK) return rc;
  rc = launch_decode_attn(p, loop, ctx, ds, stream);
  if (rc != FLASHLOOP_OK) return rc;
  return launch_decode_gemv(p, reinterpret_cast<const uint16_t*>(ds->O), w_o, 1, nullptr, nullptr, nullptr,
                            nullptr, reinterpret_cast<uint16_t*>(ds->Y), stream);
}

}  // namespace fl
