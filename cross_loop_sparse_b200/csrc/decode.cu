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
                int32_t* out, int32_t* err, cudaStream_t stream, const float* row_m = nullptr,
                const float* row_z = nullptr, float* probs_out = nullptr, const int32_t* n_dev = nullptr,
                int32_t* k_out = nullptr, const int32_t* out_map = nullptr);

namespace {

constexpr int kThreads = 256;
constexpr int kGemvWarps = 8;     // warps of a GEMV block (they split K)
constexpr int kGemvBatch = 4;     // 32-wide k steps of weight loads a lane has in flight
constexpr int kStageCols = 8;     // columns per bulk-copy stage (all heads)
constexpr int kStages = 4;        // ring depth
constexpr int kChunkCols = 128;   // columns per online-softmax chunk
constexpr int kScRow = kChunkCols + 4;  // row pitch of the per-head scores (bank spread)
constexpr int kSparseThreads = 128;
constexpr int kSparseCols = 256;  // selected columns per sparse block
constexpr int kSparseStageCols = 16;  // columns per gather stage (8 threads each)
constexpr int kSparseStages = 4;      // gather ring depth

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
  uint16_t* kv_part;    // [B*H, k, 2, dh] fp16: Khat, Vhat of the selected columns after the last sparse loop
  int write_part;       // the loop writes Khat^(loop), Vhat^(loop) to kv_part (a later loop reads them)
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
// y[b, n] = sum_k x[b, k] W[n, k] for the decode token rows, on the tensor
// cores (mma.sync m16n8k16, bf16 operands, f32 accumulators): a weight tile
// is the A operand (16 output rows x 16 k), eight token rows the B operand
// (16 k x 8 tokens; blockIdx.y picks the group of eight).  A block owns two
// 16-row tiles: rows n0.. and n0 + dh/2.. in the QKV projection (the
// rotate-half RoPE partners) or two consecutive tiles of W_o; its
// kGemvWarps warps split K and add their partial sums in shared memory.
// Within a 32-wide k step a lane reads 16 consecutive bytes (8 k) of a
// weight row: the step's two MMAs take k 8t..8t+3 and 8t+4..8t+7 of lane
// quad t, a fixed permutation of k that the token operand follows, so the
// sum over k is unchanged.
// mode 0: N = 3d (q | k | v): RoPE on q and k at the token position,
// q -> bf16 q_out [B, d], k, v -> f32 k_out, v_out [B, d].
// mode 1: N = d, y -> bf16 y_out [B, d].
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kGemvWarps * 32)
decode_gemv_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ w, int B, int K, int N,
                   int dh, int H, int mode, const float* __restrict__ rope_cs, uint16_t* q_out,
                   float* k_out, float* v_out, uint16_t* y_out) {
  __shared__ float red[kGemvWarps][2][16][8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  int n0, n1;
  if (mode == 0) {
    const int half = dh >> 1, tph = half / 16;  // tile pairs per head block
    const int hb = blockIdx.x / tph, it = blockIdx.x - hb * tph;
    n0 = hb * dh + it * 16;
    n1 = n0 + half;
  } else {
    n0 = blockIdx.x * 32;
    n1 = n0 + 16;
  }
  const int tok0 = blockIdx.y * 8;
  const bool xrow = tok0 + g < B;
  const uint16_t* xr = x + (size_t)(xrow ? tok0 + g : 0) * K;
  const uint16_t* w0g = w + (size_t)(n0 + g) * K;
  const uint16_t* w0h = w + (size_t)(n0 + g + 8) * K;
  const uint16_t* w1g = w + (size_t)(n1 + g) * K;
  const uint16_t* w1h = w + (size_t)(n1 + g + 8) * K;
  const int kw = K / kGemvWarps;  // K slice of this warp (a multiple of 32)
  const int k_begin = warp * kw, k_end = k_begin + kw;
  float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
  for (int kb = k_begin; kb < k_end; kb += 32 * kGemvBatch) {
    uint4 a0g[kGemvBatch], a0h[kGemvBatch], a1g[kGemvBatch], a1h[kGemvBatch], xb[kGemvBatch];
#pragma unroll
    for (int i = 0; i < kGemvBatch; ++i) {
      const int k = kb + 32 * i + 8 * t;
      const bool in = kb + 32 * i < k_end;
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
      a0g[i] = in ? ld_stream(w0g + k) : z;
      a0h[i] = in ? ld_stream(w0h + k) : z;
      a1g[i] = in ? ld_stream(w1g + k) : z;
      a1h[i] = in ? ld_stream(w1h + k) : z;
      xb[i] = in && xrow ? *reinterpret_cast<const uint4*>(xr + k) : z;
    }
#pragma unroll
    for (int i = 0; i < kGemvBatch; ++i) {
      const uint32_t a00[4] = {a0g[i].x, a0h[i].x, a0g[i].y, a0h[i].y};
      const uint32_t a01[4] = {a0g[i].z, a0h[i].z, a0g[i].w, a0h[i].w};
      const uint32_t a10[4] = {a1g[i].x, a1h[i].x, a1g[i].y, a1h[i].y};
      const uint32_t a11[4] = {a1g[i].z, a1h[i].z, a1g[i].w, a1h[i].w};
      mma_bf16(d0, a00, xb[i].x, xb[i].y);
      mma_bf16(d1, a10, xb[i].x, xb[i].y);
      mma_bf16(d0, a01, xb[i].z, xb[i].w);
      mma_bf16(d1, a11, xb[i].z, xb[i].w);
    }
  }
  // D fragment: d[0] = (row g, token 2t), d[1] = (g, 2t+1), d[2] = (g+8, 2t), d[3] = (g+8, 2t+1)
  red[warp][0][g][2 * t] = d0[0];
  red[warp][0][g][2 * t + 1] = d0[1];
  red[warp][0][g + 8][2 * t] = d0[2];
  red[warp][0][g + 8][2 * t + 1] = d0[3];
  red[warp][1][g][2 * t] = d1[0];
  red[warp][1][g][2 * t + 1] = d1[1];
  red[warp][1][g + 8][2 * t] = d1[2];
  red[warp][1][g + 8][2 * t + 1] = d1[3];
  __syncthreads();
  const int tid = threadIdx.x;
  if (tid >= 128) return;
  const int r = tid >> 3, tb = tid & 7, row = tok0 + tb;  // (row of both tiles, token)
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int v = 0; v < kGemvWarps; ++v) {
    s0 += red[v][0][r][tb];
    s1 += red[v][1][r][tb];
  }
  if (row >= B) return;
  if (mode == 1) {
    y_out[(size_t)row * N + n0 + r] = float_to_bf16_bits(s0);
    y_out[(size_t)row * N + n1 + r] = float_to_bf16_bits(s1);
    return;
  }
  const int d = H * dh, half = dh >> 1;
  const int hb = n0 / dh, i = n0 - hb * dh + r;  // element i of the first half of head block hb
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

// ---------------------------------------------------------------------------
// Loop 1, dense: block (range, b) walks columns [range*R, ...) of sequence b
// for all heads, in chunks of kChunkCols columns, keeping an online softmax
// per head (running max and sum in shared memory, N in registers).  Every
// chunk streams its K stages (scores), then its V stages (weighted sums);
// stages are [kStageCols, H*dh] code rows plus [kStageCols, H*dh/32] scales,
// brought in by bulk copies into a kStages-deep ring.
// Warp roles: warp kDenseConsumers issues the copies (one lane), waiting on
// a stage's `empty` barrier (one arrival per consumer warp) before reusing
// it; the consumer warps wait on its `full` barrier (one lane polls).
// Scores: thread (column, head, group of 32) with the group's 32 q values in
// registers.  Weighted sums: thread owns EPT consecutive outputs of N
// (EPT = H*dh/256).  The consumers meet at a named barrier twice per chunk
// (around the softmax step between its K and V stages).
// ---------------------------------------------------------------------------
constexpr int kDenseConsumers = 8;
constexpr int kDenseThreads = 32 * (kDenseConsumers + 1);
constexpr int kConsumerBar = 1;  // named barrier of the consumer warps

template <int DH, int EPT>
__global__ void __launch_bounds__(kDenseThreads, 2) decode_dense_kernel(DecodeArgs a) {
  constexpr int G = DH / 32;
  constexpr int kConsumerThreads = 32 * kDenseConsumers;
  const int H = a.H, HG = H * G;
  const int RB = H * DH;      // code bytes per column
  const int SB = HG * 2;      // scale bytes per column
  const int stage_bytes = kStageCols * (RB + SB);
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);  // [kStages]
  uint64_t* empty = full + kStages;                    // [kStages]
  uint8_t* ring = smem + 128;
  float* sc = reinterpret_cast<float*>(ring + (size_t)kStages * stage_bytes);  // [H][kScRow]
  float* run_m = sc + H * kScRow;       // [H]
  float* run_z = run_m + H;             // [H]
  float* alpha = run_z + H;             // [H]
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.y;
  const int c_begin = blockIdx.x * a.range;
  const int c_end = min(a.P1, c_begin + a.range);
  const int ncols = max(0, c_end - c_begin);
  const int nchunks = (ncols + kChunkCols - 1) / kChunkCols;
  int total = 0;
  for (int ch = 0; ch < nchunks; ++ch) {
    const int n = min(kChunkCols, ncols - ch * kChunkCols);
    total += 2 * ((n + kStageCols - 1) / kStageCols);
  }

  if (tid == 0) {
    s_abort = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDenseConsumers);
    }
    fence_mbar_init();
  }
  for (int h = tid; h < H; h += kDenseThreads) {
    run_m[h] = -INFINITY;
    run_z[h] = 0.f;
  }
  __syncthreads();

  if (warp == kDenseConsumers) {
    // ---------------- producer: one lane issues every stage's copies
    if (lane != 0) return;
    int s = 0;
    for (int ch = 0; ch < nchunks && !s_abort; ++ch) {
      const int chunk0 = c_begin + ch * kChunkCols;
      const int n = min(kChunkCols, ncols - ch * kChunkCols);
      const int ns = (n + kStageCols - 1) / kStageCols;
      for (int isv = 0; isv < 2 && !s_abort; ++isv) {
        for (int st = 0; st < ns; ++st, ++s) {
          const int buf = s % kStages;
          if (s >= kStages && !mbar_wait_sleep(&empty[buf], ((s / kStages) - 1) & 1)) {
            set_error(a.err, kDevErrTimeout);
            s_abort = 1;
            break;
          }
          const int col0 = chunk0 + st * kStageCols;
          const int nc = min(kStageCols, chunk0 + n - col0);
          const int n_ctx = max(0, min(nc, a.S - col0));
          const bool has_tok = col0 + nc > a.S;
          uint8_t* dst = ring + (size_t)buf * stage_bytes;
          const KVStreams& cs = isv ? a.cv : a.ck;
          const KVStreams& ts = isv ? a.tv : a.tk;
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(&full[buf], (uint32_t)(n_ctx + (has_tok ? 1 : 0)) * (RB + SB));
          if (n_ctx > 0) {
            const size_t row = (size_t)b * a.S + col0;
            bulk_load(dst, cs.base_codes + row * RB, (uint32_t)(n_ctx * RB), &full[buf]);
            bulk_load(dst + kStageCols * RB, reinterpret_cast<const uint8_t*>(cs.base_scales) + row * SB,
                      (uint32_t)(n_ctx * SB), &full[buf]);
          }
          if (has_tok) {
            const int jt = a.S - col0;
            bulk_load(dst + (size_t)jt * RB, ts.base_codes + (size_t)b * RB, (uint32_t)RB, &full[buf]);
            bulk_load(dst + kStageCols * RB + (size_t)jt * SB,
                      reinterpret_cast<const uint8_t*>(ts.base_scales) + (size_t)b * SB, (uint32_t)SB, &full[buf]);
          }
        }
      }
    }
    // copies still in flight land before the block can exit: the consumers
    // wait for every stage, or, after an abort, this lane waits here
    if (s_abort)
      for (int t = max(0, s - kStages); t < s; ++t) mbar_wait_sleep(&full[t % kStages], (t / kStages) & 1);
    return;
  }

  // ---------------- consumers
  // score role: (column-in-pass, head, group)
  const int hg = tid % HG, jsub = tid / HG;
  const int cpp = kConsumerThreads / HG;  // columns per pass
  const int sh = hg / G;
  // q of this thread's (head, group) as three int8 digits per element, so
  // that q . codes is three integer dot products (dp4a):
  //   q_k = 2^(E-21) (d2 2^16 + d1 2^8 + d0),  E = exponent of max |q_k|,
  // exact for every element within 2^14 of the group's largest.
  int qd[3][8];
  float qsc;  // 2^(E-21) log2(e)/sqrt(dh)
  {
    float q[32];
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
    float mx = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) mx = fmaxf(mx, fabsf(q[e]));
    const int E = mx > 0.f ? ilogbf(mx) : 0;
    const float up = ldexpf(1.f, 21 - E);
#pragma unroll
    for (int v = 0; v < 8; ++v) qd[0][v] = qd[1][v] = qd[2][v] = 0;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int Q = __float2int_rn(q[e] * up);  // |Q| < 2^22
      const int c0 = ((Q + 128) & 255) - 128;
      const int Q1 = (Q - c0) >> 8;
      const int c1 = ((Q1 + 128) & 255) - 128;
      const int c2 = (Q1 - c1) >> 8;
      const int sh8 = (e & 3) * 8;
      qd[0][e >> 2] |= (c0 & 255) << sh8;
      qd[1][e >> 2] |= (c1 & 255) << sh8;
      qd[2][e >> 2] |= (c2 & 255) << sh8;
    }
    qsc = ldexpf(a.kscale, E - 21);
  }
  // the two 16-byte halves of a lane's 32 codes: lanes of alternate 128-byte
  // windows read them in opposite order, so each load spreads over all banks
  const bool swap = (lane >> 2) & 1;
  // weighted-sum role: outputs [o, o + EPT) of head oh
  const int o = tid * EPT, oh = o / DH;
  float acc[EPT];
#pragma unroll
  for (int e = 0; e < EPT; ++e) acc[e] = 0.f;

  int s = 0;  // stage sequence number
  for (int ch = 0; ch < nchunks; ++ch) {
    const int chunk0 = c_begin + ch * kChunkCols;
    const int n = min(kChunkCols, ncols - ch * kChunkCols);
    const int ns = (n + kStageCols - 1) / kStageCols;
    for (int phase = 0; phase < 2; ++phase) {
      for (int st = 0; st < ns; ++st, ++s) {
        const int buf = s % kStages;
        int ok = 0;
        if (lane == 0 && !s_abort) {
          ok = mbar_wait_sleep(&full[buf], (s / kStages) & 1) ? 1 : 0;
          if (!ok) {
            set_error(a.err, kDevErrTimeout);
            s_abort = 1;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        const uint8_t* sb = ring + (size_t)buf * stage_bytes;
        const uint16_t* scl = reinterpret_cast<const uint16_t*>(sb + kStageCols * RB);
        const int nv = min(kStageCols, n - st * kStageCols);
        if (ok) {
          if (phase == 0) {
            for (int p0 = 0; p0 < kStageCols; p0 += cpp) {  // the same trip count in every lane
              const int jj = p0 + jsub;
              float part = 0.f;
              if (jj < nv) {
                const uint8_t* row = sb + (size_t)jj * RB + hg * 32;
                const uint4 ca = *reinterpret_cast<const uint4*>(row + (swap ? 16 : 0));
                const uint4 cb = *reinterpret_cast<const uint4*>(row + (swap ? 0 : 16));
                const uint4 c0 = swap ? cb : ca, c1 = swap ? ca : cb;
                const int cw[8] = {(int)c0.x, (int)c0.y, (int)c0.z, (int)c0.w,
                                   (int)c1.x, (int)c1.y, (int)c1.z, (int)c1.w};
                int D0 = 0, D1 = 0, D2 = 0;
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                  D0 = __dp4a(cw[v], qd[0][v], D0);
                  D1 = __dp4a(cw[v], qd[1][v], D1);
                  D2 = __dp4a(cw[v], qd[2][v], D2);
                }
                // |D0 + 256 D1| < 2^27: exact in int32; the 2^16 digit joins in float
                const float dot = fmaf(static_cast<float>(D2), 65536.f, static_cast<float>(D0 + D1 * 256));
                part = dot * half_bits_f(scl[jj * HG + hg]) * qsc;  // qsc differs per group
              }
#pragma unroll
              for (int off = 1; off < G; off <<= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
              if (jj < nv && (hg % G) == 0) sc[sh * kScRow + st * kStageCols + jj] = part;
            }
          } else {
            const float* wrow = sc + oh * kScRow + st * kStageCols;
#pragma unroll
            for (int jj = 0; jj < kStageCols; ++jj) {
              if (jj < nv) {
                const float f = wrow[jj] * half_bits_f(scl[jj * HG + o / 32]);
                const uint8_t* src = sb + (size_t)jj * RB + o;
                if constexpr (EPT == 8) {
                  const uint2 w2 = *reinterpret_cast<const uint2*>(src);
                  const uint32_t uu[2] = {w2.x ^ 0x80808080u, w2.y ^ 0x80808080u};
#pragma unroll
                  for (int v = 0; v < 2; ++v)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[4 * v + e] = fmaf(f, i8_at(uu[v], e), acc[4 * v + e]);
                } else if constexpr (EPT >= 4) {
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
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[buf]);
      }
      if (phase == 0) {
        // online softmax over this chunk: new running max, rescale factor,
        // weights in place of the scores, raw scores kept for the selection
        named_bar_sync(kConsumerBar, kConsumerThreads);
        for (int h = warp; h < H; h += kDenseConsumers) {
          float mx = -INFINITY;
          for (int jc = lane; jc < n; jc += 32) mx = fmaxf(mx, sc[h * kScRow + jc]);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
          const float m_new = fmaxf(run_m[h], mx);
          float z = 0.f;
          float* srow = a.scores + ((size_t)b * H + h) * a.P1 + chunk0;
          for (int jc = lane; jc < n; jc += 32) {
            const float sv = sc[h * kScRow + jc];
            srow[jc] = sv;
            const float e = ex2(sv - m_new);
            sc[h * kScRow + jc] = e;
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
        named_bar_sync(kConsumerBar, kConsumerThreads);
        const float al = alpha[oh];
#pragma unroll
        for (int e = 0; e < EPT; ++e) acc[e] *= al;
      } else {
        // the next chunk's scores overwrite sc: every warp is done with its weights
        named_bar_sync(kConsumerBar, kConsumerThreads);
      }
    }
  }
  // partials of this range
  const size_t pr = (size_t)b * a.nsplit + blockIdx.x;
  for (int h = tid; h < H; h += kConsumerThreads) {
    a.part_m[pr * H + h] = run_m[h];
    a.part_Z[pr * H + h] = run_z[h];
  }
#pragma unroll
  for (int e = 0; e < EPT; ++e) a.part_N[pr * RB + o + e] = acc[e];
}

// Combine the ranges of each (sequence, head): state slot 0 and O.  (The
// loop-1 probabilities are made from the kept scores by the selection.)
template <int DH>
__global__ void __launch_bounds__(kThreads) decode_dense_merge_kernel(DecodeArgs a, float* m_out, float* z_out,
                                                                      float* n_out, uint16_t* o_out) {
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
}

// ---------------------------------------------------------------------------
// Loop r >= 2, sparse: block (range, b*H + h) takes kSparseCols of the
// selected columns.  The block first resolves every column's rows (base row
// and the residual row of each loop 2..r, or the token's rows) into shared
// memory.  The columns' K and V bytes of every stream are then gathered by
// cp.async into a ring of kSparseStages stages of kSparseStageCols columns
// (8 threads per column), so that several stages are in flight while one is
// used.  From a stage, 8 lanes per column (DH/8 elements each) rebuild
// Khat^(r-1), Khat^(r), Vhat^(r-1), Vhat^(r) and fold
// e_new Vhat^(r) - e_old Vhat^(r-1) into an online sum with a running
// reference max per column group.
// The selection is fixed after loop 1, so loop r keeps the selected columns'
// Khat^(r), Vhat^(r) (fp16) for loop r+1: loop 2 rebuilds Khat^(1) from the
// INT8 base, and loop r >= 3 starts from the kept Khat^(r-1) and adds only
// its own residual stream (two streams instead of r).
// ---------------------------------------------------------------------------
// acc[e] += code(e) * s for E8 consecutive BITS-bit two's-complement codes
// held in little-endian words w.
// The sign bit of every field is flipped first (c + 2^(BITS-1), unsigned);
// the field then lands in the mantissa of 2^23 and 2^23 + 2^(BITS-1) comes
// off again: the exact code as a float, with no int-to-float conversion.
template <int E8, int BITS, int NW>
__device__ __forceinline__ void add_codes(const uint32_t (&w)[NW], float s, float (&acc)[E8]) {
  constexpr int PW = 32 / BITS;
  constexpr uint32_t kSign = BITS == 8 ? 0x80808080u : BITS == 4 ? 0x88888888u : 0xAAAAAAAAu;
  constexpr float kBias = 8388608.0f + (1 << (BITS - 1));
  uint32_t u[NW];
#pragma unroll
  for (int v = 0; v < NW; ++v) u[v] = w[v] ^ kSign;
#pragma unroll
  for (int e = 0; e < E8; ++e) {
    const uint32_t f = ((u[e / PW] >> ((e % PW) * BITS)) & ((1u << BITS) - 1u)) | 0x4B000000u;
    acc[e] = fmaf(__uint_as_float(f) - kBias, s, acc[e]);
  }
}

__device__ __forceinline__ void cp_async8(void* smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(smem_u32(smem)), "l"(gmem));
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(smem)), "l"(gmem));
}

// Shared-memory layout of one gather stage of kSparseStageCols columns:
// K and V codes of every stream (base, then loop 2..LOOP residuals), then the
// K and V scales of every stream.  Offsets depend on the loops' code widths.
// Streams of a loop: LOOP 2 the INT8 base and the loop-2 residual; LOOP >= 3
// the kept fp16 Khat^(LOOP-1) / Vhat^(LOOP-1) (stream 0, no scale) and the
// loop's residual (stream 1).
template <int DH, int LOOP>
struct SparseStage {
  static constexpr bool PART = LOOP >= 3;
  static constexpr int NS = PART ? 2 : LOOP;
  static constexpr int G = DH / 32;
  int rb[NS];               // bytes of one column in stream l
  int off_k[NS], off_v[NS];
  int off_ks, off_vs, bytes;
  __host__ __device__ SparseStage(const int* bits) {
    int off = 0;
#pragma unroll
    for (int l = 0; l < NS; ++l) {
      rb[l] = l == 0 ? (PART ? 2 * DH : DH) : DH * bits[PART ? LOOP - 1 : l] / 8;
      off_k[l] = off;
      off += kSparseStageCols * rb[l];
      off_v[l] = off;
      off += kSparseStageCols * rb[l];
    }
    off_ks = off;
    off += NS * kSparseStageCols * G * 2;
    off_vs = off;
    off += NS * kSparseStageCols * G * 2;
    bytes = off;
  }
};

// E8 fp16 values (this lane's slice) of a kept column row in a stage, as float.
template <int E8>
__device__ __forceinline__ void stage_part(const uint8_t* row, int e0, float (&x)[E8]) {
#pragma unroll
  for (int v = 0; v < E8 / 8; ++v) {
    const uint4 w = *reinterpret_cast<const uint4*>(row + e0 * 2 + v * 16);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ww[q]));
      x[8 * v + 2 * q] = f.x;
      x[8 * v + 2 * q + 1] = f.y;
    }
  }
}

// Store E8 values as fp16 (this lane's slice of a kept column row).
template <int E8>
__device__ __forceinline__ void store_part(uint16_t* dst, const float (&x)[E8]) {
#pragma unroll
  for (int v = 0; v < E8 / 8; ++v) {
    uint32_t ww[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __half2 hh = __floats2half2_rn(x[8 * v + 2 * q], x[8 * v + 2 * q + 1]);
      ww[q] = *reinterpret_cast<const uint32_t*>(&hh);
    }
    *reinterpret_cast<uint4*>(dst + v * 8) = make_uint4(ww[0], ww[1], ww[2], ww[3]);
  }
}

// E8 codes (this lane's slice, element e0 on) of one column of stream l in
// a stage, added times s to acc (l = 0: the INT8 base, assigned).
template <int E8>
__device__ __forceinline__ void stage_codes(const uint8_t* row, int bits, int e0, float s, float (&acc)[E8],
                                            bool assign) {
  const int nb = E8 * bits / 8;
  const uint8_t* src = row + (e0 * bits) / 8;
  uint32_t w[E8 / 4];
#pragma unroll
  for (int v = 0; v < E8 / 4; ++v) w[v] = 0u;
  if constexpr (E8 >= 16) {
    if (nb == 16) {
      const uint4 t = *reinterpret_cast<const uint4*>(src);
      w[0] = t.x; w[1] = t.y; w[2] = t.z; w[3] = t.w;
    }
  }
  if (nb == 16) {
  } else if (nb == 8) {
    const uint2 t = *reinterpret_cast<const uint2*>(src);
    w[0] = t.x; w[1] = t.y;
  } else if (nb == 4) {
    w[0] = *reinterpret_cast<const uint32_t*>(src);
  } else {
    w[0] = *reinterpret_cast<const uint16_t*>(src);
  }
  if (assign) {  // the base: INT8
#pragma unroll
    for (int v = 0; v < E8 / 4; ++v) {
      const uint32_t u = w[v] ^ 0x80808080u;
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[4 * v + e] = i8_at(u, e) * s;
    }
    return;
  }
  if (bits == 2) add_codes<E8, 2>(w, s, acc);
  else if (bits == 4) add_codes<E8, 4>(w, s, acc);
  else add_codes<E8, 8>(w, s, acc);
}

template <int DH, int LOOP>
__global__ void __launch_bounds__(kSparseThreads) decode_sparse_kernel(DecodeArgs a) {
  constexpr int E8 = DH / 8, G = DH / 32;
  using LS = SparseStage<DH, LOOP>;
  constexpr bool PART = LS::PART;
  constexpr int NS = LS::NS;
  const LS L(a.bits);
  extern __shared__ __align__(16) uint8_t sm[];
  int* srow = reinterpret_cast<int*>(sm + (size_t)kSparseStages * L.bytes);  // [LOOP][kSparseCols]
  uint8_t* stok = reinterpret_cast<uint8_t*>(srow + LOOP * kSparseCols);   // [kSparseCols]
  __shared__ float red[3][kSparseThreads / 32];
  __shared__ float nred[kSparseThreads / 32][DH];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int u = lane & 7, grp = warp * 4 + (lane >> 3);
  const int bh = blockIdx.y, b = bh / a.H, h = bh - b * a.H;
  const int c_begin = blockIdx.x * kSparseCols;
  const int n = max(0, min(kSparseCols, a.k - c_begin));
  const int e0 = u * E8;
  const int d = a.H * DH;

  // rows of every column: base row and the residual row of loops 2..LOOP
  const int32_t* cols = a.cols + (size_t)bh * a.k + c_begin;
  for (int i = tid; i < n; i += kSparseThreads) {
    int j = cols[i];
    if (j < 0 || j > a.S) {
      set_error(a.err, FLASHLOOP_DEVERR_INDEX);
      j = a.S;
    }
    const bool tok = j == a.S;
    const size_t t = (size_t)b * a.S + j;
    stok[i] = tok;
    if (PART) {  // the kept row (selection index) and the loop's residual row
      srow[i] = c_begin + i;
      srow[kSparseCols + i] = tok ? b : a.cslot[LOOP - 1][t];
    } else {
      srow[i] = tok ? b : (int)t;
#pragma unroll
      for (int l = 2; l <= LOOP; ++l) srow[(l - 1) * kSparseCols + i] = tok ? b : a.cslot[l - 1][t];
    }
  }
  __syncthreads();

  // gather of stage st: 8 threads per column
  const int nst = (n + kSparseStageCols - 1) / kSparseStageCols;
  auto issue = [&](int st) {
    const int c = st * kSparseStageCols + (tid >> 3);
    const int cu = tid & 7;
    if (c < n) {
      uint8_t* buf = sm + (size_t)(st % kSparseStages) * L.bytes;
      const int cl = tid >> 3;  // column within the stage
      const bool tok = stok[c];
#pragma unroll
      for (int kv = 0; kv < 2; ++kv) {
        const KVStreams& S = kv == 0 ? (tok ? a.tk : a.ck) : (tok ? a.tv : a.cv);
        const int* off = kv == 0 ? L.off_k : L.off_v;
#pragma unroll
        for (int l = 0; l < NS; ++l) {
          const int row = srow[l * kSparseCols + c];
          const int nch = L.rb[l] / 16;
          if (row < 0) continue;
          const uint8_t* src;
          if (PART && l == 0)  // the kept Khat / Vhat row of this selected column
            src = reinterpret_cast<const uint8_t*>(a.kv_part) + (((size_t)bh * a.k + row) * 2 + kv) * DH * 2;
          else
            src = (l == 0 ? reinterpret_cast<const uint8_t*>(S.base_codes) : S.res_codes[PART ? LOOP - 1 : l]) +
                  ((size_t)row * a.H + h) * L.rb[l];
          for (int ch = cu; ch < nch; ch += 8) cp_async16(buf + off[l] + cl * L.rb[l] + ch * 16, src + ch * 16, 16);
        }
      }
      // scales: 2*NS copies of G fp16 per column (the kept rows have none)
#pragma unroll
      for (int i = cu; i < 2 * NS; i += 8) {
        const int kv = i / NS, l = i - kv * NS;
        if (PART && l == 0) continue;
        const KVStreams& S = kv == 0 ? (tok ? a.tk : a.ck) : (tok ? a.tv : a.cv);
        const int row = srow[l * kSparseCols + c];
        uint8_t* dst = buf + (kv == 0 ? L.off_ks : L.off_vs) + ((size_t)l * kSparseStageCols + cl) * G * 2;
        if (row < 0) {  // no residual at this loop: scale 0 adds nothing
          if constexpr (G == 4) *reinterpret_cast<uint2*>(dst) = make_uint2(0u, 0u);
          else *reinterpret_cast<uint32_t*>(dst) = 0u;
        } else {
          const uint16_t* src =
              (l == 0 ? S.base_scales : S.res_scales[PART ? LOOP - 1 : l]) + ((size_t)row * a.H + h) * G;
          if constexpr (G == 4) cp_async8(dst, src);
          else cp_async4(dst, src);
        }
      }
    }
    cp_async_commit();
  };

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
#pragma unroll
  for (int st = 0; st < kSparseStages - 1; ++st) {
    if (st < nst) issue(st);
    else cp_async_commit();
  }

  float mu = -INFINITY, mxn = -INFINITY, zn = 0.f, zo = 0.f;
  float acc[E8];
#pragma unroll
  for (int e = 0; e < E8; ++e) acc[e] = 0.f;
  const int g = e0 / 32;
  for (int st = 0; st < nst; ++st) {
    cp_async_wait<kSparseStages - 2>();
    __syncthreads();  // stage st landed for every thread; stage st-1 is free
    if (st + kSparseStages - 1 < nst) issue(st + kSparseStages - 1);
    else cp_async_commit();
    const uint8_t* buf = sm + (size_t)(st % kSparseStages) * L.bytes;
    const int jl = st * kSparseStageCols + grp;
    const bool valid = jl < n;
    // K: Khat^(LOOP-1) and Khat^(LOOP) of this lane's slice
    float xo[E8], xn[E8];
    uint16_t* part_row = a.kv_part + ((size_t)bh * a.k + c_begin + jl) * 2 * DH + e0;
    {
      const uint16_t* ks = reinterpret_cast<const uint16_t*>(buf + L.off_ks);
      if (PART) {
        stage_part<E8>(buf + L.off_k[0] + grp * L.rb[0], e0, xo);
      } else {
        stage_codes<E8>(buf + L.off_k[0] + grp * L.rb[0], 8, e0, half_bits_f(ks[grp * G + g]), xo, true);
#pragma unroll
        for (int l = 1; l < LOOP - 1; ++l)
          stage_codes<E8>(buf + L.off_k[l] + grp * L.rb[l], a.bits[l], e0,
                          half_bits_f(ks[(l * kSparseStageCols + grp) * G + g]), xo, false);
      }
#pragma unroll
      for (int e = 0; e < E8; ++e) xn[e] = xo[e];
      stage_codes<E8>(buf + L.off_k[NS - 1] + grp * L.rb[NS - 1], a.bits[LOOP - 1], e0,
                      half_bits_f(ks[((NS - 1) * kSparseStageCols + grp) * G + g]), xn, false);
      if (a.write_part && valid) store_part<E8>(part_row, xn);
    }
    float dol = 0.f, dnw = 0.f;
#pragma unroll
    for (int e = 0; e < E8; ++e) {
      dol = fmaf(qo[e], xo[e], dol);
      dnw = fmaf(qn[e], xn[e], dnw);
    }
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
      dol += __shfl_xor_sync(0xffffffffu, dol, off);
      dnw += __shfl_xor_sync(0xffffffffu, dnw, off);
    }
    if (valid) {
      const float so = dol * a.kscale, sn = dnw * a.kscale;
      const float m_new = fmaxf(mu, fmaxf(so, sn));
      if (m_new > mu) {  // same decision in the column's 8 lanes
        const float rho = ex2(mu - m_new);  // 0 while mu is -inf
#pragma unroll
        for (int e = 0; e < E8; ++e) acc[e] *= rho;
        zn *= rho;
        zo *= rho;
        mu = m_new;
      }
      const float en = ex2(sn - mu), eo = ex2(so - mu);
      const uint16_t* vs = reinterpret_cast<const uint16_t*>(buf + L.off_vs);
      if (PART) {
        stage_part<E8>(buf + L.off_v[0] + grp * L.rb[0], e0, xo);
      } else {
        stage_codes<E8>(buf + L.off_v[0] + grp * L.rb[0], 8, e0, half_bits_f(vs[grp * G + g]), xo, true);
#pragma unroll
        for (int l = 1; l < LOOP - 1; ++l)
          stage_codes<E8>(buf + L.off_v[l] + grp * L.rb[l], a.bits[l], e0,
                          half_bits_f(vs[(l * kSparseStageCols + grp) * G + g]), xo, false);
      }
#pragma unroll
      for (int e = 0; e < E8; ++e) xn[e] = xo[e];
      stage_codes<E8>(buf + L.off_v[NS - 1] + grp * L.rb[NS - 1], a.bits[LOOP - 1], e0,
                      half_bits_f(vs[((NS - 1) * kSparseStageCols + grp) * G + g]), xn, false);
      if (a.write_part) store_part<E8>(part_row + DH, xn);
#pragma unroll
      for (int e = 0; e < E8; ++e) acc[e] = fmaf(en, xn[e], fmaf(-eo, xo[e], acc[e]));
      zn += en;
      zo += eo;
      mxn = fmaxf(mxn, sn);
    }
  }
  cp_async_wait<0>();
  // block reference: the largest group reference; every group rescales to it
  float mb = mu, mx = mxn;
#pragma unroll
  for (int off = 8; off < 32; off <<= 1) {
    mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, off));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  }
  if (lane == 0) {
    red[0][warp] = mb;
    red[1][warp] = mx;
  }
  __syncthreads();
  mb = red[0][0];
  mx = red[1][0];
#pragma unroll
  for (int w = 1; w < kSparseThreads / 32; ++w) {
    mb = fmaxf(mb, red[0][w]);
    mx = fmaxf(mx, red[1][w]);
  }
  __syncthreads();
  const float f = mu == -INFINITY ? 0.f : ex2(mu - mb);
#pragma unroll
  for (int e = 0; e < E8; ++e) {
    acc[e] *= f;
    acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 8);
    acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
  }
  float zd = (zn - zo) * f;  // identical in the 8 lanes of a group: count lane u == 0 only
  zd = u == 0 ? zd : 0.f;
#pragma unroll
  for (int off = 8; off < 32; off <<= 1) zd += __shfl_xor_sync(0xffffffffu, zd, off);
  if (lane < 8) {
#pragma unroll
    for (int e = 0; e < E8; ++e) nred[warp][e0 + e] = acc[e];
  }
  if (lane == 0) red[2][warp] = zd;
  __syncthreads();
  const size_t pi = (size_t)bh * gridDim.x + blockIdx.x;
  for (int e = tid; e < DH; e += kSparseThreads) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kSparseThreads / 32; ++w) v += nred[w][e];
    a.part_N[pi * DH + e] = v;
  }
  if (tid == 0) {
    float z = 0.f;
#pragma unroll
    for (int w = 0; w < kSparseThreads / 32; ++w) z += red[2][w];
    a.part_m[pi] = mx;
    a.part_mu[pi] = mb;
    a.part_Z[pi] = z;
  }
}

template <int DH, int LOOP>
static int launch_sparse_t(const DecodeArgs& a, dim3 grid, cudaStream_t stream) {
  const SparseStage<DH, LOOP> L(a.bits);
  const size_t smem = (size_t)kSparseStages * L.bytes + (size_t)LOOP * kSparseCols * 4 + kSparseCols;  // rows [LOOP][cols] (>= NS), tokens
  static size_t attr = 0;
  if (smem > attr) {
    FL_TRY(cudaFuncSetAttribute(decode_sparse_kernel<DH, LOOP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem));
    attr = smem;
  }
  decode_sparse_kernel<DH, LOOP><<<grid, kSparseThreads, smem, stream>>>(a);
  return launch_status();
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
  L.kv_part = off; off = align256(off + B * H * (size_t)k * 2 * dh * sizeof(uint16_t));
  L.total = off;
  return L;
}

size_t decode_dense_smem(const flashloop_params* p) {
  const int H = p->n_heads, RB = H * p->head_dim, SB = H * (p->head_dim / 32) * 2;
  return 128 + (size_t)kStages * kStageCols * (RB + SB) + ((size_t)H * kScRow + 3 * H) * sizeof(float);
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
  a.kv_part = ws_ptr<uint16_t>(ds->workspace, L.kv_part);
  a.write_part = loop >= 2 && loop < p->n_loops;
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
  decode_dense_kernel<DH, EPT><<<dim3(a.nsplit, a.B), kDenseThreads, smem, stream>>>(a);
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
                                                                     reinterpret_cast<uint16_t*>(ds->O));
    else
      decode_dense_merge_kernel<64><<<B * H, kThreads, 0, stream>>>(a, ds->m[0], ds->Z[0], ds->N[0],
                                                                    reinterpret_cast<uint16_t*>(ds->O));
    return launch_status();
  }
  const int si = slot_of_loop(loop - 1), so = slot_of_loop(loop);
  const dim3 grid(L.nblk, B * H);
  int rc = FLASHLOOP_ERR_UNSUPPORTED;
#define FL_SPARSE(D, LP) \
  if (dh == D && loop == LP) rc = launch_sparse_t<D, LP>(a, grid, stream);
  FL_SPARSE(128, 2) FL_SPARSE(128, 3) FL_SPARSE(128, 4) FL_SPARSE(128, 5) FL_SPARSE(128, 6)
  FL_SPARSE(128, 7) FL_SPARSE(128, 8)
  FL_SPARSE(64, 2) FL_SPARSE(64, 3) FL_SPARSE(64, 4) FL_SPARSE(64, 5) FL_SPARSE(64, 6)
  FL_SPARSE(64, 7) FL_SPARSE(64, 8)
#undef FL_SPARSE
  if (rc != FLASHLOOP_OK) return rc;
  if (dh == 128) {
    decode_sparse_merge_kernel<128><<<B * H, 128, 0, stream>>>(a, L.nblk, ds->m[si], ds->Z[si], ds->N[si], ds->m[so],
                                                               ds->Z[so], ds->N[so], reinterpret_cast<uint16_t*>(ds->O));
  } else {
    decode_sparse_merge_kernel<64><<<B * H, 64, 0, stream>>>(a, L.nblk, ds->m[si], ds->Z[si], ds->N[si], ds->m[so],
                                                             ds->Z[so], ds->N[so], reinterpret_cast<uint16_t*>(ds->O));
  }
  return launch_status();
}

// Selection of the decode token: per (sequence, head) the topk[1] columns of
// largest loop-1 probability, the same radix select as the prefill's, its
// keys made from the kept scores (and written to probs) as they are loaded.
int launch_decode_select(const flashloop_params* p, flashloop_decode_state* ds, cudaStream_t stream) {
  flashloop_params ps = *p;
  ps.n_heads = p->batch * p->n_heads;
  ps.seq = p->seq + 1;
  const DecodeLayout L = decode_layout(p);
  return launch_topk(&ps, ws_ptr<float>(ds->workspace, L.scores), nullptr, 0, p->topk[1], ds->cols, ds->err_word,
                     stream, ds->m[0], ds->Z[0], ds->probs);
}

int launch_decode_gemv(const flashloop_params* p, const uint16_t* x, const uint16_t* w, int mode,
                       const float* rope_cs, uint16_t* q_out, float* k_out, float* v_out, uint16_t* y_out,
                       cudaStream_t stream) {
  const int d = p->d_model, N = mode == 0 ? 3 * d : d;
  const dim3 grid(N / 32, (p->batch + 7) / 8);
  decode_gemv_kernel<<<grid, kGemvWarps * 32, 0, stream>>>(x, w, p->batch, d, N, p->head_dim, p->n_heads, mode,
                                                           rope_cs, q_out, k_out, v_out, y_out);
  return launch_status();
}

int launch_decode_qkv(const flashloop_params* p, int loop, const uint16_t* x_tok, const uint16_t* w_qkv,
                      flashloop_decode_state* ds, cudaStream_t stream) {
  const DecodeLayout L = decode_layout(p);
  float* k_new = ws_ptr<float>(ds->workspace, L.k_new);
  float* v_new = ws_ptr<float>(ds->workspace, L.v_new);
  int rc = launch_decode_gemv(p, x_tok, w_qkv, 0, ds->rope_cs,
                              reinterpret_cast<uint16_t*>(ds->q[slot_of_loop(loop)]), k_new, v_new, nullptr, stream);
  if (rc != FLASHLOOP_OK) return rc;
  return launch_kv_quant_rows(p->head_dim, loop, p->batch, p->n_heads, p->bits, k_new, v_new, ds->k, ds->v,
                              ds->err_word, stream);
}

int launch_decode_out(const flashloop_params* p, const uint16_t* w_o, flashloop_decode_state* ds,
                      cudaStream_t stream) {
  return launch_decode_gemv(p, reinterpret_cast<const uint16_t*>(ds->O), w_o, 1, nullptr, nullptr, nullptr,
                            nullptr, reinterpret_cast<uint16_t*>(ds->Y), stream);
}

}  // namespace fl
