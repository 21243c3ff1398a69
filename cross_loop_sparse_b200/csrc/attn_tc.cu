// (a6) Sparse attention update (and the dense loop-1 attention) on the
// sm_100a tensor cores: tcgen05.mma with Q, P and the running numerator in
// TMEM, K and V tiles streamed by TMA.
//
// [FlashLoop §3.2, §4.2, App. D.2]: for every active row i of loop r and
// selected column j <= i, the loop r-1 contribution of (i, j) is removed from
// the row's running state and the loop-r one added:
//   S_old = Q^(r-1) Khat^(r-1)^T / sqrt(dh),  S_new = Q^(r) Khat^(r)^T / sqrt(dh)
//   N' = a N + [e^(S_new - m') | -e^(S_old - m')] [Vhat^(r); Vhat^(r-1)]
//   Z' = a Z + sum e^(S_new - m') - sum e^(S_old - m')
// A block owns 128 active rows of one head at a time (persistent over
// (head, row-tile) work items) and walks the head's ascending selected columns
// in tiles of 64 up to its largest row token.
//
// TMEM (512 columns): Q_new | Q_old (fp16 pairs), N (f32, DH columns), two
// score buffers {S_new 64 | S_old 64}; P = [e_new | -e_old] (fp16 pairs) is
// written over the S_new half of its buffer and fed to the P.V MMA from TMEM.
// Roles: warps 0-7 hold two threads per row (TMEM lane), one per half of a
// tile, and do the masking, exponentials, running max and sums, the Q / N
// set-up and the write-back; warp 8 allocates TMEM and streams K (64 x DH)
// and V^T (DH x 64) tiles, new and old, by TMA into a ring of three stages;
// warp 9 issues S(t+1) while the rows process S(t), then P(t).V.
// The running maximum is a per-row reference raised only when a tile's
// maximum exceeds it by 8 (log2 units), which keeps every exponential
// <= 2^8 and represents the same (m, N, Z) state (N and Z are defined up to
// the common factor e^m).  All waits are bounded.
//
// Fixed-mass form [FlashLoop §4.2: the selection's probabilities are scaled
// to the mass the previous loop gave those columns]: the selected columns J of
// row i keep the probability mass M_i they had after loop r-1 and share it in
// proportion to e^(s_new).  With a per-row factor g (the weight of the
// selected columns relative to e^(s - m) / Z; g = 1 after the dense loop)
// that is N' = a N - g_prev sum_J e^(s_old - m') V_old + g sum_J e^(s_new - m') V_new,
// Z' = a Z, g = g_prev sum_J e^(s_old - m') / sum_J e^(s_new - m').  Two
// launches: a statistics pass (mode 1: S tiles and exponential sums only,
// no V, no N) fixes m' and g; the update pass (mode 2) then adds the
// contributions in that fixed frame, with no running maximum.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "attn_args.cuh"
#include "common.cuh"
#include "tc_util.cuh"

namespace fl {

constexpr int kAtRows = 128, kAtCols = 64, kAtStages = 3, kAtThreads = 320;
constexpr int kAtRowThreads = 256;  // warps 0-7: two threads per row, one per half of a tile
constexpr float kAtLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.f;

template <int DH>
struct AtCfg {
  static constexpr int kKBytes = kAtCols * DH * 2;  // K tile: 64 rows x DH (DH/64 swizzle chunks)
  static constexpr int kVBytes = DH * kAtCols * 2;  // V^T tile: DH rows x 64
  static constexpr int kStageBytes = 2 * kKBytes + 2 * kVBytes;
  static constexpr int kSmem = 1024 + kAtStages * kStageBytes + 512 + 8 * 128 * 4;
  static constexpr uint32_t kColQn = 0;
  static constexpr uint32_t kColQo = DH / 2;
  static constexpr uint32_t kColN = DH;
  static constexpr uint32_t kColS = 2 * DH;  // buffer b: S_new at kColS + 128 b, S_old at +64
  static constexpr uint32_t kIdescS = f16_idesc(128, kAtCols, 0);
  static constexpr uint32_t kIdescPV = f16_idesc(128, DH, 0);
};

enum AtMode { kAtRunning = 0, kAtFixedMassStats = 1, kAtFixedMassUpdate = 2 };

struct AtArgs {
  int S, H, kc, dense;
  const float* g_in;     // [H, S] selected-column factor of loop r-1 (fixed-mass modes)
  float* g_out;          // [H, S] written by mode 1 (and set to 1 by the dense loop)
  const int32_t* rows;
  const int32_t* n_rows;
  int row_cap;
  const int32_t* cols;   // [H, kc] ascending (NULL: identity)
  const uint16_t* q_new; // bf16 [S, H*DH]
  const uint16_t* q_old;
  const float* m_in;
  const float* z_in;
  const float* n_in;
  float* m_out;
  float* z_out;
  float* n_out;
  uint16_t* o;
  float scale_log2;
  int32_t* err;
  const int32_t* row_cnt;  // [H, row_cap] selected columns <= the row's token (with cols; NULL when dense)
};

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];\n" ::"l"(p));
}

// Selected columns at or before active row a's token, for head h: from the
// precomputed counts, or the identity selection (dense).
__device__ __forceinline__ int at_row_count(const AtArgs& g, int h, int a, int tok) {
  if (g.row_cnt) return __ldg(g.row_cnt + (size_t)h * g.row_cap + a);
  return min(tok + 1, g.kc);
}

// Number of column tiles work item (h, rt) needs: columns up to its last row token.
__device__ __forceinline__ int at_tiles(const AtArgs& g, int h, int rt, int n_rows) {
  int last = min(n_rows, (rt + 1) * kAtRows) - 1;
  int tok = g.rows ? __ldg(g.rows + last) : last;
  if (tok < 0) return 0;
  if (tok >= g.S) tok = g.S - 1;
  return (at_row_count(g, h, last, tok) + kAtCols - 1) / kAtCols;
}

// Barriers and the abort flag shared by a block's roles.
struct AtBars {
  uint64_t* kv_full;   // [stages]
  uint64_t* kv_empty;  // [stages]
  uint64_t* s_full;    // [2]
  uint64_t* p_full;    // [2]
  uint64_t* pv_done;   // [2]
  uint64_t* q_ready;   // [1]
  volatile int* abort_flag;
};

// Load role (one thread): the K (64 x DH) and V^T (DH x 64) tiles, new and
// old, of every work item into the ring of stages by TMA.
template <int DH, int MODE>
__device__ __forceinline__ void at_load_role(uint8_t* smem, const AtBars& B, const CUtensorMap* tkn,
                                             const CUtensorMap* tko, const CUtensorMap* tvn, const CUtensorMap* tvo,
                                             const AtArgs& g, int n_rows, int row_tiles, int total, bool has_old,
                                             int lane) {
  using C = AtCfg<DH>;
  if (lane == 0) {
    int stage = 0;
    uint32_t phase = 0;
    constexpr bool load_v = MODE != kAtFixedMassStats;
    const uint32_t bytes = (has_old ? 2 : 1) * (C::kKBytes + (load_v ? C::kVBytes : 0));
    int issued[kAtStages];
    for (int s2 = 0; s2 < kAtStages; ++s2) issued[s2] = -1;
    for (int item = blockIdx.x; item < total && !*B.abort_flag; item += gridDim.x) {
      const int h = item / row_tiles, rt = item % row_tiles;
      const int nt = at_tiles(g, h, rt, n_rows);
      for (int t = 0; t < nt && !*B.abort_flag; ++t) {
        if (!mbar_wait_sleep(&B.kv_empty[stage], phase ^ 1)) {
          set_error(g.err, kDevErrTimeout);
          *B.abort_flag = 1;
          break;
        }
        uint8_t* st = smem + stage * C::kStageBytes;
        mbar_arrive_expect_tx(&B.kv_full[stage], bytes);
#pragma unroll
        for (int c = 0; c < DH / 64; ++c)
          tma_load_3d(st + c * (kAtCols * 128), tkn, c * 64, t * kAtCols, h, &B.kv_full[stage]);
        if (load_v) tma_load_3d(st + 2 * C::kKBytes, tvn, t * kAtCols, 0, h, &B.kv_full[stage]);
        if (has_old) {
#pragma unroll
          for (int c = 0; c < DH / 64; ++c)
            tma_load_3d(st + C::kKBytes + c * (kAtCols * 128), tko, c * 64, t * kAtCols, h, &B.kv_full[stage]);
          if (load_v) tma_load_3d(st + 2 * C::kKBytes + C::kVBytes, tvo, t * kAtCols, 0, h, &B.kv_full[stage]);
        }
        issued[stage] = phase;
        if (++stage == kAtStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    // never leave with a copy in flight: wait (bounded) for the last load of every stage
    for (int s2 = 0; s2 < kAtStages; ++s2)
      if (issued[s2] >= 0) (void)mbar_wait(&B.kv_full[s2], (uint32_t)issued[s2]);
  }
}

// MMA role (one thread): S(t) = [Q_new K_new^T | Q_old K_old^T] into score
// buffer t & 1 while the rows process S(t-1), then P(t-1).V into N.
template <int DH, int MODE>
__device__ __forceinline__ void at_mma_role(uint8_t* smem, const AtBars& B, uint32_t tmem, const AtArgs& g,
                                            int n_rows, int row_tiles, int total, bool has_old, int lane) {
  using C = AtCfg<DH>;
  if (lane == 0) {
    int stage = 0;
    uint32_t phase = 0;
    uint32_t u = 0;        // global tile counter (S buffer = u & 1)
    uint32_t item_no = 0;  // items with tiles so far
    bool ok = true;
    for (int item = blockIdx.x; item < total && ok && !*B.abort_flag; item += gridDim.x) {
      const int h = item / row_tiles, rt = item % row_tiles;
      const int nt = at_tiles(g, h, rt, n_rows);
      if (nt == 0) continue;  // the rows signal q_ready only for items with tiles
      if (!mbar_wait_sleep(B.q_ready, item_no & 1)) {
        set_error(g.err, kDevErrTimeout);
        *B.abort_flag = 1;
        break;
      }
      ++item_no;
      tc_fence_after();
      int prev_stage = -1;
      for (int t = 0; t <= nt; ++t) {
        if (t < nt) {
          // S(t) into buffer u & 1
          if (!mbar_wait_sleep(&B.kv_full[stage], phase)) {
            set_error(g.err, kDevErrTimeout);
            *B.abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sb = tmem + C::kColS + (u & 1) * 128;
          const uint32_t k_addr = smem_u32(smem + stage * C::kStageBytes);
#pragma unroll
          for (int ks = 0; ks < DH / 16; ++ks) {
            const uint32_t kd = k_addr + (ks >> 2) * (kAtCols * 128) + (ks & 3) * 32;
            umma_f16_ts(sb, tmem + C::kColQn + ks * 8, sw128_kmajor_desc(kd), C::kIdescS, ks > 0);
            if (has_old)
              umma_f16_ts(sb + 64, tmem + C::kColQo + ks * 8, sw128_kmajor_desc(kd + C::kKBytes), C::kIdescS,
                          ks > 0);
          }
          umma_commit(&B.s_full[u & 1]);
        }
        if (t > 0) {
          // P(t-1).V into N
          const uint32_t up = u - 1;
          if (!mbar_wait_sleep(&B.p_full[up & 1], (up >> 1) & 1)) {
            set_error(g.err, kDevErrTimeout);
            *B.abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          if (MODE != kAtFixedMassStats) {  // the statistics pass has no P.V
            const uint32_t pcol = tmem + C::kColS + (up & 1) * 128;
            const uint32_t v_addr = smem_u32(smem + prev_stage * C::kStageBytes + 2 * C::kKBytes);
#pragma unroll
            for (int ks = 0; ks < kAtCols / 16; ++ks)
              umma_f16_ts(tmem + C::kColN, pcol + ks * 8, sw128_kmajor_desc(v_addr + ks * 32), C::kIdescPV, 1u);
            if (has_old) {
#pragma unroll
              for (int ks = 0; ks < kAtCols / 16; ++ks)
                umma_f16_ts(tmem + C::kColN, pcol + 32 + ks * 8, sw128_kmajor_desc(v_addr + C::kVBytes + ks * 32),
                            C::kIdescPV, 1u);
            }
          }
          umma_commit(&B.kv_empty[prev_stage]);
          umma_commit(&B.pv_done[up & 1]);
        }
        if (t < nt) {
          prev_stage = stage;
          if (++stage == kAtStages) {
            stage = 0;
            phase ^= 1;
          }
          ++u;
        }
      }
    }
  }
}

template <int DH, int MODE>
__global__ void __launch_bounds__(kAtThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_kn, const __grid_constant__ CUtensorMap tm_ko,
               const __grid_constant__ CUtensorMap tm_vn, const __grid_constant__ CUtensorMap tm_vo, AtArgs g) {
  using C = AtCfg<DH>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kAtStages * C::kStageBytes);
  uint64_t* kv_full = bars;                    // [stages]
  uint64_t* kv_empty = bars + kAtStages;       // [stages]
  uint64_t* s_full = bars + 2 * kAtStages;     // [2]
  uint64_t* p_full = s_full + 2;               // [2]
  uint64_t* pv_done = p_full + 2;              // [2]
  uint64_t* q_ready = pv_done + 2;             // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_ready + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool has_old = !g.dense;
  int n_rows = g.n_rows ? *g.n_rows : g.S;
  if (n_rows > g.row_cap) n_rows = g.row_cap;
  if (n_rows < 0) n_rows = 0;
  const int row_tiles = (n_rows + kAtRows - 1) / kAtRows;
  const int total = row_tiles * g.H;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kAtStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], kAtRowThreads);
      mbar_init(&pv_done[b], 1);
    }
    mbar_init(q_ready, kAtRowThreads);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const AtBars B{kv_full, kv_empty, s_full, p_full, pv_done, q_ready, abort_flag};
  if (warp == 8) {
    at_load_role<DH, MODE>(smem, B, &tm_kn, &tm_ko, &tm_vn, &tm_vo, g, n_rows, row_tiles, total, has_old, lane);
  } else if (warp == 9) {
    at_mma_role<DH, MODE>(smem, B, tmem, g, n_rows, row_tiles, total, has_old, lane);
  } else {
    // ------------------------------------------------------------ rows
    // Two threads per row: half 0 takes columns [0, 32) of each tile (and
    // Q_new / the first half of N), half 1 columns [32, 64) (and Q_old / the
    // second half of N).  The two warps of a row pair exchange tile maxima and
    // sums through shared memory at a named barrier.  A named barrier cannot
    // time out, so both warps always execute the same barrier sequence: after
    // a failed wait (or an abort raised elsewhere) a warp turns "dead" - it
    // skips waits, tensor-memory work and writes but keeps the control flow.
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int pair_bar = 1 + quarter;
    float* xchg = reinterpret_cast<float*>(tmem_slot + 4);  // [2 parities][2 halves][128] maxima, [2][128] sums, [2][128] old sums
    constexpr bool stats = MODE == kAtFixedMassStats;     // fixed-mass statistics pass
    constexpr bool fixed = MODE == kAtFixedMassUpdate;    // fixed-mass update pass
    const int HD = g.H * DH;
    constexpr int kHalfCols = DH / 2;
    bool dead = false;
    auto wait_or_die = [&](uint64_t* bar, uint32_t parity) {
      if (!dead && __any_sync(0xffffffffu, *abort_flag != 0)) dead = true;
      if (dead) return;
      if (!__all_sync(0xffffffffu, mbar_wait_sleep(bar, parity))) {
        set_error(g.err, kDevErrTimeout);
        *abort_flag = 1;
        dead = true;
        return;
      }
      tc_fence_after();
    };
    uint32_t u = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
      const int h = item / row_tiles, rt = item % row_tiles;
      const int nt = at_tiles(g, h, rt, n_rows);
      const int a = rt * kAtRows + row;
      int tok = -1;
      if (a < n_rows) {
        tok = g.rows ? __ldg(g.rows + a) : a;
        if (tok < 0 || tok >= g.S) {
          if (half == 0) set_error(g.err, FLASHLOOP_DEVERR_INDEX);
          tok = -1;
        }
      }
      // Per-row frame.  Running state (mode 0) and statistics pass: the
      // reference starts at the previous maximum and is raised lazily.  Update
      // pass: the frame is the statistics pass's reference, lifted by log2 of
      // the larger g so that the scaled exponentials stay <= 2^8; N_in and Z_in
      // are brought into it by a = 2^(m_in - m_ref).
      float m_ref = 0.f, z = 0.f, z_old = 0.f, alpha = 1.f, g_prev = 1.f;
      float off_new = 0.f, off_old = 0.f;  // update pass: exponent offsets m_ref - log2 g
      if (tok >= 0) {
        const size_t hi = (size_t)h * g.S + tok;
        m_ref = g.dense ? -INFINITY : g.m_in[hi] * kAtLog2e;
        if (MODE == kAtRunning) {
          if (!g.dense && half == 0) z = g.z_in[hi];
        } else {
          g_prev = g.g_in[hi];
          if (fixed) {
            const float g_new = g.g_out[hi];
            const float lift = fmaxf(0.f, log2f(fmaxf(g_prev, g_new)));
            const float m_in = m_ref;
            m_ref = g.m_out[hi] * kAtLog2e + lift;
            alpha = ex2(m_in - m_ref);
            off_new = m_ref - log2f(g_new);   // g = 0 gives +inf: exponentials of 0
            off_old = m_ref - log2f(g_prev);
            if (half == 0) z = alpha * g.z_in[hi];
          }
        }
      }
      // Q (fp16 pairs, exact from bf16) and this half of N into TMEM.  The
      // rebuilt keys carry the factor log2(e)/sqrt(dh), so S is in log2 units.
      if (!dead) {
        const uint16_t* qsrc = half == 0 ? g.q_new : g.q_old;
        const bool load_q = tok >= 0 && (half == 0 || has_old);
        const bool load_n = !g.dense && tok >= 0 && !stats;
        const uint32_t qcol = half == 0 ? C::kColQn : C::kColQo;
        // 32-byte accesses: one full sector per thread and instruction
        uint32_t qv[DH / 16][8];
#pragma unroll
        for (int v = 0; v < DH / 16; ++v) {
          if (load_q) {
            ld_global_v8(qsrc + (size_t)tok * HD + (size_t)h * DH + v * 16, qv[v]);
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) qv[v][e] = 0u;
          }
        }
        bool q_ok = true;  // q must fit fp16, the MMA operand type
#pragma unroll
        for (int c0 = 0; c0 < DH; c0 += 32) {
          uint32_t r[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 f = bf16x2_to_float2(qv[c0 / 16 + e / 8][e % 8]);
            q_ok = q_ok && half_range_ok(f.x) && half_range_ok(f.y);
            r[e] = bf16x2_to_half2_bits(qv[c0 / 16 + e / 8][e % 8]);
          }
          __syncwarp();
          tmem_st16(tmem + lane_base + qcol + c0 / 2, r);
        }
        if (!q_ok) set_error(g.err, FLASHLOOP_DEVERR_RANGE);
        uint32_t nv[kHalfCols / 8][8];
#pragma unroll
        for (int v = 0; v < kHalfCols / 8; ++v) {
          if (load_n) {
            ld_global_v8(g.n_in + ((size_t)h * g.S + tok) * DH + half * kHalfCols + 8 * v, nv[v]);
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) nv[v][e] = 0u;
          }
        }
#pragma unroll
        for (int c0 = 0; c0 < kHalfCols; c0 += 16) {
          uint32_t r[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(nv[c0 / 8 + e / 8][e % 8]) * alpha);
          __syncwarp();
          tmem_st16(tmem + lane_base + C::kColN + half * kHalfCols + c0, r);
        }
        tmem_wait_st();
        tc_fence_before();
        // only items with tiles: the MMA thread waits on q_ready for those
        // alone, so the rows can never run two phases ahead of it
        if (nt > 0) mbar_arrive(q_ready);
        // bring the next item's rows (this thread's q and half of N) into L2
        // while this item runs: they are the item switch's loads
        const int item_next = item + gridDim.x;
        if (item_next < total) {
          const int hn = item_next / row_tiles, an = (item_next % row_tiles) * kAtRows + row;
          const int tn = an < n_rows ? (g.rows ? __ldg(g.rows + an) : an) : -1;
          if (tn >= 0 && tn < g.S) {
            if (half == 0 || has_old) {
              const uint16_t* qn = (half == 0 ? g.q_new : g.q_old) + (size_t)tn * HD + (size_t)hn * DH;
#pragma unroll
              for (int c = 0; c < DH * 2; c += 128) prefetch_l2(reinterpret_cast<const uint8_t*>(qn) + c);
            }
            if (!g.dense && !stats) {
              const float* nn = g.n_in + ((size_t)hn * g.S + tn) * DH + half * kHalfCols;
#pragma unroll
              for (int c = 0; c < kHalfCols * 4; c += 128) prefetch_l2(reinterpret_cast<const uint8_t*>(nn) + c);
            }
          }
        }
      }

      // the row's causal prefix of the selection (columns ascend, so the
      // valid columns of every tile form a prefix of it)
      const int nc_row = tok < 0 ? 0 : at_row_count(g, h, a, tok);
      for (int t = 0; t < nt; ++t, ++u) {
        const uint32_t b = u & 1;
        const int c0 = t * kAtCols;
        const int nvalid = min(max(nc_row - c0, 0), kAtCols);
        const int first = half * 32;  // this thread's first column in the tile
        wait_or_die(&s_full[b], (u >> 1) & 1);
        uint32_t rn[32], ro[32];
        const uint32_t sbase = tmem + lane_base + C::kColS + b * 128;
        float mx = -INFINITY;
        if (!dead) {
          __syncwarp();
          tmem_ld32(sbase + first, rn);
          if (has_old) tmem_ld32(sbase + 64 + first, ro);
          tmem_wait_ld();
          if (nvalid < first + 32) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              if (first + e >= nvalid) {
                rn[e] = 0xff800000u;  // -inf
                ro[e] = 0xff800000u;
              }
            }
          }
          if (!fixed) {
            // tree reduction: 5 dependent steps instead of a 32-long chain
            float t16[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) t16[e] = fmaxf(__uint_as_float(rn[e]), __uint_as_float(rn[e + 16]));
#pragma unroll
            for (int w = 8; w > 0; w >>= 1)
#pragma unroll
              for (int e = 0; e < w; ++e) t16[e] = fmaxf(t16[e], t16[e + w]);
            mx = t16[0];
          }
        }
        if (!fixed) {  // the update pass has a fixed frame: no maxima to exchange
          float* xm = xchg + (b * 2) * 128;  // [half][128] of this parity
          xm[half * 128 + row] = mx;
          named_bar_sync(pair_bar, 64);
          mx = fmaxf(mx, xm[(1 - half) * 128 + row]);
        }
        if (dead) continue;
        const bool need = !fixed && mx > m_ref + kRescaleThreshold;
        if (__any_sync(0xffffffffu, need)) {
          // raise the reference of this warp's rows: N and Z scale by 2^(m_ref - mx)
          const float new_ref = need ? mx : m_ref;
          const float f = need ? ex2(m_ref - new_ref) : 1.f;
          if (!stats) {  // the statistics pass keeps no N
            if (t > 0) {
              const uint32_t up = u - 1;
              wait_or_die(&pv_done[up & 1], (up >> 1) & 1);
              if (dead) continue;
            }
#pragma unroll 1
            for (int cc = 0; cc < kHalfCols; cc += 16) {
              uint32_t r[16];
              __syncwarp();
              tmem_ld16(tmem + lane_base + C::kColN + half * kHalfCols + cc, r);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * f);
              __syncwarp();
              tmem_st16(tmem + lane_base + C::kColN + half * kHalfCols + cc, r);
            }
            tmem_wait_st();
          }
          z *= f;
          z_old *= f;
          m_ref = new_ref;
        }
        uint32_t pk[16];
        const float o_new = fixed ? off_new : m_ref;
        const float o_old = fixed ? off_old : m_ref;
        // four independent partial sums per matrix (short dependency chains)
        float za[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) {
          const float p0 = ex2(__uint_as_float(rn[2 * e2]) - o_new);
          const float p1 = ex2(__uint_as_float(rn[2 * e2 + 1]) - o_new);
          za[e2 & 3] += p0 + p1;
          pk[e2] = pack_half2(p0, p1);
        }
        if (!stats) {
          __syncwarp();
          tmem_st16(sbase + half * 16, pk);
        }
        float zb[4] = {0.f, 0.f, 0.f, 0.f};
        if (has_old) {
#pragma unroll
          for (int e2 = 0; e2 < 16; ++e2) {
            const float p0 = ex2(__uint_as_float(ro[2 * e2]) - o_old);
            const float p1 = ex2(__uint_as_float(ro[2 * e2 + 1]) - o_old);
            zb[e2 & 3] += p0 + p1;
            pk[e2] = pack_half2(-p0, -p1);
          }
          if (!stats) {
            __syncwarp();
            tmem_st16(sbase + 32 + half * 16, pk);
          }
        }
        if (MODE == kAtRunning) {
          z += ((za[0] + za[1]) + (za[2] + za[3])) - ((zb[0] + zb[1]) + (zb[2] + zb[3]));
        } else if (stats) {
          z += (za[0] + za[1]) + (za[2] + za[3]);
          z_old += (zb[0] + zb[1]) + (zb[2] + zb[3]);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[b]);
      }
      if (nt > 0) {
        const uint32_t up = u - 1;
        wait_or_die(&pv_done[up & 1], (up >> 1) & 1);
      }
      // combine the two halves' sums
      float* xz = xchg + 4 * 128;
      float* xzo = xchg + 6 * 128;
      xz[half * 128 + row] = z;
      xzo[half * 128 + row] = z_old;
      named_bar_sync(pair_bar, 64);
      const float z_row = xz[row] + xz[128 + row];
      const float z_old_row = xzo[row] + xzo[128 + row];
      named_bar_sync(pair_bar, 64);
      if (dead) continue;
      if (stats) {
        // the frame and the selected-column factor for the update pass:
        // g = g_prev sum_J e^(s_old - m') / sum_J e^(s_new - m'), kept when J is empty
        if (tok >= 0 && half == 0) {
          const size_t hi = (size_t)h * g.S + tok;
          g.m_out[hi] = m_ref / kAtLog2e;
          g.g_out[hi] = z_row > 0.f ? g_prev * (z_old_row / z_row) : g_prev;
        }
        continue;
      }
      const float inv = 1.f / z_row;
#pragma unroll 1
      for (int cc = 0; cc < kHalfCols; cc += 16) {
        uint32_t r[16];
        __syncwarp();
        tmem_ld16(tmem + lane_base + C::kColN + half * kHalfCols + cc, r);
        tmem_wait_ld();
        if (tok >= 0) {
          const int col = half * kHalfCols + cc;
          float* nd = g.n_out + ((size_t)h * g.S + tok) * DH + col;
          uint32_t w[8];
#pragma unroll
          for (int v = 0; v < 2; ++v) {
#pragma unroll
            for (int e = 0; e < 8; ++e) w[e] = r[8 * v + e];
            st_global_v8(nd + 8 * v, w);
          }
#pragma unroll
          for (int q = 0; q < 8; ++q)
            w[q] = (uint32_t)float_to_bf16_bits(__uint_as_float(r[2 * q]) * inv) |
                   ((uint32_t)float_to_bf16_bits(__uint_as_float(r[2 * q + 1]) * inv) << 16);
          st_global_v8(g.o + (size_t)tok * HD + (size_t)h * DH + col, w);
        }
      }
      if (tok >= 0 && half == 0) {
        g.m_out[(size_t)h * g.S + tok] = m_ref / kAtLog2e;
        g.z_out[(size_t)h * g.S + tok] = z_row;
        if (g.dense && g.g_out) g.g_out[(size_t)h * g.S + tok] = 1.f;
      }
      tc_fence_before();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The running update of loops >= 2 ("ping-pong" kernel).
//
// Row pass split by tiles: row group 0 (warps 0-3) handles the tiles with an
// even block-wide tile counter, group 1 (warps 4-7) the odd ones, one thread
// per row over all 64 new and 64 old columns of its tile.  While one group
// computes the exponentials of tile t, the other loads and reduces tile t+1.
// The row's reference (log2 units) passes from the group of tile t to the
// group of tile t+1 through shared memory at a named barrier (an arrive on
// one side, a sync on the other; one barrier per group and lane quarter).
// Only the new scores can raise it: the old scores are the previous loop's,
// already within 8 of the reference it left behind, and the reference never
// decreases.  Each group keeps its own part of Z in the frame of the last
// tile it handled; the parts are brought to the final frame at the end of the
// item.  The rare raise rescales the whole row of N (after P(t-1).V) in the
// handling thread.
//
// TMEM: Q_new | Q_old (fp16 pairs), N (f32), one score buffer
// [S_new | S_old] and two P buffers [P_new | -P_old] (fp16 pairs).  The rows
// copy S_new(t) to registers and release its half of the score buffer at
// once (then S_old(t) the same way, after the new exponentials), so S(t+1)
// is computed while they take the exponentials of S(t); P(t) goes to P
// buffer t & 1 and P(t).V runs behind.  Three threads issue the MMAs (S_new,
// S_old, P.V), each as soon as its inputs are in, so that none waits behind
// another's MMAs.  K and V arrive in two rings of kAtStages slots (a slot
// holds the new and the old tile): a K slot is released when its score MMAs
// complete, a V slot after its P.V.  One thread loads both rings.
constexpr int kPpThreads = 384;  // 8 row warps; loads (+ TMEM allocation), S_new MMAs, S_old MMAs, P.V MMAs

template <int DH>
struct PpCfg {
  static constexpr uint32_t kColQn = 0;
  static constexpr uint32_t kColQo = DH / 2;
  static constexpr uint32_t kColN = DH;
  static constexpr uint32_t kColS = 2 * DH;        // S_new at +0, S_old at +64
  static constexpr uint32_t kColP = 2 * DH + 128;  // P buffer b at +64 b: P_new at +0, -P_old at +32
};

// Score-MMA role of one half (one thread each): S_new(t) = Q_new K_new^T
// (HALF 0) or S_old(t) = Q_old K_old^T (HALF 1) into its half of the score
// buffer once the K tiles are in and the rows copied the half of S(t-1) out.
// A thread that issues tcgen05.mma waits while the tensor pipe takes its
// MMAs, so the two halves and P.V each have their own thread: none waits
// behind another's MMAs or hand-offs.  The K slot is released when both
// halves' MMAs complete (k_empty counts two commits).
// s_empty: [HALF] (one completion per tile, waited here in order).
// s_full: [HALF * 2 + (t & 1)], one barrier per half and tile parity, so that
// each row group waits only on barriers that complete on its own tiles (a
// phase it waits for is never two completions behind).
template <int DH, int HALF>
__device__ __forceinline__ void pp_s_half_role(const uint8_t* kring, uint64_t* k_full, uint64_t* k_empty,
                                               uint64_t* s_full, uint64_t* s_empty, uint64_t* q_ready,
                                               volatile int* abort_flag, uint32_t tmem, const AtArgs& g, int n_rows,
                                               int row_tiles, int total) {
  using C = AtCfg<DH>;
  using P = PpCfg<DH>;
  int ks = 0;
  uint32_t kph = 0, u = 0, item_no = 0;  // item_no counts the items that have tiles
  bool ok = true;
  for (int item = blockIdx.x; item < total && ok && !*abort_flag; item += gridDim.x) {
    const int h = item / row_tiles, rt = item % row_tiles;
    const int nt = at_tiles(g, h, rt, n_rows);
    if (nt == 0) continue;  // the rows signal q_ready only for items with tiles
    if (!mbar_wait_sleep(q_ready, item_no & 1)) {
      ok = false;
      break;
    }
    ++item_no;
    for (int t = 0; t < nt; ++t, ++u) {
      const uint32_t k_addr = smem_u32(kring + ks * 2 * C::kKBytes) + HALF * C::kKBytes;
      if (!mbar_wait_sleep(&k_full[ks], kph) || (u > 0 && !mbar_wait_sleep(&s_empty[HALF], (u - 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk) {
        const uint32_t kd = k_addr + (kk >> 2) * (kAtCols * 128) + (kk & 3) * 32;
        umma_f16_ts(tmem + P::kColS + 64 * HALF, tmem + (HALF ? P::kColQo : P::kColQn) + kk * 8,
                    sw128_kmajor_desc(kd), C::kIdescS, kk > 0);
      }
      umma_commit(&s_full[2 * HALF + (u & 1)]);
      umma_commit(&k_empty[ks]);
      if (++ks == kAtStages) {
        ks = 0;
        kph ^= 1;
      }
    }
  }
  if (!ok) {
    set_error(g.err, kDevErrTimeout);
    *abort_flag = 1;
  }
}

// Load role (one thread): for every tile the K slot ([K_new | K_old]) and
// the V slot ([V_new^T | V_old^T]) by TMA, each into its ring once free.
template <int DH>
__device__ __forceinline__ void pp_load_role(uint8_t* kring, uint8_t* vring, uint64_t* k_full, uint64_t* k_empty,
                                             uint64_t* v_full, uint64_t* v_empty, const CUtensorMap* tkn,
                                             const CUtensorMap* tko, const CUtensorMap* tvn, const CUtensorMap* tvo,
                                             const AtArgs& g, int n_rows, int row_tiles, int total,
                                             volatile int* abort_flag) {
  using C = AtCfg<DH>;
  int ks = 0, vs = 0;
  uint32_t kph = 0, vph = 0;
  int kiss[kAtStages], viss[kAtStages];
  for (int s2 = 0; s2 < kAtStages; ++s2) kiss[s2] = viss[s2] = -1;
  for (int item = blockIdx.x; item < total && !*abort_flag; item += gridDim.x) {
    const int h = item / row_tiles, rt = item % row_tiles;
    const int nt = at_tiles(g, h, rt, n_rows);
    for (int t = 0; t < nt && !*abort_flag; ++t) {
      if (!mbar_wait_sleep(&k_empty[ks], kph ^ 1)) {
        set_error(g.err, kDevErrTimeout);
        *abort_flag = 1;
        break;
      }
      uint8_t* st = kring + ks * 2 * C::kKBytes;
      mbar_arrive_expect_tx(&k_full[ks], 2 * C::kKBytes);
#pragma unroll
      for (int c = 0; c < DH / 64; ++c) tma_load_3d(st + c * (kAtCols * 128), tkn, c * 64, t * kAtCols, h, &k_full[ks]);
#pragma unroll
      for (int c = 0; c < DH / 64; ++c)
        tma_load_3d(st + C::kKBytes + c * (kAtCols * 128), tko, c * 64, t * kAtCols, h, &k_full[ks]);
      kiss[ks] = kph;
      if (++ks == kAtStages) {
        ks = 0;
        kph ^= 1;
      }
      if (!mbar_wait_sleep(&v_empty[vs], vph ^ 1)) {
        set_error(g.err, kDevErrTimeout);
        *abort_flag = 1;
        break;
      }
      uint8_t* sv = vring + vs * 2 * C::kVBytes;
      mbar_arrive_expect_tx(&v_full[vs], 2 * C::kVBytes);
      tma_load_3d(sv, tvn, t * kAtCols, 0, h, &v_full[vs]);
      tma_load_3d(sv + C::kVBytes, tvo, t * kAtCols, 0, h, &v_full[vs]);
      viss[vs] = vph;
      if (++vs == kAtStages) {
        vs = 0;
        vph ^= 1;
      }
    }
  }
  // never leave with a copy in flight: wait (bounded) for the last load of every slot
  for (int s2 = 0; s2 < kAtStages; ++s2) {
    if (kiss[s2] >= 0) (void)mbar_wait(&k_full[s2], (uint32_t)kiss[s2]);
    if (viss[s2] >= 0) (void)mbar_wait(&v_full[s2], (uint32_t)viss[s2]);
  }
}

// P.V role (one thread): N += [P_new | -P_old] [V_new; V_old] for every tile
// once its P buffer and V tiles are in, the V slot released when it completes.
// pv_done[t & 1] and pv_done4[t & 3] both complete when P(t).V has: a row
// group waits on pv_done for its own tiles and on pv_done4 for the other
// group's (four barriers keep that wait within one phase, see the rows).
template <int DH>
__device__ __forceinline__ void pp_pv_role(const uint8_t* vring, uint64_t* v_full, uint64_t* v_empty,
                                           uint64_t* p_full, uint64_t* pv_done, uint64_t* pv_done4,
                                           volatile int* abort_flag,
                                           uint32_t tmem, const AtArgs& g, int n_rows, int row_tiles, int total) {
  using C = AtCfg<DH>;
  using P = PpCfg<DH>;
  int vs = 0;
  uint32_t vph = 0, u = 0;
  bool ok = true;
  for (int item = blockIdx.x; item < total && ok && !*abort_flag; item += gridDim.x) {
    const int h = item / row_tiles, rt = item % row_tiles;
    const int nt = at_tiles(g, h, rt, n_rows);
    for (int t = 0; t < nt; ++t, ++u) {
      if (!mbar_wait_sleep(&p_full[u & 1], (u >> 1) & 1) || !mbar_wait_sleep(&v_full[vs], vph)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t pcol = tmem + P::kColP + (u & 1) * 64;
      const uint32_t v_addr = smem_u32(vring + vs * 2 * C::kVBytes);
#pragma unroll
      for (int kk = 0; kk < kAtCols / 16; ++kk)
        umma_f16_ts(tmem + P::kColN, pcol + kk * 8, sw128_kmajor_desc(v_addr + kk * 32), C::kIdescPV, 1u);
#pragma unroll
      for (int kk = 0; kk < kAtCols / 16; ++kk)
        umma_f16_ts(tmem + P::kColN, pcol + 32 + kk * 8, sw128_kmajor_desc(v_addr + C::kVBytes + kk * 32),
                    C::kIdescPV, 1u);
      umma_commit(&v_empty[vs]);
      umma_commit(&pv_done[u & 1]);
      umma_commit(&pv_done4[u & 3]);
      if (++vs == kAtStages) {
        vs = 0;
        vph ^= 1;
      }
    }
  }
  if (!ok) {
    set_error(g.err, kDevErrTimeout);
    *abort_flag = 1;
  }
}

template <int DH>
__global__ void __launch_bounds__(kPpThreads, 1)
attn_pp_kernel(const __grid_constant__ CUtensorMap tm_kn, const __grid_constant__ CUtensorMap tm_ko,
               const __grid_constant__ CUtensorMap tm_vn, const __grid_constant__ CUtensorMap tm_vo, AtArgs g) {
  using C = AtCfg<DH>;
  using P = PpCfg<DH>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // K ring: kAtStages slots of [K_new | K_old]; V ring: slots of [V_new^T | V_old^T]
  uint8_t* kring = smem;
  uint8_t* vring = smem + kAtStages * 2 * C::kKBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kAtStages * C::kStageBytes);
  uint64_t* k_full = bars;                   // [stages]
  uint64_t* k_empty = bars + kAtStages;      // [stages]
  uint64_t* v_full = bars + 2 * kAtStages;   // [stages]
  uint64_t* v_empty = bars + 3 * kAtStages;  // [stages]
  uint64_t* s_full = bars + 4 * kAtStages;   // [4] S_new(t) / S_old(t) landed: [half * 2 + (t & 1)]
  uint64_t* s_empty = s_full + 4;            // [2] the rows copied S_new(t) / S_old(t) out
  uint64_t* p_full = s_empty + 2;            // [2] P(t) in P buffer t & 1
  uint64_t* pv_done = p_full + 2;            // [2] P(t).V complete, by t & 1
  uint64_t* pv_done4 = pv_done + 2;          // [4] P(t).V complete, by t & 3
  uint64_t* q_ready = pv_done4 + 4;          // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_ready + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int n_rows = g.n_rows ? *g.n_rows : g.S;
  if (n_rows > g.row_cap) n_rows = g.row_cap;
  if (n_rows < 0) n_rows = 0;
  const int row_tiles = (n_rows + kAtRows - 1) / kAtRows;
  const int total = row_tiles * g.H;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kAtStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 2);  // both score halves
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 4; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&pv_done4[b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_empty[b], kAtRowThreads / 2);  // the 128 threads of the tile's group
      mbar_init(&p_full[b], kAtRowThreads / 2);
      mbar_init(&pv_done[b], 1);
    }
    mbar_init(q_ready, kAtRowThreads);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    if (lane == 0)
      pp_load_role<DH>(kring, vring, k_full, k_empty, v_full, v_empty, &tm_kn, &tm_ko, &tm_vn, &tm_vo, g, n_rows,
                       row_tiles, total, abort_flag);
  } else if (warp == 9) {
    if (lane == 0)
      pp_s_half_role<DH, 0>(kring, k_full, k_empty, s_full, s_empty, q_ready, abort_flag, tmem, g, n_rows, row_tiles,
                            total);
  } else if (warp == 10) {
    if (lane == 0)
      pp_s_half_role<DH, 1>(kring, k_full, k_empty, s_full, s_empty, q_ready, abort_flag, tmem, g, n_rows, row_tiles,
                            total);
  } else if (warp == 11) {
    if (lane == 0)
      pp_pv_role<DH>(vring, v_full, v_empty, p_full, pv_done, pv_done4, abort_flag, tmem, g, n_rows, row_tiles, total);
  } else {
    // A named barrier cannot time out, so both groups always execute the same
    // barrier sequence: after a failed wait (or an abort raised elsewhere) a
    // warp turns "dead" - it skips waits, tensor-memory work and writes but
    // keeps the control flow.
    const int quarter = warp & 3, grp = warp >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int bar_give = 1 + grp * 4 + quarter;          // this group's reference is ready
    const int bar_take = 1 + (grp ^ 1) * 4 + quarter;    // the other group's reference is ready
    const int bar_end = 9 + quarter;                     // end of item: the two parts of Z
    float* xm = reinterpret_cast<float*>(tmem_slot + 4);  // [2 groups][128] reference after the group's tile
    float* xz = xm + 2 * 128;                             // [2][128] part of Z
    float* xf = xz + 2 * 128;                             // [2][128] frame of that part
    const int HD = g.H * DH;
    constexpr int kHalfCols = DH / 2;
    bool dead = false;
    auto wait_or_die = [&](uint64_t* bar, uint32_t parity) {
      if (!dead && __any_sync(0xffffffffu, *abort_flag != 0)) dead = true;
      if (dead) return;
      if (!__all_sync(0xffffffffu, mbar_wait_sleep(bar, parity))) {
        set_error(g.err, kDevErrTimeout);
        *abort_flag = 1;
        dead = true;
        return;
      }
      tc_fence_after();
    };
    uint32_t u = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
      const int h = item / row_tiles, rt = item % row_tiles;
      const int nt = at_tiles(g, h, rt, n_rows);
      const int a = rt * kAtRows + row;
      int tok = -1;
      if (a < n_rows) {
        tok = g.rows ? __ldg(g.rows + a) : a;
        if (tok < 0 || tok >= g.S) {
          if (grp == 0) set_error(g.err, FLASHLOOP_DEVERR_INDEX);
          tok = -1;
        }
      }
      // the previous loop's state: reference m_in (log2 units) and Z_in,
      // carried by group 0's part of Z
      float m_init = 0.f, z_part = 0.f;
      if (tok >= 0) {
        const size_t hi = (size_t)h * g.S + tok;
        m_init = g.m_in[hi] * kAtLog2e;
        if (grp == 0) z_part = g.z_in[hi];
      }
      float frame = m_init;  // frame of z_part
      // Q (fp16 pairs, exact from bf16) and this group's half of N into TMEM:
      // group 0 Q_new and N[0, DH/2), group 1 Q_old and N[DH/2, DH).  The
      // rebuilt keys carry log2(e)/sqrt(dh), so S is in log2 units.
      if (!dead) {
        const uint16_t* qsrc = grp == 0 ? g.q_new : g.q_old;
        const uint32_t qcol = grp == 0 ? P::kColQn : P::kColQo;
        uint32_t qv[DH / 16][8];
#pragma unroll
        for (int v = 0; v < DH / 16; ++v) {
          if (tok >= 0) {
            ld_global_v8(qsrc + (size_t)tok * HD + (size_t)h * DH + v * 16, qv[v]);
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) qv[v][e] = 0u;
          }
        }
        bool q_ok = true;  // q must fit fp16, the MMA operand type
#pragma unroll
        for (int c0 = 0; c0 < DH; c0 += 32) {
          uint32_t r[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 f = bf16x2_to_float2(qv[c0 / 16 + e / 8][e % 8]);
            q_ok = q_ok && half_range_ok(f.x) && half_range_ok(f.y);
            r[e] = bf16x2_to_half2_bits(qv[c0 / 16 + e / 8][e % 8]);
          }
          __syncwarp();
          tmem_st16(tmem + lane_base + qcol + c0 / 2, r);
        }
        if (!q_ok) set_error(g.err, FLASHLOOP_DEVERR_RANGE);
        uint32_t nv[kHalfCols / 8][8];
#pragma unroll
        for (int v = 0; v < kHalfCols / 8; ++v) {
          if (tok >= 0) {
            ld_global_v8(g.n_in + ((size_t)h * g.S + tok) * DH + grp * kHalfCols + 8 * v, nv[v]);
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) nv[v][e] = 0u;
          }
        }
#pragma unroll
        for (int c0 = 0; c0 < kHalfCols; c0 += 16) {
          uint32_t r[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = nv[c0 / 8 + e / 8][e % 8];
          __syncwarp();
          tmem_st16(tmem + lane_base + P::kColN + grp * kHalfCols + c0, r);
        }
        tmem_wait_st();
        tc_fence_before();
        // only items with tiles: the score issuers wait on q_ready for those
        // alone, so the rows can never run two phases ahead of them
        if (nt > 0) mbar_arrive(q_ready);
        // bring the next item's rows (this thread's q and half of N) into L2
        const int item_next = item + gridDim.x;
        if (item_next < total) {
          const int hn = item_next / row_tiles, an = (item_next % row_tiles) * kAtRows + row;
          const int tn = an < n_rows ? (g.rows ? __ldg(g.rows + an) : an) : -1;
          if (tn >= 0 && tn < g.S) {
            const uint16_t* qn = (grp == 0 ? g.q_new : g.q_old) + (size_t)tn * HD + (size_t)hn * DH;
#pragma unroll
            for (int c = 0; c < DH * 2; c += 128) prefetch_l2(reinterpret_cast<const uint8_t*>(qn) + c);
            const float* nn = g.n_in + ((size_t)hn * g.S + tn) * DH + grp * kHalfCols;
#pragma unroll
            for (int c = 0; c < kHalfCols * 4; c += 128) prefetch_l2(reinterpret_cast<const uint8_t*>(nn) + c);
          }
        }
      }

      // the row's causal prefix of the selection (columns ascend, so the
      // valid columns of every tile form a prefix of it)
      const int nc_row = tok < 0 ? 0 : at_row_count(g, h, a, tok);
      for (int t = 0; t < nt; ++t, ++u) {
        const uint32_t b = u & 1;
        if ((int)b != grp) continue;  // the other group's tile
        const int nvalid = min(max(nc_row - t * kAtCols, 0), kAtCols);
        wait_or_die(&s_full[b], (u >> 1) & 1);
        uint32_t sc[64];
        float mx = -INFINITY;
        if (!dead) {
          // copy S_new(t) out and hand its half of the score buffer back at once
          __syncwarp();
          tmem_ld32(tmem + lane_base + P::kColS, *reinterpret_cast<uint32_t(*)[32]>(sc));
          tmem_ld32(tmem + lane_base + P::kColS + 32, *reinterpret_cast<uint32_t(*)[32]>(sc + 32));
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(&s_empty[0]);
          if (nvalid < kAtCols) {
#pragma unroll
            for (int e = 0; e < 64; ++e)
              if (e >= nvalid) sc[e] = 0xff800000u;  // -inf
          }
          mx = max64(sc);
        }
        // the reference after tile t-1 (this item's), from the other group
        float m_prev = m_init;
        if (t > 0) {
          named_bar_sync(bar_take, 64);
          m_prev = xm[(grp ^ 1) * 128 + row];
        }
        const bool need = mx > m_prev + kRescaleThreshold;
        const float m_ref = need ? mx : m_prev;
        if (t + 1 < nt) {
          xm[grp * 128 + row] = m_ref;
          named_bar_arrive(bar_give, 64);
        }
        if (dead) continue;
        // P buffer b still feeds P(u-2).V until that completes (this group's
        // own previous tile: pv_done[b] is then one phase from that wait)
        if (u >= 2) {
          wait_or_die(&pv_done[b], ((u - 2) >> 1) & 1);
          if (dead) continue;
        }
        if (__any_sync(0xffffffffu, need)) {
          // raise the reference of this warp's rows: N scales by 2^(m_prev - m_ref)
          // once P(t-1).V has landed.  P(u-2).V is complete (above), so is
          // P(u-5).V, the previous completion of pv_done4[(u-1) & 3].
          const float f = need ? ex2(m_prev - m_ref) : 1.f;
          if (t > 0) {
            const uint32_t up = u - 1;
            wait_or_die(&pv_done4[up & 3], (up >> 2) & 1);
            if (dead) continue;
          }
#pragma unroll 1
          for (int cc = 0; cc < DH; cc += 16) {
            uint32_t r[16];
            __syncwarp();
            tmem_ld16(tmem + lane_base + P::kColN + cc, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * f);
            __syncwarp();
            tmem_st16(tmem + lane_base + P::kColN + cc, r);
          }
          tmem_wait_st();
        }
        if (frame != m_ref) {
          z_part *= ex2(frame - m_ref);
          frame = m_ref;
        }
        const uint32_t pbase = tmem + lane_base + P::kColP + b * 64;
        // P_new = 2^(S_new - m_ref) over columns [0, 32) of the P buffer (fp16 pairs)
        float za[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t pk[16];
#pragma unroll
          for (int e2 = 0; e2 < 16; ++e2) {
            float x0 = __uint_as_float(sc[32 * hf + 2 * e2]), x1 = __uint_as_float(sc[32 * hf + 2 * e2 + 1]);
            sub2_rn(x0, x1, m_ref);
            const float p0 = ex2(x0), p1 = ex2(x1);
            if (e2 & 1) add2_rn(za[2], za[3], p0, p1);
            else add2_rn(za[0], za[1], p0, p1);
            pk[e2] = pack_half2(p0, p1);
          }
          __syncwarp();
          tmem_st16(pbase + 16 * hf, pk);
        }
        // -P_old = -2^(S_old - m_ref) over columns [32, 64)
        wait_or_die(&s_full[2 + b], (u >> 1) & 1);
        if (dead) continue;
        __syncwarp();
        tmem_ld32(tmem + lane_base + P::kColS + 64, *reinterpret_cast<uint32_t(*)[32]>(sc));
        tmem_ld32(tmem + lane_base + P::kColS + 96, *reinterpret_cast<uint32_t(*)[32]>(sc + 32));
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&s_empty[1]);
        if (nvalid < kAtCols) {
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (e >= nvalid) sc[e] = 0xff800000u;
        }
        float zb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t pk[16];
#pragma unroll
          for (int e2 = 0; e2 < 16; ++e2) {
            float x0 = __uint_as_float(sc[32 * hf + 2 * e2]), x1 = __uint_as_float(sc[32 * hf + 2 * e2 + 1]);
            sub2_rn(x0, x1, m_ref);
            const float p0 = ex2(x0), p1 = ex2(x1);
            if (e2 & 1) add2_rn(zb[2], zb[3], p0, p1);
            else add2_rn(zb[0], zb[1], p0, p1);
            pk[e2] = pack_half2(-p0, -p1);
          }
          __syncwarp();
          tmem_st16(pbase + 32 + 16 * hf, pk);
        }
        z_part += ((za[0] + za[1]) + (za[2] + za[3])) - ((zb[0] + zb[1]) + (zb[2] + zb[3]));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[b]);
      }
      if (nt > 0) {
        // every contribution of the item has reached N.  Each group has seen
        // P(last-2).V or P(last-3).V complete at its own last tile, so the
        // previous completion of pv_done4[last & 3], P(last-4).V, is too.
        const uint32_t up = u - 1;
        wait_or_die(&pv_done4[up & 3], (up >> 2) & 1);
      }
      // the two parts of Z in the final frame (frames only rise: the larger)
      xz[grp * 128 + row] = z_part;
      xf[grp * 128 + row] = frame;
      named_bar_sync(bar_end, 64);
      const float z_other = xz[(grp ^ 1) * 128 + row];
      const float f_other = xf[(grp ^ 1) * 128 + row];
      named_bar_sync(bar_end, 64);
      if (dead) continue;
      const float m_fin = fmaxf(frame, f_other);
      const float z_row = (frame == m_fin ? z_part : z_part * ex2(frame - m_fin)) +
                          (f_other == m_fin ? z_other : z_other * ex2(f_other - m_fin));
      const float inv = 1.f / z_row;
#pragma unroll 1
      for (int cc = 0; cc < kHalfCols; cc += 16) {
        uint32_t r[16];
        __syncwarp();
        tmem_ld16(tmem + lane_base + P::kColN + grp * kHalfCols + cc, r);
        tmem_wait_ld();
        if (tok >= 0) {
          const int col = grp * kHalfCols + cc;
          float* nd = g.n_out + ((size_t)h * g.S + tok) * DH + col;
          uint32_t w[8];
#pragma unroll
          for (int v = 0; v < 2; ++v) {
#pragma unroll
            for (int e = 0; e < 8; ++e) w[e] = r[8 * v + e];
            st_global_v8(nd + 8 * v, w);
          }
#pragma unroll
          for (int q = 0; q < 8; ++q)
            w[q] = (uint32_t)float_to_bf16_bits(__uint_as_float(r[2 * q]) * inv) |
                   ((uint32_t)float_to_bf16_bits(__uint_as_float(r[2 * q + 1]) * inv) << 16);
          st_global_v8(g.o + (size_t)tok * HD + (size_t)h * DH + col, w);
        }
      }
      if (tok >= 0 && grp == 0) {
        g.m_out[(size_t)h * g.S + tok] = m_fin / kAtLog2e;
        g.z_out[(size_t)h * g.S + tok] = z_row;
      }
      tc_fence_before();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Column mass on the tensor cores [FlashLoop §4.2, App. D.2: the loop's
// column statistics rank the next selection]:
//   c[j] = sum over rows i with token_i >= token_j of 2^(s_ij - m_i) / Z_i,
// s in log2 units (the rebuilt keys carry log2(e)/sqrt(dh)), m and Z the
// rows' final state.  Transposed score tiles S^T = Khat_tile . q_tile^T put
// one column in each TMEM lane, so a column's mass is a sum inside one
// thread (no cross-lane reduction).  A work item = 128 selected columns of
// one head; it walks 128-row tiles (M128 N128 score MMAs) from the first row
// whose token reaches the item's smallest column token.  Rows come prepared per head: fp16 q (the
// same type as the keys, as kind::f16 requires), the frame m_i + log2(Z_i)
// in log2 units (so a contribution is one exp2: 2^(s - m) / Z = 2^(s - frame))
// and the row token.
// Roles: warps 0-7 reduce and load the item's keys into TMEM (A operand):
// group 0 (warps 0-3) takes the tiles with an even block-wide tile counter,
// group 1 (warps 4-7) the odd ones, one thread per column over all 128 rows of
// the tile, so that one group's exponentials overlap the other group's waits
// and loads; warp 8 allocates TMEM and streams the row tiles (TMA for q, bulk
// copies for frames and tokens); warp 9 issues the MMAs.  All waits are
// bounded.  Three score buffers in TMEM (tile u in buffer u % 3) let the MMA
// run up to three tiles ahead of the reducers.
// ---------------------------------------------------------------------------
constexpr int kCmtCols = 128, kCmtRows = 128, kCmtStages = 4, kCmtThreads = 320;
constexpr int kCmtRowThreads = 256;

template <int DH>
struct CmtCfg {
  static constexpr int kQBytes = kCmtRows * DH * 2;  // q tile: 128 rows x DH (DH/64 swizzle chunks)
  static constexpr int kSideBytes = 1024;            // frames and tokens of the tile (2 x 512 B); keeps
                                                     // every stage's q tile on a 1024-byte swizzle atom
  static constexpr int kStageBytes = kQBytes + kSideBytes;
  static constexpr int kSmem = 1024 + kCmtStages * kStageBytes + 256 + 2 * 128 * 4;
  static constexpr uint32_t kColA = 0;       // keys, fp16 pairs: DH/2 columns
  static constexpr uint32_t kColS = 64;      // three S^T buffers of 128 columns (tile u in buffer u % 3)
  static constexpr uint32_t kIdesc = f16_idesc(128, kCmtRows, 0);
};

struct CmtArgs {
  int S, H, kc, kcp, n_cap;   // n_cap: rows allocated in the prepared arrays (multiple of 64)
  const int32_t* n_rows;      // device count of rows (NULL: S)
  int row_cap;
  const int32_t* cols;        // [H, kc] ascending tokens (NULL: identity)
  const int32_t* rtok;        // [n_cap] row tokens, -1 past the last row
  const float* m2;            // [H, n_cap] row frame m_i + log2(Z_i / g_i), log2 units (+inf: no row)
  const __half* k;            // [H, kcp, DH] rebuilt keys
  float* out;                 // [H, S], written at the column tokens
  int32_t* err;
};

__device__ __forceinline__ int cmt_first_row(const CmtArgs& g, int n_rows, int tok) {
  int lo = 0, hi = n_rows;  // first row whose token is >= tok (row tokens ascend)
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(g.rtok + mid) < tok) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

template <int DH>
__global__ void __launch_bounds__(kCmtThreads, 1)
colmass_tc_kernel(const __grid_constant__ CUtensorMap tm_q, CmtArgs g) {
  using C = CmtCfg<DH>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kCmtStages * C::kStageBytes);
  uint64_t* full = bars;                       // [stages]
  uint64_t* empty = bars + kCmtStages;         // [stages]: MMA commit + 256 reducer arrivals
  uint64_t* s_full = bars + 2 * kCmtStages;    // [3]
  uint64_t* s_empty = s_full + 3;              // [3]
  uint64_t* a_ready = s_empty + 3;             // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(a_ready + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* xsum = reinterpret_cast<float*>(smem + kCmtStages * C::kStageBytes + 256);  // [2][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int n_rows = g.n_rows ? *g.n_rows : g.S;
  if (n_rows > g.row_cap) n_rows = g.row_cap;
  if (n_rows < 0) n_rows = 0;
  const int col_tiles = (g.kc + kCmtCols - 1) / kCmtCols;
  const int total = col_tiles * g.H;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kCmtStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kCmtRowThreads / 2);  // MMA commit + the tile's row group
    }
    for (int b = 0; b < 3; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], kCmtRowThreads / 2);
    }
    mbar_init(a_ready, kCmtRowThreads);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // item -> (head, column tile); the column tiles with the most rows come first
  auto item_head = [&](int item) { return item % g.H; };
  auto item_tile = [&](int item) { return item / g.H; };
  auto item_rows = [&](int item, int& a_begin) {
    const int h = item_head(item), ct = item_tile(item);
    const int c0 = ct * kCmtCols;
    const int tok0 = g.cols ? __ldg(g.cols + (size_t)h * g.kc + c0) : c0;
    a_begin = (cmt_first_row(g, n_rows, tok0) / kCmtRows) * kCmtRows;
    return (n_rows - a_begin + kCmtRows - 1) / kCmtRows;
  };

  if (warp == 8) {
    // ------------------------------------------------------------ loads
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued[kCmtStages];
      for (int s2 = 0; s2 < kCmtStages; ++s2) issued[s2] = -1;
      for (int item = blockIdx.x; item < total && !*abort_flag; item += gridDim.x) {
        const int h = item_head(item);
        int a_begin;
        const int nt = item_rows(item, a_begin);
        for (int t = 0; t < nt && !*abort_flag; ++t) {
          if (!mbar_wait_sleep(&empty[stage], phase ^ 1)) {
            set_error(g.err, kDevErrTimeout);
            *abort_flag = 1;
            break;
          }
          uint8_t* st = smem + stage * C::kStageBytes;
          const int a0 = a_begin + t * kCmtRows;
          mbar_arrive_expect_tx(&full[stage], C::kQBytes + 2 * kCmtRows * 4);
#pragma unroll
          for (int c = 0; c < DH / 64; ++c)
            tma_load_3d(st + c * (kCmtRows * 128), &tm_q, c * 64, a0, h, &full[stage]);
          uint8_t* side = st + C::kQBytes;
          bulk_g2s(side, g.m2 + (size_t)h * g.n_cap + a0, kCmtRows * 4, &full[stage]);
          bulk_g2s(side + 512, g.rtok + a0, kCmtRows * 4, &full[stage]);
          issued[stage] = phase;
          if (++stage == kCmtStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      for (int s2 = 0; s2 < kCmtStages; ++s2)
        if (issued[s2] >= 0) (void)mbar_wait_sleep(&full[s2], (uint32_t)issued[s2]);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, u = 0, ready_no = 0;  // ready_no: items with row tiles so far
      for (int item = blockIdx.x; item < total && !*abort_flag; item += gridDim.x) {
        int a_begin;
        const int nt = item_rows(item, a_begin);
        if (nt == 0) continue;  // no row reaches the item's columns: no keys, no MMAs
        // a_ready completes once per item with row tiles, so that the reducers
        // (who fill the keys of an item only after every tile of the previous
        // such item) are never two completions ahead of this wait
        if (!mbar_wait_sleep(a_ready, ready_no & 1)) {
          set_error(g.err, kDevErrTimeout);
          *abort_flag = 1;
          break;
        }
        ++ready_no;
        tc_fence_after();
        bool ok = true;
        for (int t = 0; t < nt; ++t, ++u) {
          // buffer u % 3 was last read by tile u - 3 (released by its group)
          if (!mbar_wait_sleep(&full[stage], phase) || (u >= 3 && !mbar_wait_sleep(&s_empty[u % 3], ((u / 3) - 1) & 1))) {
            set_error(g.err, kDevErrTimeout);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sb = tmem + C::kColS + (u % 3) * kCmtRows;
          const uint32_t q_addr = smem_u32(smem + stage * C::kStageBytes);
#pragma unroll
          for (int ks = 0; ks < DH / 16; ++ks) {
            const uint32_t qd = q_addr + (ks >> 2) * (kCmtRows * 128) + (ks & 3) * 32;
            umma_f16_ts(sb, tmem + C::kColA + ks * 8, sw128_kmajor_desc(qd), C::kIdesc, ks > 0);
          }
          umma_commit(&s_full[u % 3]);
          umma_commit(&empty[stage]);
          if (++stage == kCmtStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
      }
    }
  } else {
    // ------------------------------------------------------------ reducers
    // Thread (quarter, group): TMEM lane = column quarter*32 + lane of the
    // item; group g handles the tiles with (u & 1) == g, all 128 rows (in two
    // halves of 64 loaded from TMEM one after the other).  A
    // named barrier cannot time out, so after a failed wait a warp goes on
    // through the same barriers without touching TMEM ("dead").
    const int quarter = warp & 3, half = warp >> 2;
    const int col = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int pair_bar = 1 + quarter;
    bool dead = false;
    auto wait_or_die = [&](uint64_t* bar, uint32_t parity) {
      if (!dead && __any_sync(0xffffffffu, *abort_flag != 0)) dead = true;
      if (dead) return;
      if (!__all_sync(0xffffffffu, mbar_wait_sleep(bar, parity))) {
        set_error(g.err, kDevErrTimeout);
        *abort_flag = 1;
        dead = true;
        return;
      }
      tc_fence_after();
    };
    int stage = 0;
    uint32_t phase = 0, u = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
      const int h = item_head(item), ct = item_tile(item);
      int a_begin;
      const int nt = item_rows(item, a_begin);
      const int c = ct * kCmtCols + col;
      const int ctok = c < g.kc ? (g.cols ? __ldg(g.cols + (size_t)h * g.kc + c) : c) : 0x7fffffff;
      // this column's keys into TMEM (the MMA's A operand): group h loads
      // elements [h*DH/2, (h+1)*DH/2); an item without row tiles needs none
      if (!dead && nt > 0) {
#pragma unroll 1
        for (int e0 = half * (DH / 2); e0 < (half + 1) * (DH / 2); e0 += 32) {
          uint32_t r[16];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w = make_uint4(0, 0, 0, 0);
            if (c < g.kc) w = *reinterpret_cast<const uint4*>(g.k + ((size_t)h * g.kcp + c) * DH + e0 + v * 8);
            r[4 * v] = w.x; r[4 * v + 1] = w.y; r[4 * v + 2] = w.z; r[4 * v + 3] = w.w;
          }
          __syncwarp();
          tmem_st16(tmem + lane_base + C::kColA + e0 / 2, r);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(a_ready);
      }
      float acc = 0.f;
      for (int t = 0; t < nt; ++t, ++u) {
        const int st_now = stage;
        const uint32_t ph_now = phase;
        if (++stage == kCmtStages) {
          stage = 0;
          phase ^= 1;
        }
        if ((int)(u & 1) != half) continue;  // the other group's tile
        wait_or_die(&full[st_now], ph_now);
        wait_or_die(&s_full[u % 3], (u / 3) & 1);
        if (dead) continue;
        const uint8_t* side = smem + st_now * C::kStageBytes + C::kQBytes;
        const int* stok = reinterpret_cast<const int*>(side + 512);
        const bool diag = stok[0] < ctok;
        float pa[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t r[64];
          __syncwarp();
          tmem_ld32(tmem + lane_base + C::kColS + (u % 3) * kCmtRows + hh * 64, *reinterpret_cast<uint32_t(*)[32]>(r));
          tmem_ld32(tmem + lane_base + C::kColS + (u % 3) * kCmtRows + hh * 64 + 32,
                    *reinterpret_cast<uint32_t(*)[32]>(r + 32));
          tmem_wait_ld();
          if (hh == 1) {
            tc_fence_before();
            mbar_arrive(&s_empty[u % 3]);
          }
          const float4* sm4 = reinterpret_cast<const float4*>(side) + hh * 16;
          const int* st2 = stok + hh * 64;
          if (!diag) {
#pragma unroll
            for (int e4 = 0; e4 < 16; ++e4) {
              const float4 f = sm4[e4];
              float x0 = __uint_as_float(r[4 * e4]), x1 = __uint_as_float(r[4 * e4 + 1]);
              float x2 = __uint_as_float(r[4 * e4 + 2]), x3 = __uint_as_float(r[4 * e4 + 3]);
              sub2v_rn(x0, x1, f.x, f.y);
              sub2v_rn(x2, x3, f.z, f.w);
              add2_rn(pa[0], pa[1], ex2(x0), ex2(x1));
              add2_rn(pa[2], pa[3], ex2(x2), ex2(x3));
            }
          } else {
#pragma unroll
            for (int e4 = 0; e4 < 16; ++e4) {
              const float4 f = sm4[e4];
              const float fr[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const float v = ex2(__uint_as_float(r[4 * e4 + k]) - fr[k]);
                pa[k] += st2[4 * e4 + k] >= ctok ? v : 0.f;
              }
            }
          }
        }
        acc += (pa[0] + pa[1]) + (pa[2] + pa[3]);
        mbar_arrive(&empty[st_now]);
      }
      // the two halves' sums of each column
      xsum[half * 128 + col] = acc;
      named_bar_sync(pair_bar, 64);
      if (!dead && half == 0 && c < g.kc && ctok >= 0 && ctok < g.S)
        g.out[(size_t)h * g.S + ctok] = acc + xsum[128 + col];
      named_bar_sync(pair_bar, 64);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Rows of the column mass, per head: fp16 q, the frame m + log2(Z / g) in
// log2 units, and the row tokens (-1 past the last row, up to n_cap).
template <int DH>
__global__ void __launch_bounds__(256)
colmass_prep_kernel(const ColmassArgs a, int n_cap, __half* q16, float* m2, int32_t* rtok) {
  int n_rows = a.n_rows ? *a.n_rows : a.S;
  if (n_rows > a.row_cap) n_rows = a.row_cap;
  const int lane = threadIdx.x & 31;
  const long long items = (long long)n_cap * a.H;
  for (long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); w < items; w += (long long)gridDim.x * 8) {
    const int h = (int)(w % a.H), r = (int)(w / a.H);
    int tok = -1;
    if (r < n_rows) {
      tok = a.rows ? a.rows[r] : r;
      if (tok < 0 || tok >= a.S) {
        if (lane == 0) set_error(a.err, FLASHLOOP_DEVERR_INDEX);
        tok = -1;
      }
    }
    __half* qd = q16 + ((size_t)h * n_cap + r) * DH;
    constexpr int E = DH / 32;
    float x[E];
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = 0.f;
    if (tok >= 0) {
      const uint16_t* qs = a.q + (size_t)tok * a.H * DH + (size_t)h * DH + lane * E;
#pragma unroll
      for (int e = 0; e < E; ++e) x[e] = bf16_bits_to_float(qs[e]);
    }
#pragma unroll
    for (int e = 0; e < E; ++e) qd[lane * E + e] = __float2half_rn(x[e]);
    if (lane == 0) {
      // the row's frame: 2^(s - m) * g / Z = 2^(s - (m + log2(Z / g))); no row, or
      // g = 0, gives +inf (a zero contribution)
      float fr = INFINITY;
      if (tok >= 0) {
        const size_t hi = (size_t)h * a.S + tok;
        const float gz = (a.g ? a.g[hi] : 1.f) / a.z[hi];
        if (gz > 0.f) fr = a.m[hi] * kAtLog2e - log2f(gz);
      }
      m2[(size_t)h * n_cap + r] = fr;
      if (h == 0) rtok[r] = tok;
    }
  }
}

// Per head and active row: how many of the head's selected columns lie at or
// before the row's token - the row's causal prefix of the ascending
// selection.  The attention kernels take their tile counts and masks from it
// instead of searching the selection at every work item.  An index outside
// [0, S) counts 0 (the attention kernels report it).
__global__ void __launch_bounds__(256)
attn_row_counts_kernel(const int32_t* __restrict__ rows, const int32_t* __restrict__ n_rows_ptr, int row_cap, int S,
                       int H, const int32_t* __restrict__ cols, int kc, int32_t* __restrict__ out) {
  int n_rows = n_rows_ptr ? *n_rows_ptr : S;
  if (n_rows > row_cap) n_rows = row_cap;
  if (n_rows < 0) n_rows = 0;
  const long long total = (long long)H * n_rows;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int h = (int)(i / n_rows), a = (int)(i % n_rows);
    const int tok = rows ? __ldg(rows + a) : a;
    int lo = 0;
    if (tok >= 0 && tok < S) {
      const int32_t* c = cols + (size_t)h * kc;
      int hi = kc;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(c + mid) <= tok) lo = mid + 1;
        else hi = mid;
      }
    }
    out[(size_t)h * row_cap + a] = lo;
  }
}

int launch_attn_row_counts(const AttnArgs& a, int32_t* out, cudaStream_t stream) {
  const long long total = (long long)a.H * a.row_cap;
  int grid = (int)((total + 255) / 256);
  if (grid > 148 * 8) grid = 148 * 8;
  if (grid < 1) grid = 1;
  attn_row_counts_kernel<<<grid, 256, 0, stream>>>(a.rows, a.n_rows, a.row_cap, a.S, a.H, a.cols, a.kc, out);
  return launch_status();
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// The driver's cuTensorMapEncodeTiled, looked up once (a function-local
// static: its initialisation is thread-safe).
static PFN_cuTensorMapEncodeTiled_v12000 at_encode_fn() {
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

// 3-D fp16 tensor map: dims (innermost first) d0 x d1 x d2, row pitch p1 and
// plane pitch p2 in elements, box b0 x b1 x 1, 128-byte swizzle.  Coordinates
// past d1 read as zero.
int make_tmap_f16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                     uint64_t p1, uint64_t p2, uint32_t b0, uint32_t b1) {
  auto fn = at_encode_fn();
  if (fn == nullptr) return FLASHLOOP_ERR_CUDA;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0 || (p1 * 2) % 16 != 0 || (p2 * 2) % 16 != 0)
    return FLASHLOOP_ERR_INVALID_ARG;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {p1 * 2, p2 * 2};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FLASHLOOP_OK : FLASHLOOP_ERR_CUDA;
}

int at_sm_count() {
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

// Column mass of loop `a` on the tensor cores (prep + kernel).  scratch_q
// holds [H, n_cap, dh] fp16, scratch_rows [H, n_cap] floats + [n_cap] ints.
int launch_colmass_tc(const flashloop_params* p, const ColmassArgs& a, void* scratch_q, void* scratch_rows,
                      cudaStream_t stream) {
  const int dh = p->head_dim, H = p->n_heads;
  const int n_cap = ((a.row_cap + kCmtRows - 1) / kCmtRows) * kCmtRows;
  __half* q16 = static_cast<__half*>(scratch_q);
  float* m2 = static_cast<float*>(scratch_rows);
  int32_t* rtok = reinterpret_cast<int32_t*>(m2 + (size_t)H * n_cap);
  long long items = (long long)n_cap * H;
  int pgrid = (int)((items + 7) / 8);
  if (pgrid > 148 * 16) pgrid = 148 * 16;
  if (dh == 128) colmass_prep_kernel<128><<<pgrid, 256, 0, stream>>>(a, n_cap, q16, m2, rtok);
  else colmass_prep_kernel<64><<<pgrid, 256, 0, stream>>>(a, n_cap, q16, m2, rtok);
  int rc = launch_status();
  if (rc != FLASHLOOP_OK) return rc;
  CUtensorMap tq;
  rc = make_tmap_f16_3d(&tq, q16, dh, n_cap, H, dh, (uint64_t)n_cap * dh, 64, kCmtRows);
  if (rc != FLASHLOOP_OK) return rc;
  CmtArgs g{};
  g.S = a.S; g.H = H; g.kc = a.kc; g.kcp = a.kcp; g.n_cap = n_cap; g.n_rows = a.n_rows; g.row_cap = a.row_cap;
  g.cols = a.cols; g.rtok = rtok; g.m2 = m2; g.k = a.k_new; g.out = a.out; g.err = a.err;
  const int max_items = ((a.kc + kCmtCols - 1) / kCmtCols) * H;
  int grid = at_sm_count();
  if (grid > max_items) grid = max_items;
  if (grid < 1) grid = 1;
  if (dh == 128) {
    FL_TRY(cudaFuncSetAttribute(colmass_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, CmtCfg<128>::kSmem));
    colmass_tc_kernel<128><<<grid, kCmtThreads, CmtCfg<128>::kSmem, stream>>>(tq, g);
  } else {
    FL_TRY(cudaFuncSetAttribute(colmass_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, CmtCfg<64>::kSmem));
    colmass_tc_kernel<64><<<grid, kCmtThreads, CmtCfg<64>::kSmem, stream>>>(tq, g);
  }
  return launch_status();
}

// K buffers are [H, kcp, dh], V^T buffers [H, dh, kcp] (fp16), kcp = kc rounded up to 8.
int launch_attn_dense(const flashloop_params* p, const AttnArgs& a, int kcp, cudaStream_t stream);

int launch_attn_tc(const flashloop_params* p, const AttnArgs& a, int kcp, cudaStream_t stream) {
  const int dh = p->head_dim, H = p->n_heads;
  // the dense loop: two row tiles per CTA sharing every K / V tile (attn_dense.cu)
  if (a.mode == kAtRunning && a.dense) return launch_attn_dense(p, a, kcp, stream);
  if (a.cols != nullptr && a.row_cnt == nullptr) return FLASHLOOP_ERR_INVALID_ARG;
  // the row warps move q, N and O rows in 32-byte accesses
  const void* aligned32[] = {a.q_new, a.q_old, a.n_in, a.n_out, a.o};
  for (const void* ptr : aligned32)
    if (reinterpret_cast<uintptr_t>(ptr) % 32 != 0) return FLASHLOOP_ERR_INVALID_ARG;
  CUtensorMap tkn, tko, tvn, tvo;
  int rc = make_tmap_f16_3d(&tkn, a.k_new, dh, a.kc, H, dh, (uint64_t)kcp * dh, 64, kAtCols);
  if (rc == FLASHLOOP_OK) rc = make_tmap_f16_3d(&tvn, a.v_new, a.kc, dh, H, kcp, (uint64_t)kcp * dh, kAtCols, dh);
  if (rc == FLASHLOOP_OK && !a.dense) {
    rc = make_tmap_f16_3d(&tko, a.k_old, dh, a.kc, H, dh, (uint64_t)kcp * dh, 64, kAtCols);
    if (rc == FLASHLOOP_OK) rc = make_tmap_f16_3d(&tvo, a.v_old, a.kc, dh, H, kcp, (uint64_t)kcp * dh, kAtCols, dh);
  } else {
    tko = tkn;
    tvo = tvn;
  }
  if (rc != FLASHLOOP_OK) return rc;
  AtArgs g{};
  g.S = a.S; g.H = a.H; g.kc = a.kc; g.dense = a.dense; g.rows = a.rows; g.n_rows = a.n_rows;
  g.row_cap = a.row_cap; g.cols = a.cols; g.q_new = a.q_new; g.q_old = a.q_old; g.m_in = a.m_in;
  g.z_in = a.z_in; g.n_in = a.n_in; g.m_out = a.m_out; g.z_out = a.z_out; g.n_out = a.n_out; g.o = a.o;
  g.scale_log2 = a.scale_log2; g.err = a.err;
  g.g_in = a.g_in; g.g_out = a.g_out; g.row_cnt = a.row_cnt;
  const int max_items = ((a.row_cap + kAtRows - 1) / kAtRows) * H;
  int grid = at_sm_count();
  if (grid > max_items) grid = max_items;
  if (grid < 1) grid = 1;
  if (a.mode != kAtRunning && (a.dense || !a.g_in || !a.g_out)) return FLASHLOOP_ERR_INVALID_ARG;
  auto launch = [&](auto kernel, int smem) -> int {
    FL_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    kernel<<<grid, kAtThreads, smem, stream>>>(tkn, tko, tvn, tvo, g);
    return FLASHLOOP_OK;
  };
  auto launch_pp = [&](auto kernel, int smem) -> int {
    FL_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    kernel<<<grid, kPpThreads, smem, stream>>>(tkn, tko, tvn, tvo, g);
    return FLASHLOOP_OK;
  };
  // the running update: the ping-pong row pass; the fixed-mass passes: the
  // column-split row pass of attn_tc_kernel
  if (dh == 128) {
    if (a.mode == kAtFixedMassStats) rc = launch(attn_tc_kernel<128, kAtFixedMassStats>, AtCfg<128>::kSmem);
    else if (a.mode == kAtFixedMassUpdate) rc = launch(attn_tc_kernel<128, kAtFixedMassUpdate>, AtCfg<128>::kSmem);
    else rc = launch_pp(attn_pp_kernel<128>, AtCfg<128>::kSmem);
  } else {
    if (a.mode == kAtFixedMassStats) rc = launch(attn_tc_kernel<64, kAtFixedMassStats>, AtCfg<64>::kSmem);
    else if (a.mode == kAtFixedMassUpdate) rc = launch(attn_tc_kernel<64, kAtFixedMassUpdate>, AtCfg<64>::kSmem);
    else rc = launch_pp(attn_pp_kernel<64>, AtCfg<64>::kSmem);
  }
  if (rc != FLASHLOOP_OK) return rc;
  return launch_status();
}

}  // namespace fl
