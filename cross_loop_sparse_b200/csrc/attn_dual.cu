// (a6) Sparse attention update (and the dense loop-1 attention) on the
// sm_100a tensor cores, two 128-row tiles per CTA sharing every K / V tile.
//
// [FlashLoop §3.2, §4.2, App. D.2]: for every active row i of loop r and
// selected column j <= i, the loop r-1 contribution of (i, j) is removed from
// the row's running state and the loop-r one added:
//   S_old = Q^(r-1) Khat^(r-1)^T / sqrt(dh),  S_new = Q^(r) Khat^(r)^T / sqrt(dh)
//   N' = a N + [e^(S_new - m') | -e^(S_old - m')] [Vhat^(r); Vhat^(r-1)]
//   Z' = a Z + sum e^(S_new - m') - sum e^(S_old - m')
// The dense loop 1 is the same pass with no old half and an empty state.
//
// Work item: one head and 256 consecutive active rows, as two 128-row tiles
// A and B.  Each K / V tile of 64 selected columns is loaded once per item and
// used by both tiles, so a CTA moves half the K / V bytes per row of a
// one-tile design.
//
// Shared memory: the item's queries, fp16, 128-byte swizzled K-major
// (Q_new and Q_old of A and B: 4 x 128 x DH), and a ring of K / V slots, a
// slot holding either [K_new | K_old] (64 x DH each) or [V_new^T | V_old^T]
// (DH x 64 each), filled by TMA.
// TMEM (512 columns): N_A, N_B (float32, DH columns each), then per tile a
// score buffer {S_new 64 | S_old 64}; P = [e_new | -e_old] (fp16 pairs) is
// written over the S_new half and feeds the P.V MMA from TMEM.
//
// Roles (14 warps):
//   warps 0-3 / 4-7  rows of tile A / B, one thread per row (its TMEM lane):
//                    mask, running max with a lazy reference, exponentials,
//                    sums, P; at the end of the item the write-back
//                    N_out = acc + 2^(m_in - m') N_in, O = N_out / Z', m, Z;
//   warps 8-11       the next item's queries: bf16 rows gathered by token,
//                    converted to fp16 and stored swizzled (fp16 range checked);
//   warp 12          TMEM allocation and the K / V TMA loads;
//   warp 13          MMA issue, alternating the tiles:
//                    S_A(0) S_B(0) | PV_A(t) S_A(t+1) | PV_B(t) S_B(t+1) | ...
//                    so that one tile's rows work while the tensor core serves
//                    the other.
// The numerator accumulates from zero within an item (the first P.V does not
// accumulate) and the previous state enters at the write-back, so an item
// starts as soon as its queries are in shared memory.  The running maximum is
// a per-row reference raised only when a tile's maximum exceeds it by 8 (log2
// units), keeping every exponential <= 2^8.  Every wait is bounded; a wait
// that gives up sets FLASHLOOP_DEVERR_TIMEOUT and the CTA unwinds.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "attn_args.cuh"
#include "common.cuh"
#include "tc_util.cuh"

namespace fl {

constexpr int kAdRows = 128;     // rows per tile (TMEM lanes)
constexpr int kAdCols = 64;      // selected columns per K / V tile
constexpr int kAdThreads = 448;  // 14 warps
constexpr int kAdWarpQ = 8;      // warps 8-11
constexpr int kAdWarpTma = 12;
constexpr int kAdWarpMma = 13;
constexpr float kAdLog2e = 1.4426950408889634f;
constexpr float kAdRescale = 8.f;

template <int DH>
struct AdCfg {
  static constexpr int kQChunk = kAdRows * 128;     // 128 rows x 128 B (64 elements)
  static constexpr int kQBytes = kAdRows * DH * 2;  // one query matrix
  static constexpr int kKChunk = kAdCols * 128;     // 64 rows x 128 B
  static constexpr int kKBytes = kAdCols * DH * 2;  // one K tile (64 x DH)
  static constexpr int kVBytes = DH * kAdCols * 2;  // one V^T tile (DH x 64)
  static constexpr int kSlotBytes = 2 * kKBytes;    // [K_new | K_old] or [V_new^T | V_old^T]
  static constexpr int kStages = DH == 128 ? 3 : 6;
  static constexpr int kRingOff = 4 * kQBytes;
  static constexpr int kBarOff = kRingOff + kStages * kSlotBytes;
  static constexpr int kSmem = 1024 + kBarOff + 512;
  static constexpr uint32_t kColS = 256;  // tile X: scores at 256 + 128 X; numerator at X * DH
  static constexpr uint32_t kIdescS = f16_idesc(128, kAdCols, 0);
  static constexpr uint32_t kIdescPV = f16_idesc(128, DH, 0);
  static_assert(kKBytes == kVBytes, "K and V^T tiles share the slot layout");
  static_assert(kSmem <= 232448, "shared memory per block");
};

struct AdArgs {
  int S, H, kc;
  const int32_t* rows;    // active tokens (NULL: identity)
  const int32_t* n_rows;  // device count (NULL: S)
  int row_cap;
  const int32_t* cols;    // [H, kc] ascending (NULL: identity)
  const uint16_t* q_new;  // bf16 [S, H*DH]
  const uint16_t* q_old;
  const float* m_in;      // [H, S]
  const float* z_in;
  const float* n_in;      // [H, S, DH]
  float* m_out;
  float* z_out;
  float* n_out;
  uint16_t* o;            // bf16 [S, H*DH]
  float* g_out;           // dense loop of the fixed-mass form: g = 1 (NULL otherwise)
  int32_t* err;
};

__device__ __forceinline__ int ad_count_le(const int32_t* cols, int n, int tok) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(cols + mid) <= tok) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// Column tiles that tile X (0 = A, 1 = B) of row pair p needs: the columns up
// to its last (largest) row token; 0 when the tile has no rows.
__device__ __forceinline__ int ad_tiles(const AdArgs& g, int h, int p, int X, int n_rows) {
  const int first = p * 2 * kAdRows + X * kAdRows;
  if (first >= n_rows) return 0;
  const int last = min(n_rows, first + kAdRows) - 1;
  int tok = g.rows ? __ldg(g.rows + last) : last;
  if (tok < 0) return 0;
  if (tok >= g.S) tok = g.S - 1;
  const int nc = g.cols ? ad_count_le(g.cols + (size_t)h * g.kc, g.kc, tok) : min(tok + 1, g.kc);
  return (nc + kAdCols - 1) / kAdCols;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];\n" ::"l"(p));
}

// 2^x on the FMA pipe, for x <= 8 (inputs below -125 give 2^-125): the
// Cody-Waite split x = n + f with n = rint(x), found by adding 1.5 * 2^23
// (the integer lands in the low mantissa bits), f in [-1/2, 1/2]; 2^f by a
// degree-3 polynomial whose coefficients were fitted for minimal relative
// error on that interval by a Remez exchange (7.5e-5, below half an fp16
// step); 2^n is added to the exponent field.  Part of a tile's exponentials
// take this path so that the MUFU unit and the FMA pipe share the work.
__device__ __forceinline__ float ex2_fma(float x) {
  x = fmaxf(x, -125.f);
  const float t = x + 12582912.f;
  const float n = t - 12582912.f;
  const float f = x - n;
  const float p = fmaf(fmaf(fmaf(0.0551716685f, f, 0.2426111251f), f, 0.6932609677f), f, 0.9999280572f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// One in kAdPolyEvery exponentials of a row's tile is evaluated by ex2_fma
// (0: all on the MUFU unit).
#ifndef FL_AD_POLY_EVERY
#define FL_AD_POLY_EVERY 0
#endif
constexpr int kAdPolyEvery = FL_AD_POLY_EVERY;

// Exponential of element e of a row's tile (e is a constant once the loops
// over a tile are unrolled, so the choice costs nothing at run time).
__device__ __forceinline__ float ad_exp2(float x, int e) {
  if (kAdPolyEvery > 0 && (e % kAdPolyEvery) == kAdPolyEvery - 1) return ex2_fma(x);
  return ex2(x);
}

template <int DH, bool DENSE>
__global__ void __launch_bounds__(kAdThreads, 1)
attn_dual_kernel(const __grid_constant__ CUtensorMap tm_kn, const __grid_constant__ CUtensorMap tm_ko,
                 const __grid_constant__ CUtensorMap tm_vn, const __grid_constant__ CUtensorMap tm_vo, AdArgs g) {
  using C = AdCfg<DH>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* kv_full = bars;                 // [stages] TMA bytes landed
  uint64_t* kv_empty = bars + C::kStages;   // [stages] MMAs done with the slot
  uint64_t* s_full = bars + 2 * C::kStages; // [2] scores of a tile in TMEM
  uint64_t* p_full = s_full + 2;            // [2] P of a tile written (128 row threads)
  uint64_t* pv_done = p_full + 2;           // [2] a tile's P.V completed
  uint64_t* acc_full = pv_done + 2;         // [2] the item's last P.V of a tile completed
  uint64_t* n_free = acc_full + 2;          // [2] the write-back has read the numerator (128 threads)
  uint64_t* q_full = n_free + 2;            // [2] a tile's queries stored (128 threads)
  uint64_t* q_empty = q_full + 2;           // [2] the item's S MMAs of a tile completed
  uint64_t* fin = q_empty + 2;              // [1] every MMA completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* ring = smem + C::kRingOff;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int n_rows = g.n_rows ? *g.n_rows : g.S;
  if (n_rows > g.row_cap) n_rows = g.row_cap;
  if (n_rows < 0) n_rows = 0;
  const int pairs = (n_rows + 2 * kAdRows - 1) / (2 * kAdRows);
  const int total = pairs * g.H;
  const int HD = g.H * DH;
  // item -> (head, row pair), head-major so that the CTAs in flight share a
  // head or two and its K / V tiles stay in L2; within a head the pairs with
  // the most column tiles come first
  auto item_h = [&](int item) { return item / pairs; };
  auto item_p = [&](int item) { return pairs - 1 - item % pairs; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], kAdRows);
      mbar_init(&pv_done[x], 1);
      mbar_init(&acc_full[x], 1);
      mbar_init(&n_free[x], kAdRows);
      mbar_init(&q_full[x], kAdRows);
      mbar_init(&q_empty[x], 1);
    }
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kAdWarpTma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&]() {
    set_error(g.err, kDevErrTimeout);
    *abort_flag = 1;
  };

  if (warp == kAdWarpTma) {
    // ------------------------------------------------------------ K / V loads
    if (lane == 0) {
      constexpr uint32_t kBytes = (DENSE ? 1 : 2) * C::kKBytes;
      int issued[C::kStages];
      for (int s = 0; s < C::kStages; ++s) issued[s] = -1;
      uint32_t seq = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
        const int h = item_h(item), p = item_p(item);
        const int nt = max(ad_tiles(g, h, p, 0, n_rows), ad_tiles(g, h, p, 1, n_rows));
        for (int t = 0; t < nt && ok; ++t) {
          for (int kv = 0; kv < 2; ++kv, ++seq) {
            const int slot = seq % C::kStages;
            const uint32_t ph = (seq / C::kStages) & 1;
            if (*abort_flag || !mbar_wait_sleep(&kv_empty[slot], ph ^ 1)) {
              fail();
              ok = false;
              break;
            }
            uint8_t* st = ring + slot * C::kSlotBytes;
            mbar_arrive_expect_tx(&kv_full[slot], kBytes);
            if (kv == 0) {
#pragma unroll
              for (int c = 0; c < DH / 64; ++c)
                tma_load_3d(st + c * C::kKChunk, &tm_kn, c * 64, t * kAdCols, h, &kv_full[slot]);
              if (!DENSE) {
#pragma unroll
                for (int c = 0; c < DH / 64; ++c)
                  tma_load_3d(st + C::kKBytes + c * C::kKChunk, &tm_ko, c * 64, t * kAdCols, h, &kv_full[slot]);
              }
            } else {
              tma_load_3d(st, &tm_vn, t * kAdCols, 0, h, &kv_full[slot]);
              if (!DENSE) tma_load_3d(st + C::kVBytes, &tm_vo, t * kAdCols, 0, h, &kv_full[slot]);
            }
            issued[slot] = (int)ph;
          }
        }
      }
      // never leave with a copy in flight: wait (bounded) for the last load of every slot
      for (int s = 0; s < C::kStages; ++s)
        if (issued[s] >= 0) (void)mbar_wait(&kv_full[s], (uint32_t)issued[s]);
    }
  } else if (warp == kAdWarpMma) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      uint32_t seq = 0, item_no = 0;
      uint32_t pc[2] = {0u, 0u};
      bool ok = true;
      auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        if (*abort_flag || !mbar_wait_sleep(bar, parity)) {
          fail();
          ok = false;
          return false;
        }
        tc_fence_after();
        return true;
      };
      auto slot_of = [&](uint32_t s) { return (int)(s % C::kStages); };
      auto par_of = [&](uint32_t s) { return (s / C::kStages) & 1u; };
      auto issue_s = [&](int x, int slot) {
        const uint32_t qn = smem_u32(smem + (2 * x) * C::kQBytes);
        const uint32_t qo = smem_u32(smem + (2 * x + 1) * C::kQBytes);
        const uint32_t kn = smem_u32(ring + slot * C::kSlotBytes);
        const uint32_t d = tmem + C::kColS + 128u * x;
#pragma unroll
        for (int ks = 0; ks < DH / 16; ++ks) {
          const uint32_t qoff = (ks >> 2) * C::kQChunk + (ks & 3) * 32;
          const uint32_t koff = (ks >> 2) * C::kKChunk + (ks & 3) * 32;
          umma_f16(d, sw128_kmajor_desc(qn + qoff), sw128_kmajor_desc(kn + koff), C::kIdescS, ks > 0);
          if (!DENSE)
            umma_f16(d + 64, sw128_kmajor_desc(qo + qoff), sw128_kmajor_desc(kn + C::kKBytes + koff), C::kIdescS,
                     ks > 0);
        }
      };
      auto issue_pv = [&](int x, int slot, bool acc) {
        const uint32_t v = smem_u32(ring + slot * C::kSlotBytes);
        const uint32_t pcol = tmem + C::kColS + 128u * x;
        const uint32_t d = tmem + (uint32_t)(x * DH);
#pragma unroll
        for (int ks = 0; ks < kAdCols / 16; ++ks)
          umma_f16_ts(d, pcol + ks * 8, sw128_kmajor_desc(v + ks * 32), C::kIdescPV, (acc || ks > 0) ? 1u : 0u);
        if (!DENSE) {
#pragma unroll
          for (int ks = 0; ks < kAdCols / 16; ++ks)
            umma_f16_ts(d, pcol + 32 + ks * 8, sw128_kmajor_desc(v + C::kVBytes + ks * 32), C::kIdescPV, 1u);
        }
      };
      for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++item_no) {
        const int h = item_h(item), p = item_p(item);
        const int ntx[2] = {ad_tiles(g, h, p, 0, n_rows), ad_tiles(g, h, p, 1, n_rows)};
        const int nt = max(ntx[0], ntx[1]);
        if (!wait(&q_full[0], item_no & 1) || !wait(&q_full[1], item_no & 1)) break;
        for (int x = 0; x < 2; ++x)
          if (ntx[x] == 0) umma_commit(&q_empty[x]);
        const uint32_t base = seq;
        if (nt > 0) {
          if (!wait(&kv_full[slot_of(base)], par_of(base))) break;
          for (int x = 0; x < 2; ++x) {
            if (ntx[x] == 0) continue;
            issue_s(x, slot_of(base));
            umma_commit(&s_full[x]);
            if (ntx[x] == 1) umma_commit(&q_empty[x]);
          }
          umma_commit(&kv_empty[slot_of(base)]);
        }
        for (int t = 0; t < nt && ok; ++t) {
          const uint32_t vs = base + 2 * t + 1, ks_next = base + 2 * t + 2;
          if (!wait(&kv_full[slot_of(vs)], par_of(vs))) break;
          bool k_next = false;
          for (int x = 0; x < 2 && ok; ++x) {
            if (t >= ntx[x]) continue;
            if (t == 0 && item_no > 0 && !wait(&n_free[x], (item_no - 1) & 1)) break;
            if (!wait(&p_full[x], pc[x] & 1)) break;
            ++pc[x];
            issue_pv(x, slot_of(vs), t > 0);
            umma_commit(&pv_done[x]);
            if (t == ntx[x] - 1) umma_commit(&acc_full[x]);
            if (t + 1 < ntx[x]) {
              if (!k_next) {
                if (!wait(&kv_full[slot_of(ks_next)], par_of(ks_next))) break;
                k_next = true;
              }
              issue_s(x, slot_of(ks_next));
              umma_commit(&s_full[x]);
              if (t + 1 == ntx[x] - 1) umma_commit(&q_empty[x]);
            }
          }
          if (!ok) break;
          umma_commit(&kv_empty[slot_of(vs)]);
          if (t + 1 < nt) umma_commit(&kv_empty[slot_of(ks_next)]);
        }
        if (!ok) break;
        for (int x = 0; x < 2 && ok; ++x) {
          if (ntx[x] != 0) continue;
          if (item_no > 0 && !wait(&n_free[x], (item_no - 1) & 1)) break;
          umma_commit(&acc_full[x]);
        }
        seq = base + 2 * nt;
      }
      // every MMA issued has completed before TMEM is released
      umma_commit(fin);
      (void)mbar_wait(fin, 0);
    }
  } else if (warp >= kAdWarpQ) {
    // ------------------------------------------------------------ queries
    const int row = (warp - kAdWarpQ) * 32 + lane;
    auto load_q = [&](int item, int x) {
      const int h = item_h(item), p = item_p(item);
      const int a = p * 2 * kAdRows + x * kAdRows + row;
      int tok = -1;
      if (a < n_rows) {
        tok = g.rows ? __ldg(g.rows + a) : a;
        if (tok < 0 || tok >= g.S) tok = -1;  // reported by the row threads
      }
      bool in_range = true;
#pragma unroll 1
      for (int mat = 0; mat < (DENSE ? 1 : 2); ++mat) {
        const uint16_t* src = (mat == 0 ? g.q_new : g.q_old) + (size_t)(tok < 0 ? 0 : tok) * HD + (size_t)h * DH;
        const uint32_t dst = smem_u32(smem + (2 * x + mat) * C::kQBytes) + row * 128;
        uint32_t qv[DH / 16][8];
#pragma unroll
        for (int v = 0; v < DH / 16; ++v) {
          if (tok >= 0) {
            ld_global_v8(src + v * 16, qv[v]);
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) qv[v][e] = 0u;
          }
        }
#pragma unroll
        for (int v = 0; v < DH / 16; ++v) {
          uint32_t hv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float2 f = bf16x2_to_float2(qv[v][e]);
            in_range = in_range && half_range_ok(f.x) && half_range_ok(f.y);
            hv[e] = bf16x2_to_half2_bits(qv[v][e]);
          }
          // elements [16v, 16v + 16): 16-byte units u and u + 1 of chunk 16v / 64
          const int chunk = (v * 16) / 64, u = ((v * 16) % 64) / 8;
          const uint32_t base = dst + chunk * C::kQChunk;
          st_shared_v4(base + ((u ^ (row & 7)) << 4), hv[0], hv[1], hv[2], hv[3]);
          st_shared_v4(base + (((u + 1) ^ (row & 7)) << 4), hv[4], hv[5], hv[6], hv[7]);
        }
      }
      if (!in_range) set_error(g.err, FLASHLOOP_DEVERR_RANGE);
      fence_proxy_async_smem();
    };
    uint32_t item_no = 0;
    if ((int)blockIdx.x < total) {
      for (int x = 0; x < 2; ++x) {
        load_q(blockIdx.x, x);
        mbar_arrive(&q_full[x]);
      }
    }
    bool ok = true;
    for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++item_no) {
      const int next = item + gridDim.x;
      if (next >= total) break;
      for (int x = 0; x < 2; ++x) {
        if (*abort_flag || !__all_sync(0xffffffffu, mbar_wait_sleep(&q_empty[x], item_no & 1))) {
          fail();
          ok = false;
          break;
        }
        load_q(next, x);
        mbar_arrive(&q_full[x]);
      }
    }
  } else {
    // ------------------------------------------------------------ rows
    const int x = warp >> 2, quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t sbase = tmem + lane_base + C::kColS + 128u * x;
    const uint32_t nbase = tmem + lane_base + (uint32_t)(x * DH);
    uint32_t u = 0, item_no = 0;
    bool ok = true;
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      if (*abort_flag || !__all_sync(0xffffffffu, mbar_wait_sleep(bar, parity))) {
        fail();
        ok = false;
        return false;
      }
      tc_fence_after();
      return true;
    };
    for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++item_no) {
      const int h = item_h(item), p = item_p(item);
      const int nt = ad_tiles(g, h, p, x, n_rows);
      const int a = p * 2 * kAdRows + x * kAdRows + row;
      int tok = -1;
      if (a < n_rows) {
        tok = g.rows ? __ldg(g.rows + a) : a;
        if (tok < 0 || tok >= g.S) {
          set_error(g.err, FLASHLOOP_DEVERR_INDEX);
          tok = -1;
        }
      }
      const size_t hi = (size_t)h * g.S + (tok < 0 ? 0 : tok);
      float m_start = 0.f, z = 0.f;
      if (tok >= 0) {
        if (DENSE) {
          m_start = -INFINITY;
        } else {
          m_start = g.m_in[hi] * kAdLog2e;
          z = g.z_in[hi];
          const float* nrow = g.n_in + hi * DH;
#pragma unroll
          for (int c = 0; c < DH * 4; c += 128) prefetch_l2(nrow + c / 4);
        }
      }
      float m_ref = m_start;
      const int32_t* hcols = g.cols ? g.cols + (size_t)h * g.kc : nullptr;
      int wmin = tok < 0 ? 0x7fffffff : tok;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) wmin = min(wmin, __shfl_xor_sync(0xffffffffu, wmin, o));
      for (int t = 0; t < nt; ++t, ++u) {
        const int c0 = t * kAdCols;
        const int c_end = min(c0 + kAdCols, g.kc);
        const int last_tok = hcols ? __ldg(hcols + c_end - 1) : c_end - 1;
        int nvalid = kAdCols;
        if (c0 + kAdCols > g.kc || last_tok > wmin) {
          // the valid columns of this tile for this row form a prefix (columns ascend)
          if (tok < 0) {
            nvalid = 0;
          } else {
            int lo = c0, hi2 = c_end;
            while (lo < hi2) {
              const int mid = (lo + hi2) >> 1;
              const int ct = hcols ? __ldg(hcols + mid) : mid;
              if (ct <= tok) lo = mid + 1;
              else hi2 = mid;
            }
            nvalid = lo - c0;
          }
        }
        if (!wait(&s_full[x], u & 1)) break;
        uint32_t s[64];
        {
          uint32_t (&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[0]);
          uint32_t (&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32]);
          tmem_ld32(sbase, s0);
          tmem_ld32(sbase + 32, s1);
          tmem_wait_ld();
        }
        if (nvalid < kAdCols) {
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (e >= nvalid) s[e] = 0xff800000u;  // -inf
        }
        float t32[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) t32[e] = fmaxf(__uint_as_float(s[e]), __uint_as_float(s[e + 32]));
#pragma unroll
        for (int w = 16; w > 0; w >>= 1)
#pragma unroll
          for (int e = 0; e < w; ++e) t32[e] = fmaxf(t32[e], t32[e + w]);
        const float mx = t32[0];
        const bool need = mx > m_ref + kAdRescale;
        if (__any_sync(0xffffffffu, need)) {
          // raise the reference: the numerator accumulated in this item and Z
          // scale by 2^(m_ref - mx); the previous numerator enters later,
          // scaled from m_start
          const float new_ref = need ? mx : m_ref;
          const float f = need ? ex2(m_ref - new_ref) : 1.f;
          if (t > 0) {
            if (!wait(&pv_done[x], (u - 1) & 1)) break;
#pragma unroll 1
            for (int cc = 0; cc < DH; cc += 16) {
              uint32_t r[16];
              tmem_ld16(nbase + cc, r);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * f);
              tmem_st16(nbase + cc, r);
            }
            tmem_wait_st();
          }
          z *= f;
          m_ref = new_ref;
        }
        const float mr = tok < 0 ? 0.f : m_ref;
        float za[4] = {0.f, 0.f, 0.f, 0.f};
        {
          uint32_t pk[32];
#pragma unroll
          for (int e2 = 0; e2 < 32; ++e2) {
            const float p0 = ad_exp2(__uint_as_float(s[2 * e2]) - mr, 2 * e2);
            const float p1 = ad_exp2(__uint_as_float(s[2 * e2 + 1]) - mr, 2 * e2 + 1);
            za[e2 & 3] += p0 + p1;
            pk[e2] = pack_half2(p0, p1);
          }
          tmem_st32(sbase, pk);
        }
        float zb[4] = {0.f, 0.f, 0.f, 0.f};
        if (!DENSE) {
          {
            uint32_t (&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[0]);
            uint32_t (&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32]);
            tmem_ld32(sbase + 64, s0);
            tmem_ld32(sbase + 96, s1);
            tmem_wait_ld();
          }
          if (nvalid < kAdCols) {
#pragma unroll
            for (int e = 0; e < 64; ++e)
              if (e >= nvalid) s[e] = 0xff800000u;
          }
          uint32_t pk[32];
#pragma unroll
          for (int e2 = 0; e2 < 32; ++e2) {
            const float p0 = ad_exp2(__uint_as_float(s[2 * e2]) - mr, 2 * e2);
            const float p1 = ad_exp2(__uint_as_float(s[2 * e2 + 1]) - mr, 2 * e2 + 1);
            zb[e2 & 3] += p0 + p1;
            pk[e2] = pack_half2(-p0, -p1);
          }
          tmem_st32(sbase + 32, pk);
        }
        z += ((za[0] + za[1]) + (za[2] + za[3])) - ((zb[0] + zb[1]) + (zb[2] + zb[3]));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[x]);
      }
      if (!ok) break;
      // write-back: N_out = acc + 2^(m_start - m') N_in, O = N_out / Z'
      if (!wait(&acc_full[x], item_no & 1)) break;
      const float nscale = (DENSE || tok < 0) ? 0.f : ex2(m_start - m_ref);
      const float inv = 1.f / z;
#pragma unroll 1
      for (int cc = 0; cc < DH; cc += 32) {
        uint32_t r[32];
        if (nt > 0) {
          tmem_ld32(nbase + cc, r);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = 0u;
        }
        if (tok >= 0) {
          float* nd = g.n_out + hi * DH + cc;
          if (!DENSE) {
            const float* ns = g.n_in + hi * DH + cc;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint32_t w[8];
              ld_global_v8(ns + 8 * v, w);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                r[8 * v + e] = __float_as_uint(fmaf(nscale, __uint_as_float(w[e]), __uint_as_float(r[8 * v + e])));
            }
          }
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint32_t w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) w[e] = r[8 * v + e];
            st_global_v8(nd + 8 * v, w);
          }
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            uint32_t w[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
              w[q] = (uint32_t)float_to_bf16_bits(__uint_as_float(r[16 * v + 2 * q]) * inv) |
                     ((uint32_t)float_to_bf16_bits(__uint_as_float(r[16 * v + 2 * q + 1]) * inv) << 16);
            st_global_v8(g.o + (size_t)tok * HD + (size_t)h * DH + cc + 16 * v, w);
          }
        }
      }
      if (tok >= 0) {
        g.m_out[hi] = m_ref / kAdLog2e;
        g.z_out[hi] = z;
        if (DENSE && g.g_out) g.g_out[hi] = 1.f;
      }
      tc_fence_before();
      mbar_arrive(&n_free[x]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kAdWarpTma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int make_tmap_f16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t p1,
                     uint64_t p2, uint32_t b0, uint32_t b1);
int at_sm_count();

// The running update (and the dense loop 1) with two row tiles per CTA.
// K buffers are [H, kcp, dh], V^T buffers [H, dh, kcp] (fp16), kcp = kc rounded up to 8.
int launch_attn_dual(const flashloop_params* p, const AttnArgs& a, int kcp, cudaStream_t stream) {
  const int dh = p->head_dim, H = p->n_heads;
  const void* aligned32[] = {a.q_new, a.q_old, a.n_in, a.n_out, a.o};
  for (const void* ptr : aligned32)
    if (ptr != nullptr && reinterpret_cast<uintptr_t>(ptr) % 32 != 0) return FLASHLOOP_ERR_INVALID_ARG;
  CUtensorMap tkn, tko, tvn, tvo;
  int rc = make_tmap_f16_3d(&tkn, a.k_new, dh, a.kc, H, dh, (uint64_t)kcp * dh, 64, kAdCols);
  if (rc == FLASHLOOP_OK) rc = make_tmap_f16_3d(&tvn, a.v_new, a.kc, dh, H, kcp, (uint64_t)kcp * dh, kAdCols, dh);
  if (rc == FLASHLOOP_OK && !a.dense) {
    rc = make_tmap_f16_3d(&tko, a.k_old, dh, a.kc, H, dh, (uint64_t)kcp * dh, 64, kAdCols);
    if (rc == FLASHLOOP_OK) rc = make_tmap_f16_3d(&tvo, a.v_old, a.kc, dh, H, kcp, (uint64_t)kcp * dh, kAdCols, dh);
  } else {
    tko = tkn;
    tvo = tvn;
  }
  if (rc != FLASHLOOP_OK) return rc;
  AdArgs g{};
  g.S = a.S; g.H = a.H; g.kc = a.kc; g.rows = a.rows; g.n_rows = a.n_rows; g.row_cap = a.row_cap;
  g.cols = a.cols; g.q_new = a.q_new; g.q_old = a.dense ? a.q_new : a.q_old; g.m_in = a.m_in; g.z_in = a.z_in;
  g.n_in = a.n_in; g.m_out = a.m_out; g.z_out = a.z_out; g.n_out = a.n_out; g.o = a.o;
  g.g_out = a.dense ? a.g_out : nullptr; g.err = a.err;
  const int max_items = ((a.row_cap + 2 * kAdRows - 1) / (2 * kAdRows)) * H;
  int grid = at_sm_count();
  if (grid > max_items) grid = max_items;
  if (grid < 1) grid = 1;
  auto launch = [&](auto kernel, int smem) -> int {
    FL_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    kernel<<<grid, kAdThreads, smem, stream>>>(tkn, tko, tvn, tvo, g);
    return FLASHLOOP_OK;
  };
  if (dh == 128) rc = a.dense ? launch(attn_dual_kernel<128, true>, AdCfg<128>::kSmem)
                              : launch(attn_dual_kernel<128, false>, AdCfg<128>::kSmem);
  else rc = a.dense ? launch(attn_dual_kernel<64, true>, AdCfg<64>::kSmem)
                    : launch(attn_dual_kernel<64, false>, AdCfg<64>::kSmem);
  if (rc != FLASHLOOP_OK) return rc;
  return launch_status();
}

}  // namespace fl
