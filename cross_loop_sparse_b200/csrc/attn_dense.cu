// The dense loop-1 attention [FlashLoop App. D.1: the early loops run dense]
// on the sm_100a tensor cores: for every token i and every column j <= i,
//   m_i = max_j s_ij,  Z_i = sum_j e^(s_ij - m_i),  N_i = sum_j e^(s_ij - m_i) Vhat_j,
//   s_ij = q_i . Khat_j / sqrt(dh),  O_i = N_i / Z_i,
// over the reconstructed loop-1 base (the keys arrive scaled by
// log2(e)/sqrt(dh), so scores are in log2 units).  The column mass that ranks
// loop 2's selection is a separate pass (colmass_tc_kernel).
//
// Work item: one head and 256 consecutive tokens, as two 128-row tiles A and
// B that share every K / V tile of 128 columns (loaded once per item).
// Shared memory: the item's queries (fp16, 128-byte swizzled K-major, 2 x 128
// x DH) and a ring of five K / V slots of 128 columns, a slot holding a K tile
// (128 x DH) or a V^T tile (DH x 128), filled by TMA.
// TMEM (512 columns): N_A, N_B (float32, DH columns each), then per tile a
// 128-column score region of two 64-column halves; the P of a half (fp16
// pairs, 32 columns) is written over the first columns of its scores and
// feeds that half's P.V MMA from TMEM.
//
// Each K / V tile is taken as two halves of 64 columns, each with its own
// score MMA (M128 N64), its own P and its own P.V (K = 64), so the scores of
// the next tile's first half are computed while the rows work on the second
// half of this one: the rows never wait for a whole P.V + score round trip.
//
// Roles (15 warps):
//   warps 0-3 / 4-7  rows of tile A / B, one thread per row (its TMEM lane),
//                    per half: the causal mask, the running maximum (a per-row
//                    reference raised only when a half's maximum exceeds it by
//                    8 in log2 units; raising it rescales the numerator once
//                    the P.V of the previous half has completed), exponentials,
//                    sums and P; at the end of the item the write-back
//                    O = N / Z, N, m, Z;
//   warps 8-11       the next item's queries: bf16 rows converted to fp16 and
//                    stored swizzled (fp16 range checked);
//   warp 12          TMEM allocation and the K / V TMA loads;
//   warps 13 / 14    MMA issue for tile A / B (one thread each: a thread that
//                    issues tcgen05.mma waits while the tensor pipe takes its
//                    MMAs, so each tile has its own issuer), in the order
//                    PV(t, 0) S(t+1, 0) PV(t, 1) S(t+1, 1); a K / V slot is
//                    released when both issuers are done with it.
// Every wait is bounded; a wait that gives up sets FLASHLOOP_DEVERR_TIMEOUT and
// the CTA unwinds.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "attn_args.cuh"
#include "common.cuh"
#include "tc_util.cuh"

namespace fl {

constexpr int kDnRows = 128;     // rows per tile (TMEM lanes)
constexpr int kDnCols = 128;     // columns per K / V tile
constexpr int kDnThreads = 480;  // 15 warps
constexpr int kDnWarpQ = 8;      // warps 8-11
constexpr int kDnWarpTma = 12;
constexpr int kDnWarpMma = 13;   // warps 13 (tile A) and 14 (tile B)
constexpr float kDnLog2e = 1.4426950408889634f;
constexpr float kDnRescale = 8.f;

template <int DH>
struct DnCfg {
  static constexpr int kQChunk = kDnRows * 128;     // 128 rows x 128 B (64 elements)
  static constexpr int kQBytes = kDnRows * DH * 2;  // one tile's queries
  static constexpr int kKChunk = kDnCols * 128;     // K tile: 128 rows x 128 B per 64 elements of dh
  static constexpr int kVChunk = DH * 128;          // V^T tile: DH rows x 128 B per 64 columns
  static constexpr int kSlotBytes = kDnCols * DH * 2;
  static constexpr int kStages = DH == 128 ? 5 : 10;
  static constexpr int kRingOff = 2 * kQBytes;
  static constexpr int kBarOff = kRingOff + kStages * kSlotBytes;
  static constexpr int kSmem = 1024 + kBarOff + 512;
  static constexpr uint32_t kColS = 256;  // tile X: scores at 256 + 128 X (half h at +64 h); numerator at X * DH
  static constexpr uint32_t kIdescS = f16_idesc(128, 64, 0);
  static constexpr uint32_t kIdescPV = f16_idesc(128, DH, 0);
  static_assert(kSmem <= 232448, "shared memory per block");
  static_assert((2 * kStages + 21) * 8 + 8 <= 512, "barriers");
};

struct DnArgs {
  int S, H;
  const uint16_t* q;  // bf16 [S, H*DH]
  float* m_out;       // [H, S]
  float* z_out;
  float* n_out;       // [H, S, DH]
  uint16_t* o;        // bf16 [S, H*DH]
  float* g_out;       // fixed-mass form: g = 1 (NULL otherwise)
  int32_t* err;
};

__device__ __forceinline__ void dn_st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// Column tiles of tile X (0 = A, 1 = B) of row pair p: columns up to its last token.
__device__ __forceinline__ int dn_tiles(int S, int p, int X) {
  const int first = p * 2 * kDnRows + X * kDnRows;
  if (first >= S) return 0;
  const int last = min(S, first + kDnRows) - 1;
  return (last + kDnCols) / kDnCols;
}

template <int DH>
__global__ void __launch_bounds__(kDnThreads, 1)
attn_dense_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, DnArgs g) {
  using C = DnCfg<DH>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* kv_full = bars;                 // [stages] TMA bytes landed
  uint64_t* kv_empty = bars + C::kStages;   // [stages] both issuers done with the slot (2 arrivals)
  uint64_t* s_full = bars + 2 * C::kStages; // [X * 2 + h] scores of a half in TMEM
  uint64_t* p_full = s_full + 4;            // [X * 2 + h] P of a half written (128 row threads)
  uint64_t* pv_done = p_full + 4;           // [X] a half's P.V completed (two completions per tile)
  uint64_t* acc_full = pv_done + 2;         // [X] the item's last P.V of a tile completed
  uint64_t* n_free = acc_full + 2;          // [X] the write-back has read the numerator (128 threads)
  uint64_t* q_full = n_free + 2;            // [X] a tile's queries stored (128 threads)
  uint64_t* q_empty = q_full + 2;           // [X] the item's S MMAs of a tile completed
  uint64_t* fin = q_empty + 2;              // [1] every MMA of both issuers completed (2 commits)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* ring = smem + C::kRingOff;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pairs = (g.S + 2 * kDnRows - 1) / (2 * kDnRows);
  const int total = pairs * g.H;
  const int HD = g.H * DH;
  // item -> (head, row pair), head-major; within a head the pairs with the
  // most column tiles first
  auto item_h = [&](int item) { return item / pairs; };
  auto item_p = [&](int item) { return pairs - 1 - item % pairs; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 2);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], kDnRows);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&pv_done[x], 1);
      mbar_init(&acc_full[x], 1);
      mbar_init(&n_free[x], kDnRows);
      mbar_init(&q_full[x], kDnRows);
      mbar_init(&q_empty[x], 1);
    }
    mbar_init(fin, 2);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kDnWarpTma) {
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

  if (warp == kDnWarpTma) {
    // ------------------------------------------------------------ K / V loads
    if (lane == 0) {
      int issued[C::kStages];
      for (int s = 0; s < C::kStages; ++s) issued[s] = -1;
      uint32_t seq = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
        const int h = item_h(item), p = item_p(item);
        const int nt = max(dn_tiles(g.S, p, 0), dn_tiles(g.S, p, 1));
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
            mbar_arrive_expect_tx(&kv_full[slot], C::kSlotBytes);
            if (kv == 0) {
#pragma unroll
              for (int c = 0; c < DH / 64; ++c)
                tma_load_3d(st + c * C::kKChunk, &tm_k, c * 64, t * kDnCols, h, &kv_full[slot]);
            } else {
#pragma unroll
              for (int c = 0; c < kDnCols / 64; ++c)
                tma_load_3d(st + c * C::kVChunk, &tm_v, t * kDnCols + c * 64, 0, h, &kv_full[slot]);
            }
            issued[slot] = (int)ph;
          }
        }
      }
      // never leave with a copy in flight: wait (bounded) for the last load of every slot
      for (int s = 0; s < C::kStages; ++s)
        if (issued[s] >= 0) (void)mbar_wait(&kv_full[s], (uint32_t)issued[s]);
    }
  } else if (warp == kDnWarpMma || warp == kDnWarpMma + 1) {
    // ------------------------------------------------------------ MMA issue, one thread per tile
    if (lane == 0) {
      const int x = warp - kDnWarpMma;
      uint32_t seq = 0, item_no = 0, u = 0;
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
      const uint32_t q = smem_u32(smem + x * C::kQBytes);
      const uint32_t scol = tmem + C::kColS + 128u * x;
      // S(., hf) = Q K[64 hf, 64 hf + 64)^T into the half's 64 columns
      auto issue_s = [&](int slot, int hf) {
        const uint32_t k = smem_u32(ring + slot * C::kSlotBytes) + hf * 64 * 128;
#pragma unroll
        for (int ks = 0; ks < DH / 16; ++ks)
          umma_f16(scol + 64u * hf, sw128_kmajor_desc(q + (ks >> 2) * C::kQChunk + (ks & 3) * 32),
                   sw128_kmajor_desc(k + (ks >> 2) * C::kKChunk + (ks & 3) * 32), C::kIdescS, ks > 0);
      };
      // N += P(., hf) V[64 hf, 64 hf + 64)
      auto issue_pv = [&](int slot, int hf, bool acc) {
        const uint32_t v = smem_u32(ring + slot * C::kSlotBytes) + hf * C::kVChunk;
        const uint32_t pcol = scol + 64u * hf;
        const uint32_t d = tmem + (uint32_t)(x * DH);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          umma_f16_ts(d, pcol + ks * 8, sw128_kmajor_desc(v + ks * 32), C::kIdescPV, (acc || ks > 0) ? 1u : 0u);
      };
      // a slot this tile does not read: released once its load has landed
      auto skip = [&](uint32_t s) -> bool {
        if (!wait(&kv_full[slot_of(s)], par_of(s))) return false;
        mbar_arrive(&kv_empty[slot_of(s)]);
        return true;
      };
      for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++item_no) {
        const int p = item_p(item);
        const int my = dn_tiles(g.S, p, x);
        const int nt = max(dn_tiles(g.S, p, 0), dn_tiles(g.S, p, 1));
        if (!wait(&q_full[x], item_no & 1)) break;
        if (my == 0) umma_commit(&q_empty[x]);
        const uint32_t base = seq;
        if (nt > 0) {
          if (my > 0) {
            if (!wait(&kv_full[slot_of(base)], par_of(base))) break;
            for (int hf = 0; hf < 2; ++hf) {
              issue_s(slot_of(base), hf);
              umma_commit(&s_full[2 * x + hf]);
            }
            if (my == 1) umma_commit(&q_empty[x]);
            umma_commit(&kv_empty[slot_of(base)]);
          } else if (!skip(base)) {
            break;
          }
        }
        for (int t = 0; t < nt && ok; ++t) {
          const uint32_t vs = base + 2 * t + 1, ks_next = base + 2 * t + 2;
          if (t >= my) {
            if (!skip(vs)) break;
            if (t + 1 < nt && !skip(ks_next)) break;
            continue;
          }
          if (!wait(&kv_full[slot_of(vs)], par_of(vs))) break;
          for (int hf = 0; hf < 2 && ok; ++hf, ++u) {
            if (t == 0 && hf == 0 && item_no > 0 && !wait(&n_free[x], (item_no - 1) & 1)) break;
            if (!wait(&p_full[2 * x + hf], (u >> 1) & 1)) break;
            issue_pv(slot_of(vs), hf, t > 0 || hf > 0);
            umma_commit(&pv_done[x]);
            if (t == my - 1 && hf == 1) umma_commit(&acc_full[x]);
            if (t + 1 < my) {
              if (hf == 0 && !wait(&kv_full[slot_of(ks_next)], par_of(ks_next))) break;
              issue_s(slot_of(ks_next), hf);
              umma_commit(&s_full[2 * x + hf]);
              if (t + 1 == my - 1 && hf == 1) umma_commit(&q_empty[x]);
            }
          }
          if (!ok) break;
          umma_commit(&kv_empty[slot_of(vs)]);
          if (t + 1 < nt) {
            if (t + 1 < my) {
              umma_commit(&kv_empty[slot_of(ks_next)]);
            } else if (!skip(ks_next)) {
              break;
            }
          }
        }
        if (!ok) break;
        if (my == 0) {
          if (item_no > 0 && !wait(&n_free[x], (item_no - 1) & 1)) break;
          umma_commit(&acc_full[x]);
        }
        seq = base + 2 * nt;
      }
      // every MMA issued has completed before TMEM is released
      umma_commit(fin);
      (void)mbar_wait(fin, 0);
    }
  } else if (warp >= kDnWarpQ) {
    // ------------------------------------------------------------ queries
    const int row = (warp - kDnWarpQ) * 32 + lane;
    auto load_q = [&](int item, int x) {
      const int h = item_h(item), p = item_p(item);
      const int tok = p * 2 * kDnRows + x * kDnRows + row;
      const bool valid = tok < g.S;
      const uint16_t* src = g.q + (size_t)(valid ? tok : 0) * HD + (size_t)h * DH;
      const uint32_t dst = smem_u32(smem + x * C::kQBytes) + row * 128;
      bool in_range = true;
      uint32_t qv[DH / 16][8];
#pragma unroll
      for (int v = 0; v < DH / 16; ++v) {
        if (valid) {
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
        dn_st_shared_v4(base + ((u ^ (row & 7)) << 4), hv[0], hv[1], hv[2], hv[3]);
        dn_st_shared_v4(base + (((u + 1) ^ (row & 7)) << 4), hv[4], hv[5], hv[6], hv[7]);
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
    uint32_t u = 0, item_no = 0;  // u: halves of this tile so far (two per column tile)
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
      const int nt = dn_tiles(g.S, p, x);
      const int tok0 = p * 2 * kDnRows + x * kDnRows + row;
      const int tok = tok0 < g.S ? tok0 : -1;
      float m_ref = -INFINITY, z = 0.f;
      for (int t = 0; t < nt && ok; ++t) {
#pragma unroll 1
        for (int hf = 0; hf < 2; ++hf, ++u) {
          if (!wait(&s_full[2 * x + hf], (u >> 1) & 1)) break;
          // columns [128t + 64hf, +64): the valid ones (j <= tok) form a prefix
          const int nvalid = tok < 0 ? 0 : min(max(tok + 1 - (t * kDnCols + 64 * hf), 0), 64);
          const uint32_t shalf = sbase + 64u * hf;
          uint32_t s[64];
          {
            uint32_t (&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[0]);
            uint32_t (&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32]);
            tmem_ld32(shalf, s0);
            tmem_ld32(shalf + 32, s1);
            tmem_wait_ld();
          }
          if (nvalid < 64) {
#pragma unroll
            for (int e = 0; e < 64; ++e)
              if (e >= nvalid) s[e] = 0xff800000u;  // -inf
          }
          const float mx = max64(s);
          const bool need = mx > m_ref + kDnRescale;
          if (__any_sync(0xffffffffu, need)) {
            // raise the reference: the numerator accumulated so far and Z
            // scale by 2^(m_ref - mx); the numerator once the previous half's
            // P.V (the last one issued for this tile) has completed
            const float new_ref = need ? mx : m_ref;
            const float f = need ? ex2(m_ref - new_ref) : 1.f;
            if (t > 0 || hf > 0) {
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
            }
            z *= f;
            m_ref = new_ref;
          }
          const float mr = tok < 0 ? 0.f : m_ref;
          float za[4] = {0.f, 0.f, 0.f, 0.f};
          uint32_t pk[32];
#pragma unroll
          for (int e2 = 0; e2 < 32; ++e2) {
            float x0 = __uint_as_float(s[2 * e2]), x1 = __uint_as_float(s[2 * e2 + 1]);
            sub2_rn(x0, x1, mr);
            const float p0 = ex2(x0), p1 = ex2(x1);
            if (e2 & 1) add2_rn(za[2], za[3], p0, p1);
            else add2_rn(za[0], za[1], p0, p1);
            pk[e2] = pack_half2(p0, p1);
          }
          tmem_st32(shalf, pk);
          z += (za[0] + za[1]) + (za[2] + za[3]);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&p_full[2 * x + hf]);
        }
      }
      if (!ok) break;
      // write-back: O = N / Z, N, m, Z
      if (!wait(&acc_full[x], item_no & 1)) break;
      const float inv = 1.f / z;
      const size_t hi = (size_t)h * g.S + (tok < 0 ? 0 : tok);
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
        g.m_out[hi] = m_ref / kDnLog2e;
        g.z_out[hi] = z;
        if (g.g_out) g.g_out[hi] = 1.f;
      }
      tc_fence_before();
      mbar_arrive(&n_free[x]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kDnWarpTma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int make_tmap_f16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t p1,
                     uint64_t p2, uint32_t b0, uint32_t b1);
int at_sm_count();

// The dense loop-1 attention: keys [H, kcp, dh], values transposed [H, dh, kcp]
// (fp16, kcp = S rounded up to 8), the identity selection.
int launch_attn_dense(const flashloop_params* p, const AttnArgs& a, int kcp, cudaStream_t stream) {
  const int dh = p->head_dim, H = p->n_heads;
  if (!a.dense || a.rows != nullptr || a.cols != nullptr) return FLASHLOOP_ERR_INVALID_ARG;
  const void* aligned32[] = {a.q_new, a.n_out, a.o};
  for (const void* ptr : aligned32)
    if (reinterpret_cast<uintptr_t>(ptr) % 32 != 0) return FLASHLOOP_ERR_INVALID_ARG;
  CUtensorMap tk, tv;
  int rc = make_tmap_f16_3d(&tk, a.k_new, dh, a.kc, H, dh, (uint64_t)kcp * dh, 64, kDnCols);
  if (rc == FLASHLOOP_OK) rc = make_tmap_f16_3d(&tv, a.v_new, a.kc, dh, H, kcp, (uint64_t)kcp * dh, 64, dh);
  if (rc != FLASHLOOP_OK) return rc;
  DnArgs g{};
  g.S = a.S; g.H = H; g.q = a.q_new; g.m_out = a.m_out; g.z_out = a.z_out; g.n_out = a.n_out; g.o = a.o;
  g.g_out = a.g_out; g.err = a.err;
  const int max_items = ((a.S + 2 * kDnRows - 1) / (2 * kDnRows)) * H;
  int grid = at_sm_count();
  if (grid > max_items) grid = max_items;
  if (grid < 1) grid = 1;
  if (dh == 128) {
    FL_TRY(cudaFuncSetAttribute(attn_dense_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, DnCfg<128>::kSmem));
    attn_dense_kernel<128><<<grid, kDnThreads, DnCfg<128>::kSmem, stream>>>(tk, tv, g);
  } else {
    FL_TRY(cudaFuncSetAttribute(attn_dense_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, DnCfg<64>::kSmem));
    attn_dense_kernel<64><<<grid, kDnThreads, DnCfg<64>::kSmem, stream>>>(tk, tv, g);
  }
  return launch_status();
}

}  // namespace fl
