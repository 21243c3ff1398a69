// Sparse attention update (and the dense loop-1 attention) on SM pairs:
// tcgen05.mma with cta_group::2, 256 rows per tile, each SM holding 128 of
// them and half of every K / V tile.
//
// [FlashLoop §3.2, §4.2, App. D.2]: the same update as attn_tc.cu (running
// (m, N, Z) state, lazy reference, P = [e_new | -e_old]).  What changes is
// where the operands live.  Two CTAs of a cluster take row tiles 2p and
// 2p + 1 of one head.  Each keeps its 128 rows' Q, N and S in its own TMEM.
// Each loads, per 64-column tile, the keys [32 c, 32 c + 32) of K_new and
// K_old and the head-dim rows [DH/2 c, DH/2 (c + 1)) of V_new^T and V_old^T
// (c = its rank in the pair): 32 KB per SM and tile instead of 64 KB.  One
// thread of CTA 0 issues M = 256 MMAs that read A (Q, then P) from both CTAs'
// TMEM and B from both CTAs' shared memory and write both CTAs' TMEM.
// Loads land in the loading CTA's shared memory and count on CTA 0's
// barrier (cta_group::2 bulk tensor loads, no multicast); a tcgen05.commit
// to each CTA's barrier signals both.  Row warps of CTA 1 report to CTA 0
// with remote mbarrier arrivals.  All waits are bounded.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "attn_args.cuh"
#include "common.cuh"
#include "tc_util.cuh"

namespace fl {

constexpr int k2Rows = 128, k2Cols = 64, k2Stages = 6, k2Threads = 320;
constexpr int k2TmaWarp = 8, k2MmaWarp = 9;
constexpr float k2Log2e = 1.4426950408889634f;
constexpr float k2RescaleThreshold = 8.f;

template <int DH>
struct A2Cfg {
  static constexpr int kKHalf = (k2Cols / 2) * DH * 2;   // 32 keys x DH, DH/64 swizzle chunks of 4 KB
  static constexpr int kVHalf = (DH / 2) * k2Cols * 2;   // DH/2 rows of V^T x 64 keys
  static constexpr int kKChunk = (k2Cols / 2) * 128;     // one 64-element swizzle chunk of the K half
  static constexpr int kStageBytes = 2 * kKHalf + 2 * kVHalf;  // K_new | K_old | V_new^T | V_old^T halves
  static constexpr int kSmem = 1024 + k2Stages * kStageBytes + 512 + 8 * 128 * 4;
  static constexpr uint32_t kColQn = 0;
  static constexpr uint32_t kColQo = DH / 2;
  static constexpr uint32_t kColN = DH;
  static constexpr uint32_t kColS = 2 * DH;  // buffer b: S_new at kColS + 128 b, S_old at +64
  static constexpr uint32_t kIdescS = f16_idesc(256, k2Cols, 0);
  static constexpr uint32_t kIdescPV = f16_idesc(256, DH, 0);
};

// ---------------------------------------------------------------- pair PTX
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Arrival on a barrier of either CTA of the pair (default semantics: what it
// orders are the arriving thread's TMEM stores, through tcgen05 fences).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];\n" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(slot)),
               "r"(ncols));
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;\n" ::);
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols));
}
// D (+)= A * B over the pair: A from TMEM (each CTA its 128 rows), B from
// shared memory (each CTA half of N), D into each CTA's TMEM.
__device__ __forceinline__ void umma_f16_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8, %9, %10, %11, %12}, p;\n\t}\n"
      ::"r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u),
      "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}
// Arrive on the barrier at this offset in both CTAs once the issued MMAs
// complete: one commit per CTA, the second addressed to the peer's copy.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  const uint32_t own = smem_u32(bar);
  const uint32_t peer = mapa_shared(own, 1);
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(own) : "memory");
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(peer) : "memory");
}
// 3-D tile load into this CTA's shared memory, bytes counted on `bar_cluster`
// (a barrier of either CTA of the pair).
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const void* tmap, int x, int y, int z,
                                                 uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];\n"
      ::"r"(smem_u32(dst)), "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(bar_cluster)
      : "memory");
}

struct A2Args {
  int S, H, kc, dense;
  const int32_t* rows;
  const int32_t* n_rows;
  int row_cap;
  const int32_t* cols;
  const uint16_t* q_new;
  const uint16_t* q_old;
  const float* m_in;
  const float* z_in;
  const float* n_in;
  float* m_out;
  float* z_out;
  float* n_out;
  uint16_t* o;
  int32_t* err;
  float* g_out;  // [H, S] selected-column factor, set to 1 by the dense loop (fixed-mass runs), or NULL
};

// Column tiles a pair needs: columns up to the pair's last row token.
__device__ __forceinline__ int a2_tiles(const A2Args& g, int h, int rp, int n_rows) {
  const int last = min(n_rows, (rp + 1) * 2 * k2Rows) - 1;
  int tok = g.rows ? __ldg(g.rows + last) : last;
  if (tok < 0) return 0;
  if (tok >= g.S) tok = g.S - 1;
  int nc;
  if (g.cols) {
    const int32_t* c = g.cols + (size_t)h * g.kc;
    int lo = 0, hi = g.kc;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(c + mid) <= tok) lo = mid + 1;
      else hi = mid;
    }
    nc = lo;
  } else {
    nc = min(tok + 1, g.kc);
  }
  return (nc + k2Cols - 1) / k2Cols;
}

template <int DH>
__global__ void __launch_bounds__(k2Threads, 1)
attn_pair_kernel(const __grid_constant__ CUtensorMap tm_kn, const __grid_constant__ CUtensorMap tm_ko,
                 const __grid_constant__ CUtensorMap tm_vn, const __grid_constant__ CUtensorMap tm_vo, A2Args g) {
  using C = A2Cfg<DH>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + k2Stages * C::kStageBytes);
  uint64_t* kv_full = bars;                    // [stages] (CTA 0's count both CTAs' bytes)
  uint64_t* kv_empty = bars + k2Stages;        // [stages]
  uint64_t* s_full = bars + 2 * k2Stages;      // [2]
  uint64_t* p_full = s_full + 2;               // [2]  (CTA 0: one arrival per row warp of the pair)
  uint64_t* pv_done = p_full + 2;              // [2]
  uint64_t* q_ready = pv_done + 2;             // [1]  (CTA 0: one arrival per row warp of the pair)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_ready + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* xchg = reinterpret_cast<float*>(smem + k2Stages * C::kStageBytes + 512);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool has_old = !g.dense;
  int n_rows = g.n_rows ? *g.n_rows : g.S;
  if (n_rows > g.row_cap) n_rows = g.row_cap;
  if (n_rows < 0) n_rows = 0;
  const int row_tiles = (n_rows + k2Rows - 1) / k2Rows;
  const int pairs = (row_tiles + 1) / 2;
  const int total = pairs * g.H;
  const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < k2Stages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 16);
      mbar_init(&pv_done[b], 1);
    }
    mbar_init(q_ready, 16);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == k2TmaWarp) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs exist before any remote arrival or load
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == k2TmaWarp) {
    // ------------------------------------------------------------ TMA loads (both CTAs)
    if (lane == 0) {
      const uint32_t half_bytes = (has_old ? 2 : 1) * (C::kKHalf + C::kVHalf);
      const uint32_t full_bar0 = mapa_shared(smem_u32(kv_full), 0);
      int stage = 0;
      uint32_t phase = 0;
      int issued[k2Stages];
      for (int s2 = 0; s2 < k2Stages; ++s2) issued[s2] = -1;
      for (int item = cluster; item < total && !*abort_flag; item += n_clusters) {
        const int h = item / pairs, rp = item % pairs;
        const int nt = a2_tiles(g, h, rp, n_rows);
        for (int t = 0; t < nt && !*abort_flag; ++t) {
          if (!mbar_wait_sleep(&kv_empty[stage], phase ^ 1)) {
            set_error(g.err, kDevErrTimeout);
            *abort_flag = 1;
            break;
          }
          uint8_t* st = smem + stage * C::kStageBytes;
          const uint32_t bar = full_bar0 + stage * 8;  // CTA 0's kv_full[stage]
          if (rank == 0) mbar_arrive_expect_tx(&kv_full[stage], 2 * half_bytes);
          const int key0 = t * k2Cols + (int)rank * (k2Cols / 2);
#pragma unroll
          for (int c = 0; c < DH / 64; ++c)
            tma_load_3d_pair(st + c * C::kKChunk, &tm_kn, c * 64, key0, h, bar);
          tma_load_3d_pair(st + 2 * C::kKHalf, &tm_vn, t * k2Cols, (int)rank * (DH / 2), h, bar);
          if (has_old) {
#pragma unroll
            for (int c = 0; c < DH / 64; ++c)
              tma_load_3d_pair(st + C::kKHalf + c * C::kKChunk, &tm_ko, c * 64, key0, h, bar);
            tma_load_3d_pair(st + 2 * C::kKHalf + C::kVHalf, &tm_vo, t * k2Cols, (int)rank * (DH / 2), h, bar);
          }
          issued[stage] = (int)phase;
          if (++stage == k2Stages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // CTA 0's barriers count both CTAs' bytes: never leave with a copy in flight
      if (rank == 0)
        for (int s2 = 0; s2 < k2Stages; ++s2)
          if (issued[s2] >= 0) (void)mbar_wait(&kv_full[s2], (uint32_t)issued[s2]);
    }
  } else if (warp == k2MmaWarp) {
    // ------------------------------------------------------------ MMA issue (CTA 0)
    if (lane == 0 && rank == 0) {
      int stage = 0, prev_stage = 0;
      uint32_t phase = 0;
      uint32_t u = 0;
      uint32_t item_no = 0;
      bool ok = true;
      for (int item = cluster; item < total && ok && !*abort_flag; item += n_clusters, ++item_no) {
        const int h = item / pairs, rp = item % pairs;
        const int nt = a2_tiles(g, h, rp, n_rows);
        if (!mbar_wait_sleep(q_ready, item_no & 1)) {
          set_error(g.err, kDevErrTimeout);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        for (int t = 0; t <= nt && ok; ++t) {
          if (t < nt) {
            // S(t) into buffer u & 1 of both CTAs
            if (!mbar_wait_sleep(&kv_full[stage], phase)) {
              set_error(g.err, kDevErrTimeout);
              *abort_flag = 1;
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sb = tmem + C::kColS + (u & 1) * 128;
            const uint32_t k_addr = smem_u32(smem + stage * C::kStageBytes);
#pragma unroll
            for (int ks = 0; ks < DH / 16; ++ks) {
              const uint32_t kd = k_addr + (ks >> 2) * C::kKChunk + (ks & 3) * 32;
              umma_f16_ts_pair(sb, tmem + C::kColQn + ks * 8, sw128_kmajor_desc(kd), C::kIdescS, ks > 0);
              if (has_old)
                umma_f16_ts_pair(sb + 64, tmem + C::kColQo + ks * 8, sw128_kmajor_desc(kd + C::kKHalf), C::kIdescS,
                                 ks > 0);
            }
            umma_commit_pair(&s_full[u & 1]);
          }
          if (t > 0) {
            // P(t-1).V into N of both CTAs
            const uint32_t up = u - 1;
            if (!mbar_wait_sleep(&p_full[up & 1], (up >> 1) & 1)) {
              set_error(g.err, kDevErrTimeout);
              *abort_flag = 1;
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t pcol = tmem + C::kColS + (up & 1) * 128;
            const uint32_t v_addr = smem_u32(smem + prev_stage * C::kStageBytes + 2 * C::kKHalf);
#pragma unroll
            for (int ks = 0; ks < k2Cols / 16; ++ks)
              umma_f16_ts_pair(tmem + C::kColN, pcol + ks * 8, sw128_kmajor_desc(v_addr + ks * 32), C::kIdescPV, 1u);
            if (has_old) {
#pragma unroll
              for (int ks = 0; ks < k2Cols / 16; ++ks)
                umma_f16_ts_pair(tmem + C::kColN, pcol + 32 + ks * 8,
                                 sw128_kmajor_desc(v_addr + C::kVHalf + ks * 32), C::kIdescPV, 1u);
            }
            umma_commit_pair(&kv_empty[prev_stage]);
            umma_commit_pair(&pv_done[up & 1]);
          }
          if (t < nt) {
            prev_stage = stage;
            if (++stage == k2Stages) {
              stage = 0;
              phase ^= 1;
            }
            ++u;
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ rows (both CTAs)
    // Two threads per row, as in attn_tc.cu; each warp reports P and Q
    // readiness with one arrival on CTA 0's barrier.
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int pair_bar = 1 + quarter;
    const int HD = g.H * DH;
    constexpr int kHalfCols = DH / 2;
    const uint32_t p_full0 = mapa_shared(smem_u32(p_full), 0);
    const uint32_t q_ready0 = mapa_shared(smem_u32(q_ready), 0);
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
    // after this thread's TMEM stores: one arrival per warp on CTA 0's barrier
    auto warp_arrive = [&](uint32_t bar0) {
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(bar0);
    };
    uint32_t u = 0;
    for (int item = cluster; item < total; item += n_clusters) {
      const int h = item / pairs, rp = item % pairs;
      const int nt = a2_tiles(g, h, rp, n_rows);
      const int a = (rp * 2 + (int)rank) * k2Rows + row;
      int tok = -1;
      if (a < n_rows) {
        tok = g.rows ? __ldg(g.rows + a) : a;
        if (tok < 0 || tok >= g.S) {
          if (half == 0) set_error(g.err, FLASHLOOP_DEVERR_INDEX);
          tok = -1;
        }
      }
      // Q (fp16 pairs, exact from bf16) and this half of N into TMEM, in
      // 32-byte accesses; S is in log2 units (the keys carry log2(e)/sqrt(dh)).
      if (!dead) {
        const uint16_t* qsrc = half == 0 ? g.q_new : g.q_old;
        const bool load_q = tok >= 0 && (half == 0 || has_old);
        const bool load_n = !g.dense && tok >= 0;
        const uint32_t qcol = half == 0 ? C::kColQn : C::kColQo;
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
#pragma unroll
        for (int c0 = 0; c0 < DH; c0 += 32) {
          uint32_t r[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = bf16x2_to_half2_bits(qv[c0 / 16 + e / 8][e % 8]);
          __syncwarp();
          tmem_st16(tmem + lane_base + qcol + c0 / 2, r);
        }
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
          for (int e = 0; e < 16; ++e) r[e] = nv[c0 / 8 + e / 8][e % 8];
          __syncwarp();
          tmem_st16(tmem + lane_base + C::kColN + half * kHalfCols + c0, r);
        }
        warp_arrive(q_ready0);
      }
      float m_ref = 0.f, z = 0.f;
      if (tok >= 0) {
        m_ref = g.dense ? -INFINITY : g.m_in[(size_t)h * g.S + tok] * k2Log2e;
        if (!g.dense && half == 0) z = g.z_in[(size_t)h * g.S + tok];
      }

      const int32_t* hcols = g.cols ? g.cols + (size_t)h * g.kc : nullptr;
      int wmin = tok < 0 ? 0x7fffffff : tok;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) wmin = min(wmin, __shfl_xor_sync(0xffffffffu, wmin, o));
      // the token of each tile's last column is loaded one tile ahead
      auto tile_last = [&](int tt) -> int {
        const int ce = min((tt + 1) * k2Cols, g.kc);
        return hcols ? __ldg(hcols + ce - 1) : ce - 1;
      };
      int next_last = nt > 0 ? tile_last(0) : 0;
      for (int t = 0; t < nt; ++t, ++u) {
        const uint32_t b = u & 1;
        const int c0 = t * k2Cols;
        const int c_end = min(c0 + k2Cols, g.kc);
        const int last_tok = next_last;
        if (t + 1 < nt) next_last = tile_last(t + 1);
        const bool need_mask = (c0 + k2Cols > g.kc) || (last_tok > wmin);
        int nvalid = k2Cols;
        if (need_mask) {
          if (tok < 0) {
            nvalid = 0;
          } else {
            int lo = c0, hi = c_end;
            while (lo < hi) {
              const int mid = (lo + hi) >> 1;
              const int ct = hcols ? __ldg(hcols + mid) : mid;
              if (ct <= tok) lo = mid + 1;
              else hi = mid;
            }
            nvalid = lo - c0;
          }
        }
        const int first = half * 32;
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
                rn[e] = 0xff800000u;
                ro[e] = 0xff800000u;
              }
            }
          }
          float t16[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) t16[e] = fmaxf(__uint_as_float(rn[e]), __uint_as_float(rn[e + 16]));
#pragma unroll
          for (int w = 8; w > 0; w >>= 1)
#pragma unroll
            for (int e = 0; e < w; ++e) t16[e] = fmaxf(t16[e], t16[e + w]);
          mx = t16[0];
        }
        float* xm = xchg + (b * 2) * 128;
        xm[half * 128 + row] = mx;
        named_bar_sync(pair_bar, 64);
        mx = fmaxf(mx, xm[(1 - half) * 128 + row]);
        if (dead) continue;
        const bool need = mx > m_ref + k2RescaleThreshold;
        if (__any_sync(0xffffffffu, need)) {
          const float new_ref = need ? mx : m_ref;
          const float f = need ? ex2(m_ref - new_ref) : 1.f;
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
          z *= f;
          m_ref = new_ref;
        }
        uint32_t pk[16];
        float za[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) {
          const float p0 = ex2(__uint_as_float(rn[2 * e2]) - m_ref);
          const float p1 = ex2(__uint_as_float(rn[2 * e2 + 1]) - m_ref);
          za[e2 & 3] += p0 + p1;
          pk[e2] = pack_half2(p0, p1);
        }
        __syncwarp();
        tmem_st16(sbase + half * 16, pk);
        if (has_old) {
          float zb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int e2 = 0; e2 < 16; ++e2) {
            const float p0 = ex2(__uint_as_float(ro[2 * e2]) - m_ref);
            const float p1 = ex2(__uint_as_float(ro[2 * e2 + 1]) - m_ref);
            zb[e2 & 3] += p0 + p1;
            pk[e2] = pack_half2(-p0, -p1);
          }
          __syncwarp();
          tmem_st16(sbase + 32 + half * 16, pk);
#pragma unroll
          for (int i = 0; i < 4; ++i) za[i] -= zb[i];
        }
        z += (za[0] + za[1]) + (za[2] + za[3]);
        warp_arrive(p_full0 + b * 8);
      }
      if (nt > 0) {
        const uint32_t up = u - 1;
        wait_or_die(&pv_done[up & 1], (up >> 1) & 1);
      }
      float* xz = xchg + 4 * 128;
      xz[half * 128 + row] = z;
      named_bar_sync(pair_bar, 64);
      const float z_row = xz[row] + xz[128 + row];
      named_bar_sync(pair_bar, 64);
      if (dead) continue;
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
        g.m_out[(size_t)h * g.S + tok] = m_ref / k2Log2e;
        g.z_out[(size_t)h * g.S + tok] = z_row;
        if (g.dense && g.g_out) g.g_out[(size_t)h * g.S + tok] = 1.f;
      }
      tc_fence_before();
    }
  }
  // neither CTA leaves (or frees TMEM) while the pair's MMAs, loads or
  // arrivals may still touch it
  tc_fence_before();
  cluster_sync_all();
  if (warp == k2TmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}


constexpr int k4Threads = 576, k4TmaWarp = 16, k4MmaWarp = 17;  // 16 row warps (four threads per row)
template <int DH>
constexpr int a4_smem() { return 1024 + k2Stages * A2Cfg<DH>::kStageBytes + 512 + 12 * 128 * 4; }

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n"
               ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

template <int DH>
__global__ void __launch_bounds__(k4Threads, 1)
attn_pair4_kernel(const __grid_constant__ CUtensorMap tm_kn, const __grid_constant__ CUtensorMap tm_ko,
                 const __grid_constant__ CUtensorMap tm_vn, const __grid_constant__ CUtensorMap tm_vo, A2Args g) {
  using C = A2Cfg<DH>;
  constexpr int kSmemXchg = 512;  // offset of the row exchange after the barriers
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + k2Stages * C::kStageBytes);
  uint64_t* kv_full = bars;                    // [stages] (CTA 0's count both CTAs' bytes)
  uint64_t* kv_empty = bars + k2Stages;        // [stages]
  uint64_t* s_full = bars + 2 * k2Stages;      // [2]
  uint64_t* p_full = s_full + 2;               // [2]  (CTA 0: one arrival per row warp of the pair)
  uint64_t* pv_done = p_full + 2;              // [2]
  uint64_t* q_ready = pv_done + 2;             // [1]  (CTA 0: one arrival per row warp of the pair)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_ready + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* xchg = reinterpret_cast<float*>(smem + k2Stages * C::kStageBytes + kSmemXchg);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool has_old = !g.dense;
  int n_rows = g.n_rows ? *g.n_rows : g.S;
  if (n_rows > g.row_cap) n_rows = g.row_cap;
  if (n_rows < 0) n_rows = 0;
  const int row_tiles = (n_rows + k2Rows - 1) / k2Rows;
  const int pairs = (row_tiles + 1) / 2;
  const int total = pairs * g.H;
  const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < k2Stages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 32);
      mbar_init(&pv_done[b], 1);
    }
    mbar_init(q_ready, 32);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == k4TmaWarp) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs exist before any remote arrival or load
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == k4TmaWarp) {
    // ------------------------------------------------------------ TMA loads (both CTAs)
    if (lane == 0) {
      const uint32_t half_bytes = (has_old ? 2 : 1) * (C::kKHalf + C::kVHalf);
      const uint32_t full_bar0 = mapa_shared(smem_u32(kv_full), 0);
      int stage = 0;
      uint32_t phase = 0;
      int issued[k2Stages];
      for (int s2 = 0; s2 < k2Stages; ++s2) issued[s2] = -1;
      for (int item = cluster; item < total && !*abort_flag; item += n_clusters) {
        const int h = item / pairs, rp = item % pairs;
        const int nt = a2_tiles(g, h, rp, n_rows);
        for (int t = 0; t < nt && !*abort_flag; ++t) {
          if (!mbar_wait_sleep(&kv_empty[stage], phase ^ 1)) {
            set_error(g.err, kDevErrTimeout);
            *abort_flag = 1;
            break;
          }
          uint8_t* st = smem + stage * C::kStageBytes;
          const uint32_t bar = full_bar0 + stage * 8;  // CTA 0's kv_full[stage]
          if (rank == 0) mbar_arrive_expect_tx(&kv_full[stage], 2 * half_bytes);
          const int key0 = t * k2Cols + (int)rank * (k2Cols / 2);
#pragma unroll
          for (int c = 0; c < DH / 64; ++c)
            tma_load_3d_pair(st + c * C::kKChunk, &tm_kn, c * 64, key0, h, bar);
          tma_load_3d_pair(st + 2 * C::kKHalf, &tm_vn, t * k2Cols, (int)rank * (DH / 2), h, bar);
          if (has_old) {
#pragma unroll
            for (int c = 0; c < DH / 64; ++c)
              tma_load_3d_pair(st + C::kKHalf + c * C::kKChunk, &tm_ko, c * 64, key0, h, bar);
            tma_load_3d_pair(st + 2 * C::kKHalf + C::kVHalf, &tm_vo, t * k2Cols, (int)rank * (DH / 2), h, bar);
          }
          issued[stage] = (int)phase;
          if (++stage == k2Stages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // CTA 0's barriers count both CTAs' bytes: never leave with a copy in flight
      if (rank == 0)
        for (int s2 = 0; s2 < k2Stages; ++s2)
          if (issued[s2] >= 0) (void)mbar_wait(&kv_full[s2], (uint32_t)issued[s2]);
    }
  } else if (warp == k4MmaWarp) {
    // ------------------------------------------------------------ MMA issue (CTA 0)
    if (lane == 0 && rank == 0) {
      int stage = 0, prev_stage = 0;
      uint32_t phase = 0;
      uint32_t u = 0;
      uint32_t item_no = 0;
      bool ok = true;
      for (int item = cluster; item < total && ok && !*abort_flag; item += n_clusters, ++item_no) {
        const int h = item / pairs, rp = item % pairs;
        const int nt = a2_tiles(g, h, rp, n_rows);
        if (!mbar_wait_sleep(q_ready, item_no & 1)) {
          set_error(g.err, kDevErrTimeout);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        for (int t = 0; t <= nt && ok; ++t) {
          if (t < nt) {
            // S(t) into buffer u & 1 of both CTAs
            if (!mbar_wait_sleep(&kv_full[stage], phase)) {
              set_error(g.err, kDevErrTimeout);
              *abort_flag = 1;
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sb = tmem + C::kColS + (u & 1) * 128;
            const uint32_t k_addr = smem_u32(smem + stage * C::kStageBytes);
#pragma unroll
            for (int ks = 0; ks < DH / 16; ++ks) {
              const uint32_t kd = k_addr + (ks >> 2) * C::kKChunk + (ks & 3) * 32;
              umma_f16_ts_pair(sb, tmem + C::kColQn + ks * 8, sw128_kmajor_desc(kd), C::kIdescS, ks > 0);
              if (has_old)
                umma_f16_ts_pair(sb + 64, tmem + C::kColQo + ks * 8, sw128_kmajor_desc(kd + C::kKHalf), C::kIdescS,
                                 ks > 0);
            }
            umma_commit_pair(&s_full[u & 1]);
          }
          if (t > 0) {
            // P(t-1).V into N of both CTAs
            const uint32_t up = u - 1;
            if (!mbar_wait_sleep(&p_full[up & 1], (up >> 1) & 1)) {
              set_error(g.err, kDevErrTimeout);
              *abort_flag = 1;
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t pcol = tmem + C::kColS + (up & 1) * 128;
            const uint32_t v_addr = smem_u32(smem + prev_stage * C::kStageBytes + 2 * C::kKHalf);
#pragma unroll
            for (int ks = 0; ks < k2Cols / 16; ++ks)
              umma_f16_ts_pair(tmem + C::kColN, pcol + ks * 8, sw128_kmajor_desc(v_addr + ks * 32), C::kIdescPV, 1u);
            if (has_old) {
#pragma unroll
              for (int ks = 0; ks < k2Cols / 16; ++ks)
                umma_f16_ts_pair(tmem + C::kColN, pcol + 32 + ks * 8,
                                 sw128_kmajor_desc(v_addr + C::kVHalf + ks * 32), C::kIdescPV, 1u);
            }
            umma_commit_pair(&kv_empty[prev_stage]);
            umma_commit_pair(&pv_done[up & 1]);
          }
          if (t < nt) {
            prev_stage = stage;
            if (++stage == k2Stages) {
              stage = 0;
              phase ^= 1;
            }
            ++u;
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ rows (both CTAs)
    // Four threads per row: part p (warps 4p..4p+3) takes columns
    // [16 p, 16 p + 16) of S_new and S_old of each tile, a quarter of Q
    // (parts 0-1 Q_new, 2-3 Q_old) and N columns [p DH/4, (p + 1) DH/4).
    // The four warps of a lane quarter exchange tile maxima and sums through
    // shared memory at a named barrier of 128 threads; dead mode as in
    // attn_tc.cu.  Each warp reports with one arrival on CTA 0's barrier.
    const int quarter = warp & 3, part = warp >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int quad_bar = 1 + quarter;
    const int HD = g.H * DH;
    constexpr int kPartCols = DH / 4;   // N columns of a part
    constexpr int kQElems = DH / 2;     // Q elements of a part (half of one matrix)
    const uint32_t p_full0 = mapa_shared(smem_u32(p_full), 0);
    const uint32_t q_ready0 = mapa_shared(smem_u32(q_ready), 0);
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
    auto warp_arrive = [&](uint32_t bar0) {
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(bar0);
    };
    uint32_t u = 0;
    for (int item = cluster; item < total; item += n_clusters) {
      const int h = item / pairs, rp = item % pairs;
      const int nt = a2_tiles(g, h, rp, n_rows);
      const int a = (rp * 2 + (int)rank) * k2Rows + row;
      int tok = -1;
      if (a < n_rows) {
        tok = g.rows ? __ldg(g.rows + a) : a;
        if (tok < 0 || tok >= g.S) {
          if (part == 0) set_error(g.err, FLASHLOOP_DEVERR_INDEX);
          tok = -1;
        }
      }
      if (!dead) {
        const bool old_q = part >= 2;
        const uint16_t* qsrc = old_q ? g.q_old : g.q_new;
        const bool load_q = tok >= 0 && (!old_q || has_old);
        const bool load_n = !g.dense && tok >= 0;
        const uint32_t qcol = (old_q ? C::kColQo : C::kColQn) + (part & 1) * (kQElems / 2);
        const int q0 = (part & 1) * kQElems;   // first Q element of this part
        uint32_t qv[kQElems / 16][8];
#pragma unroll
        for (int v = 0; v < kQElems / 16; ++v) {
          if (load_q) {
            ld_global_v8(qsrc + (size_t)tok * HD + (size_t)h * DH + q0 + v * 16, qv[v]);
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) qv[v][e] = 0u;
          }
        }
#pragma unroll
        for (int c0 = 0; c0 < kQElems; c0 += 32) {
          uint32_t r[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = bf16x2_to_half2_bits(qv[c0 / 16 + e / 8][e % 8]);
          __syncwarp();
          tmem_st16(tmem + lane_base + qcol + c0 / 2, r);
        }
        uint32_t nv[kPartCols / 8][8];
#pragma unroll
        for (int v = 0; v < kPartCols / 8; ++v) {
          if (load_n) {
            ld_global_v8(g.n_in + ((size_t)h * g.S + tok) * DH + part * kPartCols + 8 * v, nv[v]);
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) nv[v][e] = 0u;
          }
        }
#pragma unroll
        for (int c0 = 0; c0 < kPartCols; c0 += 16) {
          uint32_t r[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = nv[c0 / 8 + e / 8][e % 8];
          __syncwarp();
          tmem_st16(tmem + lane_base + C::kColN + part * kPartCols + c0, r);
        }
        warp_arrive(q_ready0);
      }
      float m_ref = 0.f, z = 0.f;
      if (tok >= 0) {
        m_ref = g.dense ? -INFINITY : g.m_in[(size_t)h * g.S + tok] * k2Log2e;
        if (!g.dense && part == 0) z = g.z_in[(size_t)h * g.S + tok];
      }
      const int32_t* hcols = g.cols ? g.cols + (size_t)h * g.kc : nullptr;
      int wmin = tok < 0 ? 0x7fffffff : tok;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) wmin = min(wmin, __shfl_xor_sync(0xffffffffu, wmin, o));
      auto tile_last = [&](int tt) -> int {
        const int ce = min((tt + 1) * k2Cols, g.kc);
        return hcols ? __ldg(hcols + ce - 1) : ce - 1;
      };
      int next_last = nt > 0 ? tile_last(0) : 0;
      for (int t = 0; t < nt; ++t, ++u) {
        const uint32_t b = u & 1;
        const int c0 = t * k2Cols;
        const int c_end = min(c0 + k2Cols, g.kc);
        const int last_tok = next_last;
        if (t + 1 < nt) next_last = tile_last(t + 1);
        const bool need_mask = (c0 + k2Cols > g.kc) || (last_tok > wmin);
        int nvalid = k2Cols;
        if (need_mask) {
          if (tok < 0) {
            nvalid = 0;
          } else {
            int lo = c0, hi = c_end;
            while (lo < hi) {
              const int mid = (lo + hi) >> 1;
              const int ct = hcols ? __ldg(hcols + mid) : mid;
              if (ct <= tok) lo = mid + 1;
              else hi = mid;
            }
            nvalid = lo - c0;
          }
        }
        const int first = part * 16;
        wait_or_die(&s_full[b], (u >> 1) & 1);
        uint32_t rn[16], ro[16];
        const uint32_t sbase = tmem + lane_base + C::kColS + b * 128;
        float mx = -INFINITY;
        if (!dead) {
          __syncwarp();
          tmem_ld16(sbase + first, rn);
          if (has_old) tmem_ld16(sbase + 64 + first, ro);
          tmem_wait_ld();
          if (nvalid < first + 16) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              if (first + e >= nvalid) {
                rn[e] = 0xff800000u;
                ro[e] = 0xff800000u;
              }
            }
          }
          float t8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) t8[e] = fmaxf(__uint_as_float(rn[e]), __uint_as_float(rn[e + 8]));
#pragma unroll
          for (int w = 4; w > 0; w >>= 1)
#pragma unroll
            for (int e = 0; e < w; ++e) t8[e] = fmaxf(t8[e], t8[e + w]);
          mx = t8[0];
        }
        float* xm = xchg + b * 4 * 128;  // [part][128] of this parity
        xm[part * 128 + row] = mx;
        named_bar_sync(quad_bar, 128);
        mx = fmaxf(fmaxf(xm[row], xm[128 + row]), fmaxf(xm[256 + row], xm[384 + row]));
        if (dead) continue;
        const bool need = mx > m_ref + k2RescaleThreshold;
        if (__any_sync(0xffffffffu, need)) {
          const float new_ref = need ? mx : m_ref;
          const float f = need ? ex2(m_ref - new_ref) : 1.f;
          if (t > 0) {
            const uint32_t up = u - 1;
            wait_or_die(&pv_done[up & 1], (up >> 1) & 1);
            if (dead) continue;
          }
#pragma unroll 1
          for (int cc = 0; cc < kPartCols; cc += 16) {
            uint32_t r[16];
            __syncwarp();
            tmem_ld16(tmem + lane_base + C::kColN + part * kPartCols + cc, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * f);
            __syncwarp();
            tmem_st16(tmem + lane_base + C::kColN + part * kPartCols + cc, r);
          }
          tmem_wait_st();
          z *= f;
          m_ref = new_ref;
        }
        uint32_t pk[8];
        float za[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) {
          const float p0 = ex2(__uint_as_float(rn[2 * e2]) - m_ref);
          const float p1 = ex2(__uint_as_float(rn[2 * e2 + 1]) - m_ref);
          za[e2 & 3] += p0 + p1;
          pk[e2] = pack_half2(p0, p1);
        }
        __syncwarp();
        tmem_st8(sbase + part * 8, pk);
        if (has_old) {
          float zb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int e2 = 0; e2 < 8; ++e2) {
            const float p0 = ex2(__uint_as_float(ro[2 * e2]) - m_ref);
            const float p1 = ex2(__uint_as_float(ro[2 * e2 + 1]) - m_ref);
            zb[e2 & 3] += p0 + p1;
            pk[e2] = pack_half2(-p0, -p1);
          }
          __syncwarp();
          tmem_st8(sbase + 32 + part * 8, pk);
#pragma unroll
          for (int i = 0; i < 4; ++i) za[i] -= zb[i];
        }
        z += (za[0] + za[1]) + (za[2] + za[3]);
        warp_arrive(p_full0 + b * 8);
      }
      if (nt > 0) {
        const uint32_t up = u - 1;
        wait_or_die(&pv_done[up & 1], (up >> 1) & 1);
      }
      float* xz = xchg + 8 * 128;   // [part][128]
      xz[part * 128 + row] = z;
      named_bar_sync(quad_bar, 128);
      const float z_row = (xz[row] + xz[128 + row]) + (xz[256 + row] + xz[384 + row]);
      named_bar_sync(quad_bar, 128);
      if (dead) continue;
      const float inv = 1.f / z_row;
#pragma unroll 1
      for (int cc = 0; cc < kPartCols; cc += 16) {
        uint32_t r[16];
        __syncwarp();
        tmem_ld16(tmem + lane_base + C::kColN + part * kPartCols + cc, r);
        tmem_wait_ld();
        if (tok >= 0) {
          const int col = part * kPartCols + cc;
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
      if (tok >= 0 && part == 0) {
        g.m_out[(size_t)h * g.S + tok] = m_ref / k2Log2e;
        g.z_out[(size_t)h * g.S + tok] = z_row;
        if (g.dense && g.g_out) g.g_out[(size_t)h * g.S + tok] = 1.f;
      }
      tc_fence_before();
    }
  }
  // neither CTA leaves (or frees TMEM) while the pair's MMAs, loads or
  // arrivals may still touch it
  tc_fence_before();
  cluster_sync_all();
  if (warp == k4TmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
int make_tmap_f16_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1_elems,
                     uint64_t s2_elems, uint32_t b0, uint32_t b1);
int at_sm_count();

// Pairs of SMs the device can run at once for a kernel (clusters of 2).
static int a2_max_pairs(const void* kernel, int threads, int smem, int slot) {
  static int cached[4][64] = {{0}};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[slot][dev] != 0) return cached[slot][dev];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * 74, 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = -1;
  }
  cached[slot][dev] = n;
  return n;
}

// The running update on SM pairs (params.attn_pairs: 1 two threads per row,
// 2 four threads per row); returns FLASHLOOP_ERR_UNSUPPORTED when the device
// cannot co-schedule pairs (the caller then uses one SM per tile).
int launch_attn_pair(const flashloop_params* p, const AttnArgs& a, int kcp, cudaStream_t stream) {
  const int dh = p->head_dim, H = p->n_heads;
  if (dh != 128 && dh != 64) return FLASHLOOP_ERR_UNSUPPORTED;
  const void* aligned32[] = {a.q_new, a.q_old, a.n_in, a.n_out, a.o};
  for (const void* ptr : aligned32)
    if (reinterpret_cast<uintptr_t>(ptr) % 32 != 0) return FLASHLOOP_ERR_INVALID_ARG;
  const bool four = p->attn_pairs == 2;
  const void* kernel = four ? (dh == 128 ? (const void*)attn_pair4_kernel<128> : (const void*)attn_pair4_kernel<64>)
                            : (dh == 128 ? (const void*)attn_pair_kernel<128> : (const void*)attn_pair_kernel<64>);
  const int threads = four ? k4Threads : k2Threads;
  const int smem = four ? (dh == 128 ? a4_smem<128>() : a4_smem<64>()) : (dh == 128 ? A2Cfg<128>::kSmem : A2Cfg<64>::kSmem);
  FL_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  const int max_pairs = a2_max_pairs(kernel, threads, smem, (four ? 2 : 0) + (dh == 128 ? 1 : 0));
  if (max_pairs <= 0) return FLASHLOOP_ERR_UNSUPPORTED;
  // K halves: 32 keys x 64 head-dim elements per box; V^T halves: 64 keys x DH/2 rows
  CUtensorMap tkn, tko, tvn, tvo;
  int rc = make_tmap_f16_3d(&tkn, a.k_new, dh, a.kc, H, dh, (uint64_t)kcp * dh, 64, k2Cols / 2);
  if (rc == FLASHLOOP_OK) rc = make_tmap_f16_3d(&tvn, a.v_new, a.kc, dh, H, kcp, (uint64_t)kcp * dh, k2Cols, dh / 2);
  if (rc == FLASHLOOP_OK && !a.dense) {
    rc = make_tmap_f16_3d(&tko, a.k_old, dh, a.kc, H, dh, (uint64_t)kcp * dh, 64, k2Cols / 2);
    if (rc == FLASHLOOP_OK) rc = make_tmap_f16_3d(&tvo, a.v_old, a.kc, dh, H, kcp, (uint64_t)kcp * dh, k2Cols, dh / 2);
  } else {
    tko = tkn;
    tvo = tvn;
  }
  if (rc != FLASHLOOP_OK) return rc;
  A2Args g{};
  g.S = a.S; g.H = a.H; g.kc = a.kc; g.dense = a.dense; g.rows = a.rows; g.n_rows = a.n_rows;
  g.row_cap = a.row_cap; g.cols = a.cols; g.q_new = a.q_new; g.q_old = a.q_old; g.m_in = a.m_in;
  g.z_in = a.z_in; g.n_in = a.n_in; g.m_out = a.m_out; g.z_out = a.z_out; g.n_out = a.n_out; g.o = a.o;
  g.err = a.err;
  g.g_out = a.g_out;
  const int max_items = ((a.row_cap + 2 * k2Rows - 1) / (2 * k2Rows)) * H;
  int n_pairs = at_sm_count() / 2;
  if (n_pairs > max_pairs) n_pairs = max_pairs;
  if (n_pairs > max_items) n_pairs = max_items;
  if (n_pairs < 1) n_pairs = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * n_pairs, 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (four) {
    if (dh == 128) FL_TRY(cudaLaunchKernelEx(&cfg, attn_pair4_kernel<128>, tkn, tko, tvn, tvo, g));
    else FL_TRY(cudaLaunchKernelEx(&cfg, attn_pair4_kernel<64>, tkn, tko, tvn, tvo, g));
  } else {
    if (dh == 128) FL_TRY(cudaLaunchKernelEx(&cfg, attn_pair_kernel<128>, tkn, tko, tvn, tvo, g));
    else FL_TRY(cudaLaunchKernelEx(&cfg, attn_pair_kernel<64>, tkn, tko, tvn, tvo, g));
  }
  return launch_status();
}

}  // namespace fl
