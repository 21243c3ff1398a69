// (a4) Column selection: per-head top-k of the previous loop's column mass.
//
// [FlashLoop §3.2, §4.2, App. D.2]: the preceding loop's attention
// statistics rank the key columns; the top-k are recomputed.  One block per
// head keeps the head's keys in shared memory (n <= 49152), finds the k-th
// largest key by a 4-pass, 8-bit radix select, then keeps every key above
// it and the lowest-index keys equal to it (ties go to the lower index), and
// writes the indices in ascending order with two block scans.  Keys are the
// float32 bits mapped to an order-preserving uint32 (-0 counted as +0).
// Each warp counts into its own histogram (masses crowd into few bins, and
// one shared bin would serialise every warp's atomics); the 32 are summed
// per pass.  Optionally the key is a probability made on the fly from a
// row of log2-unit scores, 2^(s - m) / Z, which is also written out.
#include "common.cuh"
#include "mma_util.cuh"

namespace fl {

constexpr int kTopkThreads = 1024;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkMaxN = 49152;

__device__ __forceinline__ uint32_t order_key(float v) {
  uint32_t b = __float_as_uint(v);
  if (b == 0x80000000u) b = 0u;  // -0 == +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(const float* __restrict__ mass, int S, const int32_t* __restrict__ cand, int n_cand,
            int k, int32_t* __restrict__ out, int32_t* err, const float* __restrict__ row_m,
            const float* __restrict__ row_z, float* __restrict__ probs_out, const int32_t* __restrict__ n_dev,
            int32_t* __restrict__ k_out, const int32_t* __restrict__ out_map) {
  extern __shared__ uint32_t keys[];  // [n_alloc], then the warps' histograms [kTopkWarps][256]
  __shared__ int hist[256];
  __shared__ int warp_sums[32];
  __shared__ uint32_t s_prefix;
  __shared__ int s_remaining;
  const int h = blockIdx.x;
  const int n_alloc = cand ? n_cand : S;
  // a device count may shorten the list (keys n_dev.. are not candidates)
  const int n = n_dev ? max(0, min(n_alloc, *n_dev)) : n_alloc;
  if (k > n) k = n;
  if (k_out != nullptr && threadIdx.x == 0) k_out[h] = k;
  const int32_t* hc = cand ? cand + (size_t)h * n_cand : nullptr;
  const float* hm = mass + (size_t)h * S;
  int* whist = reinterpret_cast<int*>(keys + n_alloc);
  const bool probs = row_m != nullptr;
  const float pm = probs ? row_m[h] : 0.f;
  const float prz = probs ? 1.f / row_z[h] : 0.f;
  // eight loads in flight per thread before the keys are stored
  constexpr int kBatch = 8;
  for (int c0 = threadIdx.x; c0 < n; c0 += kBatch * blockDim.x) {
    float v[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int c = c0 + i * blockDim.x;
      int j = c;
      if (hc != nullptr && c < n) j = hc[c];
      if (c < n && (j < 0 || j >= S)) {
        set_error(err, FLASHLOOP_DEVERR_INDEX);
        j = 0;
      }
      v[i] = c < n ? hm[j] : 0.f;
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int c = c0 + i * blockDim.x;
      if (c < n) {
        float x = v[i];
        if (probs) {
          x = ex2(x - pm) * prz;
          probs_out[(size_t)h * S + c] = x;
        }
        keys[c] = order_key(x);
      }
    }
  }
  if (threadIdx.x == 0) {
    s_prefix = 0u;
    s_remaining = k;
  }
  __syncthreads();

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int* my_hist = whist + warp * 256;
  uint32_t mask = 0u;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = threadIdx.x; b < kTopkWarps * 256; b += blockDim.x) whist[b] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix;
    // Keys crowd into few bins (masses share their exponent bits): the lanes
    // of a warp whose bin is that of the warp's first counted lane add once,
    // with their count; the others add one by one.
    for (int base = 0; base < n; base += blockDim.x) {
      const int c = base + threadIdx.x;
      const uint32_t key = c < n ? keys[c] : 0u;
      const bool in = c < n && (key & mask) == prefix;
      const uint32_t bin = (key >> shift) & 255u;
      const uint32_t in_mask = __ballot_sync(0xffffffffu, in);
      const uint32_t lead = __shfl_sync(0xffffffffu, bin, in_mask ? __ffs(in_mask) - 1 : 0);
      const uint32_t same = __ballot_sync(0xffffffffu, in && bin == lead);
      if (in) {
        if (bin != lead) atomicAdd(&my_hist[bin], 1);
        else if (lane == __ffs(same) - 1) atomicAdd(&my_hist[bin], __popc(same));
      }
    }
    __syncthreads();
    if (threadIdx.x < 256) {
      int t = 0;
#pragma unroll 8
      for (int w = 0; w < kTopkWarps; ++w) t += whist[w * 256 + threadIdx.x];
      hist[threadIdx.x] = t;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // bins in descending order, 8 per lane: the bin where the count from
      // the top first reaches the number still to keep
      int cnt[8], tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        cnt[i] = hist[255 - (lane * 8 + i)];
        tot += cnt[i];
      }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int rem = s_remaining;
      int run = incl - tot;
      const bool last_lane_b0 = lane == 31;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const bool bottom = last_lane_b0 && i == 7;  // bin 0 takes whatever is left
        if (run < rem && (run + cnt[i] >= rem || bottom)) {
          s_remaining = rem - run;
          s_prefix = prefix | (static_cast<uint32_t>(255 - (lane * 8 + i)) << shift);
        }
        run += cnt[i];
      }
    }
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t thr = s_prefix;
  const int need_eq = s_remaining;  // keys equal to thr that are kept

  // Ascending output: rank of equal keys, then the final compaction.
  const int items = (n + blockDim.x - 1) / blockDim.x;
  int running_eq = 0, running_out = 0;
  for (int base = 0; base < n; base += blockDim.x * items) {
    const int first = base + threadIdx.x * items;
    int eq_cnt = 0;
    for (int q = 0; q < items; ++q) {
      const int c = first + q;
      if (c < n && keys[c] == thr) ++eq_cnt;
    }
    int eq_total;
    const int eq_start = running_eq + block_exclusive_scan(eq_cnt, warp_sums, &eq_total);
    int keep_cnt = 0;
    int eq_rank = eq_start;
    for (int q = 0; q < items; ++q) {
      const int c = first + q;
      if (c < n) {
        const uint32_t key = keys[c];
        if (key > thr) ++keep_cnt;
        else if (key == thr) {
          if (eq_rank < need_eq) ++keep_cnt;
          ++eq_rank;
        }
      }
    }
    int keep_total;
    int pos = running_out + block_exclusive_scan(keep_cnt, warp_sums, &keep_total);
    eq_rank = eq_start;
    for (int q = 0; q < items; ++q) {
      const int c = first + q;
      if (c < n) {
        const uint32_t key = keys[c];
        bool keep = false;
        if (key > thr) keep = true;
        else if (key == thr) {
          keep = eq_rank < need_eq;
          ++eq_rank;
        }
        if (keep) {
          if (pos < k) out[(size_t)h * k + pos] = out_map ? out_map[c] : (hc ? hc[c] : c);
          ++pos;
        }
      }
    }
    running_eq += eq_total;
    running_out += keep_total;
  }
}

int launch_topk(const flashloop_params* p, const float* mass, const int32_t* cand, int n_cand,
                int k, int32_t* out, int32_t* err, cudaStream_t stream, const float* row_m,
                const float* row_z, float* probs_out, const int32_t* n_dev, int32_t* k_out,
                const int32_t* out_map) {
  const int n = cand ? n_cand : p->seq;
  const size_t smem = ((size_t)n + kTopkWarps * 256) * sizeof(uint32_t);
  static bool attr_set = false;
  if (!attr_set) {
    FL_TRY(cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)((kTopkMaxN + kTopkWarps * 256) * sizeof(uint32_t))));
    attr_set = true;
  }
  topk_kernel<<<p->n_heads, kTopkThreads, smem, stream>>>(mass, p->seq, cand, n_cand, k, out, err, row_m, row_z,
                                                          probs_out, n_dev, k_out, out_map);
  return launch_status();
}

}  // namespace fl
