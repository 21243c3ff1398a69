// (a4) Column selection: per-head top-k of the previous loop's column mass.
//
// [FlashLoop §3.2, §4.2, App. D.2]: the preceding loop's attention
// statistics rank the key columns; the top-k are recomputed.  One block per
// head keeps the head's keys in shared memory (n <= 53248), finds the k-th
// largest key by a 4-pass, 8-bit radix select, then keeps every key above
// it and the lowest-index keys equal to it (ties go to the lower index), and
// writes the indices in ascending order with two block scans.  Keys are the
// float32 bits mapped to an order-preserving uint32 (-0 counted as +0).
#include "common.cuh"

namespace fl {

constexpr int kTopkThreads = 1024;
constexpr int kTopkMaxN = 53248;

__device__ __forceinline__ uint32_t order_key(float v) {
  uint32_t b = __float_as_uint(v);
  if (b == 0x80000000u) b = 0u;  // -0 == +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(const float* __restrict__ mass, int S, const int32_t* __restrict__ cand, int n_cand,
            int k, int32_t* __restrict__ out, int32_t* err) {
  extern __shared__ uint32_t keys[];
  __shared__ int hist[256];
  __shared__ int warp_sums[32];
  __shared__ uint32_t s_prefix;
  __shared__ int s_remaining;
  const int h = blockIdx.x;
  const int n = cand ? n_cand : S;
  const int32_t* hc = cand ? cand + (size_t)h * n_cand : nullptr;
  const float* hm = mass + (size_t)h * S;
  for (int c = threadIdx.x; c < n; c += blockDim.x) {
    int j = hc ? hc[c] : c;
    if (j < 0 || j >= S) {
      set_error(err, FLASHLOOP_DEVERR_INDEX);
      j = 0;
    }
    keys[c] = order_key(hm[j]);
  }
  if (threadIdx.x == 0) {
    s_prefix = 0u;
    s_remaining = k;
  }
  __syncthreads();

  uint32_t mask = 0u;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix;
    for (int c = threadIdx.x; c < n; c += blockDim.x) {
      const uint32_t key = keys[c];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int rem = s_remaining;
      int b = 255;
      for (; b > 0; --b) {
        if (hist[b] >= rem) break;
        rem -= hist[b];
      }
      s_remaining = rem;
      s_prefix = prefix | (static_cast<uint32_t>(b) << shift);
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
          if (pos < k) out[(size_t)h * k + pos] = hc ? hc[c] : c;
          ++pos;
        }
      }
    }
    running_eq += eq_total;
    running_out += keep_total;
  }
}

int launch_topk(const flashloop_params* p, const float* mass, const int32_t* cand, int n_cand,
                int k, int32_t* out, int32_t* err, cudaStream_t stream) {
  const int n = cand ? n_cand : p->seq;
  const size_t smem = (size_t)n * sizeof(uint32_t);
  static bool attr_set = false;
  if (!attr_set) {
    FL_TRY(cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(kTopkMaxN * sizeof(uint32_t))));
    attr_set = true;
  }
  topk_kernel<<<p->n_heads, kTopkThreads, smem, stream>>>(mass, p->seq, cand, n_cand, k, out, err);
  return launch_status();
}

}  // namespace fl
