// (a1) Token change gate and stream compaction.
//
// [FlashLoop §3.1, §4.1, App. D.1]: later loops recompute only a nested set
// of tokens whose hidden state still changes; the candidates are the
// previous active set.  One warp reduces one candidate row (16-byte loads,
// float32 sums of (x_cur - x_prev)^2 and x_prev^2); the last block to finish
// (atomic ticket, no waiting) scans the decisions into the ascending active
// list, the slot map and the device count.  HBM-bound: 4 * d_model bytes
// per candidate row.
#include "common.cuh"

namespace fl {

constexpr int kGateThreads = 256;
constexpr int kGateItems = 16;  // decisions per thread per scan chunk

__global__ void __launch_bounds__(kGateThreads)
gate_kernel(const uint16_t* __restrict__ x_cur, const uint16_t* __restrict__ x_prev, int S, int d,
            const int32_t* __restrict__ prev_active, const int32_t* __restrict__ n_prev_ptr,
            int prev_cap, float tau2, uint8_t* __restrict__ flags, unsigned int* __restrict__ ticket,
            int32_t* __restrict__ active_out, int32_t* __restrict__ slot_out,
            int32_t* __restrict__ n_out, int out_cap, int32_t* __restrict__ err) {
  __shared__ int warp_sums[32];
  __shared__ unsigned int s_is_last;
  int n_prev = prev_active ? *n_prev_ptr : S;
  if (n_prev > prev_cap) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_error(err, FLASHLOOP_DEVERR_CAPACITY);
    n_prev = prev_cap;
  }
  if (n_prev < 0) n_prev = 0;

  // Every slot starts inactive; the compaction below marks the active ones.
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < S; i += gridDim.x * blockDim.x)
    slot_out[i] = -1;

  const int lane = threadIdx.x & 31;
  const int warps_per_block = blockDim.x >> 5;
  const int vecs = d >> 3;  // 8 bf16 per 16-byte load
  for (int c = blockIdx.x * warps_per_block + (threadIdx.x >> 5); c < n_prev;
       c += gridDim.x * warps_per_block) {
    const int t = prev_active ? prev_active[c] : c;
    if (t < 0 || t >= S) {
      if (lane == 0) {
        set_error(err, FLASHLOOP_DEVERR_INDEX);
        flags[c] = 0;
      }
      continue;
    }
    const uint4* xc = reinterpret_cast<const uint4*>(x_cur + (size_t)t * d);
    const uint4* xp = reinterpret_cast<const uint4*>(x_prev + (size_t)t * d);
    float dsum = 0.f, psum = 0.f;
    for (int v = lane; v < vecs; v += 32) {
      const uint4 a = __ldcs(xc + v);
      const uint4 b = __ldcs(xp + v);
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
      const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 fa = bf16x2_to_float2(aw[u]);
        const float2 fb = bf16x2_to_float2(bw[u]);
        const float d0 = fa.x - fb.x, d1 = fa.y - fb.y;
        dsum = fmaf(d0, d0, dsum);
        dsum = fmaf(d1, d1, dsum);
        psum = fmaf(fb.x, fb.x, psum);
        psum = fmaf(fb.y, fb.y, psum);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
      psum += __shfl_xor_sync(0xffffffffu, psum, o);
    }
    if (lane == 0) flags[c] = (dsum >= tau2 * psum) ? 1 : 0;
  }

  // Last-block-done: the block that takes the final ticket compacts.
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_is_last = (atomicAdd(ticket, 1u) == gridDim.x - 1) ? 1u : 0u;
  __syncthreads();
  if (!s_is_last) return;
  __threadfence();

  int running = 0;
  const int chunk = blockDim.x * kGateItems;
  for (int base = 0; base < n_prev; base += chunk) {
    const int first = base + threadIdx.x * kGateItems;
    uint8_t f[kGateItems];
    int cnt = 0;
#pragma unroll
    for (int q = 0; q < kGateItems; ++q) {
      const int c = first + q;
      f[q] = (c < n_prev) ? __ldcg(flags + c) : 0;
      cnt += f[q];
    }
    int total;
    int pos = running + block_exclusive_scan(cnt, warp_sums, &total);
#pragma unroll
    for (int q = 0; q < kGateItems; ++q) {
      if (f[q]) {
        const int c = first + q;
        const int t = prev_active ? prev_active[c] : c;
        if (pos < out_cap) {
          active_out[pos] = t;
          slot_out[t] = pos;
        }
        ++pos;
      }
    }
    running += total;
  }
  if (threadIdx.x == 0) {
    if (running > out_cap) set_error(err, FLASHLOOP_DEVERR_CAPACITY);
    *n_out = running < out_cap ? running : out_cap;
    *ticket = 0u;  // ready for the next launch
  }
}

int launch_gate(const flashloop_params* p, const uint16_t* x_cur, const uint16_t* x_prev,
                const int32_t* prev_active, const int32_t* n_prev, int prev_cap, int32_t* active_out,
                int32_t* slot_out, int32_t* n_active_out, int out_cap, void* workspace,
                int32_t* err_word, cudaStream_t stream) {
  const Workspace w = workspace_layout(p);
  const int rows_per_block = kGateThreads / 32;
  int grid = (prev_cap + rows_per_block - 1) / rows_per_block;
  const int max_grid = 148 * 8;
  if (grid > max_grid) grid = max_grid;
  if (grid < 1) grid = 1;
  const float tau2 = p->tau * p->tau;
  gate_kernel<<<grid, kGateThreads, 0, stream>>>(
      x_cur, x_prev, p->seq, p->d_model, prev_active, n_prev, prev_cap, tau2,
      ws_ptr<uint8_t>(workspace, w.flags), ws_ptr<unsigned int>(workspace, w.ticket), active_out,
      slot_out, n_active_out, out_cap, err_word);
  return launch_status();
}

// (a1, top-k retention) [FlashLoop §4.1, App. D.1]: the normalised change
// ||x_cur - x_prev||^2 / ||x_prev||^2 of every candidate (float32 sums, IEEE
// division; a zero previous row gets +inf if it changed, 0 if not), written
// compactly at the candidate's position.  One warp per candidate row.
__global__ void __launch_bounds__(kGateThreads)
gate_key_kernel(const uint16_t* __restrict__ x_cur, const uint16_t* __restrict__ x_prev, int S, int d,
                const int32_t* __restrict__ prev_active, const int32_t* __restrict__ n_prev_ptr, int prev_cap,
                float* __restrict__ key, int32_t* __restrict__ err) {
  int n_prev = prev_active ? *n_prev_ptr : S;
  if (n_prev > prev_cap) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_error(err, FLASHLOOP_DEVERR_CAPACITY);
    n_prev = prev_cap;
  }
  const int lane = threadIdx.x & 31;
  const int warps_per_block = blockDim.x >> 5;
  const int vecs = d >> 3;
  for (int c = blockIdx.x * warps_per_block + (threadIdx.x >> 5); c < n_prev; c += gridDim.x * warps_per_block) {
    const int t = prev_active ? prev_active[c] : c;
    if (t < 0 || t >= S) {
      if (lane == 0) {
        set_error(err, FLASHLOOP_DEVERR_INDEX);
        key[c] = -INFINITY;
      }
      continue;
    }
    const uint4* xc = reinterpret_cast<const uint4*>(x_cur + (size_t)t * d);
    const uint4* xp = reinterpret_cast<const uint4*>(x_prev + (size_t)t * d);
    float dsum = 0.f, psum = 0.f;
    for (int v = lane; v < vecs; v += 32) {
      const uint4 a = __ldcs(xc + v);
      const uint4 b = __ldcs(xp + v);
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
      const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 fa = bf16x2_to_float2(aw[u]);
        const float2 fb = bf16x2_to_float2(bw[u]);
        const float d0 = fa.x - fb.x, d1 = fa.y - fb.y;
        dsum = fmaf(d0, d0, dsum);
        dsum = fmaf(d1, d1, dsum);
        psum = fmaf(fb.x, fb.x, psum);
        psum = fmaf(fb.y, fb.y, psum);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
      psum += __shfl_xor_sync(0xffffffffu, psum, o);
    }
    if (lane == 0) key[c] = psum > 0.f ? __fdiv_rn(dsum, psum) : (dsum > 0.f ? INFINITY : 0.f);
  }
}

// slot[t] = position of token t in the ascending list active[0..*n), else -1.
__global__ void slot_map_kernel(const int32_t* __restrict__ active, const int32_t* __restrict__ n_ptr, int S,
                                int32_t* __restrict__ slot) {
  const int n = *n_ptr;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < S; t += gridDim.x * blockDim.x) {
    int lo = 0, hi = n;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (active[mid] < t) lo = mid + 1;
      else hi = mid;
    }
    slot[t] = (lo < n && active[lo] == t) ? lo : -1;
  }
}

int launch_topk(const flashloop_params*, const float*, const int32_t*, int, int, int32_t*, int32_t*,
                cudaStream_t, const float* row_m = nullptr, const float* row_z = nullptr,
                float* probs_out = nullptr, const int32_t* n_dev = nullptr, int32_t* k_out = nullptr,
                const int32_t* out_map = nullptr);

// Top-k retention: keys, then the radix select over the candidates' keys
// (positions mapped back to tokens, ascending), then the slot map.
int launch_gate_topk(const flashloop_params* p, const uint16_t* x_cur, const uint16_t* x_prev,
                     const int32_t* prev_active, const int32_t* n_prev, int prev_cap, int budget,
                     int32_t* active_out, int32_t* slot_out, int32_t* n_active_out, void* workspace,
                     int32_t* err_word, cudaStream_t stream) {
  const Workspace w = workspace_layout(p);
  float* key = ws_ptr<float>(workspace, w.keys);
  const int rows_per_block = kGateThreads / 32;
  int grid = (prev_cap + rows_per_block - 1) / rows_per_block;
  if (grid > 148 * 8) grid = 148 * 8;
  if (grid < 1) grid = 1;
  gate_key_kernel<<<grid, kGateThreads, 0, stream>>>(x_cur, x_prev, p->seq, p->d_model, prev_active, n_prev,
                                                     prev_cap, key, err_word);
  int rc = launch_status();
  if (rc != FLASHLOOP_OK) return rc;
  flashloop_params ps = *p;
  ps.n_heads = 1;
  ps.seq = prev_cap;
  rc = launch_topk(&ps, key, nullptr, 0, budget, active_out, err_word, stream, nullptr, nullptr, nullptr,
                   prev_active ? n_prev : nullptr, n_active_out, prev_active);
  if (rc != FLASHLOOP_OK) return rc;
  int sgrid = (p->seq + 255) / 256;
  if (sgrid > 148 * 8) sgrid = 148 * 8;
  slot_map_kernel<<<sgrid, 256, 0, stream>>>(active_out, n_active_out, p->seq, slot_out);
  return launch_status();
}

}  // namespace fl
