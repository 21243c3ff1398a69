// Launch arguments of the attention-update and column-mass kernels.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

namespace fl {

struct AttnArgs {
  int S, H, kc;                 // kc = selected columns per head (S when dense)
  int dense;                    // loop 1: no removal, state starts empty
  const int32_t* rows;          // active tokens (NULL: identity)
  const int32_t* n_rows;        // device count (NULL: S)
  int row_cap;
  const int32_t* cols;          // [H, kc] ascending (NULL: identity)
  const __half* k_new;          // [H, kc, DH]
  const __half* v_new;
  const __half* k_old;
  const __half* v_old;
  const uint16_t* q_new;        // bf16 [S, H*DH]
  const uint16_t* q_old;
  const float* m_in;            // [H, S]
  const float* z_in;
  const float* n_in;            // [H, S, DH]
  float* m_out;
  float* z_out;
  float* n_out;
  uint16_t* o;                  // bf16 [S, H*DH]
  float scale_log2;             // log2(e) / sqrt(dh)
  int32_t* err;
  int mode;                     // 0 running state, 1 / 2 fixed-mass statistics / update pass
  const float* g_in;            // [H, S] selected-column factor of loop r-1 (fixed-mass passes)
  float* g_out;                 // [H, S] (statistics pass; the dense loop writes 1 when set)
  const int32_t* row_cnt;       // [H, row_cap]: selected columns <= the row's token (required with cols)
};

struct ColmassArgs {
  int S, H, kc, kcp;          // kcp = row pitch of k_new
  const int32_t* rows;
  const int32_t* n_rows;
  int row_cap;
  const int32_t* cols;     // [H, kc] ascending (NULL: identity)
  const __half* k_new;     // [H, kcp, DH]
  const uint16_t* q;       // bf16 [S, H*DH]
  const float* m;          // [H, S] final row max (natural units)
  const float* z;          // [H, S]
  float* out;              // [H, S], written at the column tokens
  float scale_log2;
  int32_t* err;
  const float* g;          // [H, S] selected-column factor of the rows (NULL: 1)
};

}  // namespace fl
