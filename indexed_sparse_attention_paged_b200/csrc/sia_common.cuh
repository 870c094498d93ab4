// sia_common.cuh -- small device helpers shared by the libsia kernels.
#pragma once

#include <cstdint>

namespace sia {

// Position of query j of sequence b: q_pos[b][j] when given, else seq_len - J + j (the new
// tokens are the last J positions of the context).  Returns -1 when that position is not
// inside the context (>= seq_len or past the page table), i.e. the query sees nothing.
__device__ __forceinline__ int query_position(const int32_t* seq_lens, const int32_t* q_pos,
                                              int J, int b, int j, long long Lpad,
                                              bool* bad = nullptr) {
  const int L = seq_lens[b];
  const int p = q_pos ? q_pos[(long long)b * J + j] : L - J + j;
  if (p >= L || (long long)p >= Lpad || (q_pos && p < 0)) {
    if (bad) *bad = true;
    return -1;
  }
  return p < 0 ? -1 : p;
}

}  // namespace sia
