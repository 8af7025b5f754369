// Top-k commit of a block-decoding step: the k still-masked positions of
// highest top-1 probability are committed, lower position first on ties
// [Look Only When Needed, background on confidence-guided unmasking: the
// baseline dVLM schedule unmasks a fixed number k of the most confident
// positions per step].  It runs on the fused LM head's per-row outputs (top-1
// id and probability); one CTA ranks at most 128 rows.
#include <cuda_runtime.h>

#include <cstdint>

namespace dvlm {

constexpr int kTopkMaxRows = 128;

// Row r's rank among the masked rows in the order (descending p1, ascending
// position); r commits when it is masked and its rank is below k.  Every
// thread reads the whole row set from shared memory before any write, so the
// in-place update of masked[] cannot race with the ranking.
__global__ void topk_commit_kernel(const float* __restrict__ p1, const int32_t* __restrict__ ids,
                                   uint8_t* masked, int32_t* tokens, int R, int k, uint8_t* commit,
                                   int32_t* n_commit) {
  __shared__ float s_p[kTopkMaxRows];
  __shared__ uint8_t s_m[kTopkMaxRows];
  const int r = threadIdx.x;
  if (r < R) {
    s_p[r] = p1[r];
    s_m[r] = masked[r] != 0;
  }
  __syncthreads();
  int n_masked = 0, rank = 0;
  const float mine = r < R ? s_p[r] : 0.f;
  for (int s = 0; s < R; ++s) {
    if (!s_m[s]) continue;
    ++n_masked;
    if (s_p[s] > mine || (s_p[s] == mine && s < r)) ++rank;
  }
  if (r < R) {
    const bool c = s_m[r] && rank < k;
    if (c) {
      tokens[r] = ids[r];
      masked[r] = 0;
    }
    if (commit) commit[r] = c ? 1 : 0;
  }
  if (r == 0 && n_commit) *n_commit = n_masked < k ? n_masked : k;
}

cudaError_t launch_topk_commit(const float* p1, const int32_t* ids, uint8_t* masked, int32_t* tokens, int R, int k,
                               uint8_t* commit, int32_t* n_commit, cudaStream_t s) {
  topk_commit_kernel<<<1, kTopkMaxRows, 0, s>>>(p1, ids, masked, tokens, R, k, commit, n_commit);
  return cudaGetLastError();
}

}  // namespace dvlm
