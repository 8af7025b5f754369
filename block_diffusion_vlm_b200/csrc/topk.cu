// Top-k commit of a block-decoding step: the k still-masked positions of
// highest top-1 probability are committed, lower position first on ties
// [Look Only When Needed, background on confidence-guided unmasking: the
// baseline dVLM schedule unmasks a fixed number k of the most confident
// positions per step], and the divergence-first variant of certificate-guided
// routing's FULL branch [Look Only When Needed, method step (3): positions
// whose TEXT-ONLY top-1 differs from the FULL top-1 first, each group by FULL
// confidence].  It runs on the fused LM head's per-row outputs (top-1 id and
// probability); one CTA ranks at most 128 rows.
#include <cuda_runtime.h>

#include <cstdint>

namespace dvlm {

constexpr int kTopkMaxRows = 128;

// Row r's rank among the masked rows in the order (descending p1, ascending
// position) -- with kDivergentFirst, rows whose other_ids differ from ids
// (divergent) come before the agreeing ones, each group in that order -- and
// r commits when it is masked and its rank is below k.  Every thread reads
// the whole row set from shared memory before any write, so the in-place
// update of masked[] cannot race with the ranking.
template <bool kDivergentFirst>
__global__ void topk_commit_kernel(const float* __restrict__ p1, const int32_t* __restrict__ ids,
                                   const int32_t* __restrict__ other_ids, uint8_t* masked, int32_t* tokens, int R,
                                   int k, uint8_t* commit, int32_t* n_commit) {
  __shared__ float s_p[kTopkMaxRows];
  __shared__ uint8_t s_m[kTopkMaxRows];
  __shared__ uint8_t s_a[kTopkMaxRows];   // 1 = agrees (kDivergentFirst)
  const int r = threadIdx.x;
  if (r < R) {
    s_p[r] = p1[r];
    s_m[r] = masked[r] != 0;
    s_a[r] = kDivergentFirst ? (other_ids[r] == ids[r]) : 0;
  }
  __syncthreads();
  int n_masked = 0, rank = 0;
  const float mine = r < R ? s_p[r] : 0.f;
  const int my_a = r < R ? s_a[r] : 0;
  for (int s = 0; s < R; ++s) {
    if (!s_m[s]) continue;
    ++n_masked;
    const bool before_in_group = s_p[s] > mine || (s_p[s] == mine && s < r);
    if (s_a[s] < my_a || (s_a[s] == my_a && before_in_group)) ++rank;
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

cudaError_t launch_topk_commit(const float* p1, const int32_t* ids, const int32_t* other_ids, uint8_t* masked,
                               int32_t* tokens, int R, int k, uint8_t* commit, int32_t* n_commit, cudaStream_t s) {
  if (other_ids)
    topk_commit_kernel<true><<<1, kTopkMaxRows, 0, s>>>(p1, ids, other_ids, masked, tokens, R, k, commit, n_commit);
  else
    topk_commit_kernel<false><<<1, kTopkMaxRows, 0, s>>>(p1, ids, nullptr, masked, tokens, R, k, commit, n_commit);
  return cudaGetLastError();
}

}  // namespace dvlm
