// Small kernels of the decode step: embedding gather, block bookkeeping and
// the decode driver's speculative accept.
#include "kernels.h"
#include "ptx.cuh"

namespace dvlm {

// Row t < n_src copies rows_in[t]; row t >= n_src gathers E[id] with
// id = tokens[t - n_src], or the [MASK] row when masked[t - n_src] != 0
// [Fast-dVLM walkthrough (itsolotime.com), section 4: vision tokens enter as
// embeddings, masked response positions as [MASK]].  Also writes the row's
// sum of squares per 128 features (ssq_out[p][t], p = feature tile) for the
// first RMSNorm.  One CTA (4 warps) per row; warp w owns feature tiles
// w, w+4, ...  Rows n_rows..NT-1 are left untouched.
__global__ void embed_bf16_kernel(const bf16* __restrict__ E, const bf16* __restrict__ rows_in, int n_src,
                                  const int32_t* __restrict__ tokens, const uint8_t* __restrict__ masked,
                                  int mask_id, int H, int V, bf16* __restrict__ x, float* __restrict__ ssq_out,
                                  int NT, int* status) {
  griddep_wait();
  griddep_launch_dependents();
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bf16* src;
  if (t < n_src) {
    src = rows_in + static_cast<size_t>(t) * H;
  } else {
    const int j = t - n_src;
    int id = (masked && masked[j]) ? mask_id : tokens[j];
    if (id < 0 || id >= V) {
      record_error(status, DVLM_ERR_BOUNDS);
      id = 0;
    }
    src = E + static_cast<size_t>(id) * H;
  }
  bf16* dst = x ? x + static_cast<size_t>(t) * H : nullptr;  // NULL: sums of squares only
  for (int p = warp; p < H / 128; p += 4) {
    const int c = p * 128 + lane * 4;
    const uint2 w = *reinterpret_cast<const uint2*>(src + c);
    if (dst) *reinterpret_cast<uint2*>(dst + c) = w;
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&w);
    const float2 a = __bfloat1622float2(h2[0]), b = __bfloat1622float2(h2[1]);
    float s = a.x * a.x + a.y * a.y + b.x * b.x + b.y * b.y;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) ssq_out[p * NT + t] = s;
  }
}

cudaError_t launch_embed_bf16(const bf16* E, const bf16* rows_in, int n_src, const int32_t* tokens,
                              const uint8_t* masked, int mask_id, int n_rows, int H, int V, bf16* x,
                              float* ssq_out, int NT, int* status, bool pdl, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_rows);
  cfg.blockDim = dim3(128);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, embed_bf16_kernel, E, rows_in, n_src, tokens, masked, mask_id, H, V, x, ssq_out,
                            NT, status);
}

// Start of a threshold block: position 0 holds the AR seed (committed when
// ar_seed != 0), every other position is [MASK]
// [Fast-dVLM technical overview (ocdem.com), section 2.2.2: causal-context
// decoding seeds each block with one AR token].
__global__ void block_init_kernel(int32_t* tokens, uint8_t* masked, const int32_t* seed, int B, int mask_id,
                                  int ar_seed, int32_t* n_remaining) {
  const int j = threadIdx.x;
  if (j < B) {
    const bool first_fixed = ar_seed && j == 0;
    tokens[j] = first_fixed ? *seed : mask_id;
    masked[j] = first_fixed ? 0 : 1;
  }
  if (j == 0) *n_remaining = B - (ar_seed ? 1 : 0);
}

cudaError_t launch_block_init(int32_t* tokens, uint8_t* masked, const int32_t* seed, int B, int mask_id,
                              int ar_seed, int32_t* n_remaining, cudaStream_t s) {
  block_init_kernel<<<1, 32, 0, s>>>(tokens, masked, seed, B, mask_id, ar_seed, n_remaining);
  return cudaGetLastError();
}

// Append n tokens to the output (capped at max_new) and advance its count.
__global__ void emit_kernel(const int32_t* tokens, int n, int32_t* out, int32_t* n_out, int max_new) {
  griddep_wait();
  griddep_launch_dependents();
  const int base = *n_out;
  for (int j = threadIdx.x; j < n; j += blockDim.x)
    if (base + j < max_new) out[base + j] = tokens[j];
  __syncthreads();
  if (threadIdx.x == 0) *n_out = base + n < max_new ? base + n : max_new;
}

cudaError_t launch_emit(const int32_t* tokens, int n, int32_t* out, int32_t* n_out, int max_new, bool pdl,
                        cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(32);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, emit_kernel, tokens, n, out, n_out, max_new);
}

// Decode driver's accept after the causal verify pass (which advanced L by B):
// vids[j] is the verifier's token for position j (j >= 1; position 0 is the
// AR seed and always kept, so k >= 1), k = longest prefix on which
// vids[j] == draft[j], L -= B - k, the next
// seed is vids[k] (the verifier's prediction right after the accepted
// prefix), and the accepted draft tokens are emitted
// [Fast-dVLM technical overview (ocdem.com), section 2.3.1].
__global__ void decode_accept_kernel(const int32_t* vids, const int32_t* draft, int B, int32_t* d_len,
                                     int32_t* seed, int32_t* out, int32_t* n_out, int max_new,
                                     int64_t* accept_hist, int32_t* k_out, int* status) {
  griddep_wait();
  griddep_launch_dependents();
  if (threadIdx.x != 0) return;
  int k = 1;
  while (k < B && vids[k] == draft[k]) ++k;
  if (k_out) *k_out = k;
  *d_len -= B - k;
  *seed = vids[k];
  const int base = *n_out;
  for (int j = 0; j < k && base + j < max_new; ++j) out[base + j] = draft[j];
  *n_out = base + k < max_new ? base + k : max_new;
  if (accept_hist && k < DVLM_HIST) atomicAdd(reinterpret_cast<unsigned long long*>(&accept_hist[k]), 1ull);
}

cudaError_t launch_decode_accept(const int32_t* vids, const int32_t* draft, int B, int32_t* d_len, int32_t* seed,
                                 int32_t* out, int32_t* n_out, int max_new, int64_t* accept_hist, int32_t* k_out,
                                 int* status, bool pdl, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(32);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_accept_kernel, vids, draft, B, d_len, seed, out, n_out, max_new,
                            accept_hist, k_out, status);
}

// Input tokens of the fused draft+verify forward: the draft's B tokens, then
// B candidate blocks of B [MASK] tokens [Fast-dVLM technical overview
// (ocdem.com), section 2.3.1].
__global__ void quad_tokens_kernel(const int32_t* draft, int B, int mask_id, int32_t* qtok) {
  for (int j = threadIdx.x; j < B + B * B; j += blockDim.x) qtok[j] = j < B ? draft[j] : mask_id;
}

cudaError_t launch_quad_tokens(const int32_t* draft, int B, int mask_id, int32_t* qtok, cudaStream_t s) {
  quad_tokens_kernel<<<1, 256, 0, s>>>(draft, B, mask_id, qtok);
  return cudaGetLastError();
}

// Rows of the chosen candidate block (k accepted: block k - 1, rows
// B + (k-1)*B + r of src) into the decode rows x[r], r < B, with each row's
// sum of squares per 128 features (ssq_out[p * NT + r]) for the final norm.
__global__ void select_cand_rows_kernel(const bf16* __restrict__ src, int H, const int32_t* k_dev, int B,
                                        bf16* __restrict__ x, float* __restrict__ ssq_out, int NT) {
  const int r = blockIdx.x;
  const int k = *k_dev;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bf16* row = src + static_cast<size_t>(B + (k - 1) * B + r) * H;
  bf16* dst = x + static_cast<size_t>(r) * H;
  for (int p = warp; p < H / 128; p += 4) {
    const int c = p * 128 + lane * 4;
    const uint2 w = *reinterpret_cast<const uint2*>(row + c);
    *reinterpret_cast<uint2*>(dst + c) = w;
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&w);
    const float2 a = __bfloat1622float2(h2[0]), b = __bfloat1622float2(h2[1]);
    float sq = a.x * a.x + a.y * a.y + b.x * b.x + b.y * b.y;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (lane == 0) ssq_out[p * NT + r] = sq;
  }
}

cudaError_t launch_select_cand_rows(const bf16* src, int H, const int32_t* k_dev, int B, bf16* x, float* ssq_out,
                                    int NT, cudaStream_t s) {
  select_cand_rows_kernel<<<B, 128, 0, s>>>(src, H, k_dev, B, x, ssq_out, NT);
  return cudaGetLastError();
}

// Failure-detection self-test: an mbarrier that expects two arrivals gets
// one, so its phase never completes; the bounded wait must give up after
// `budget` cycles, record DVLM_ERR_TIMEOUT and let the kernel finish.
__global__ void selftest_timeout_kernel(long long budget, int* status, int* waited_out) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 2);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive(&bar);
    const bool ok = mbar_wait_budget(&bar, 0, budget, status);
    *waited_out = ok ? 0 : 1;
  }
}

cudaError_t launch_selftest_timeout(long long budget, int* status, int* waited_out, cudaStream_t s) {
  selftest_timeout_kernel<<<1, 32, 0, s>>>(budget, status, waited_out);
  return cudaGetLastError();
}

}  // namespace dvlm
