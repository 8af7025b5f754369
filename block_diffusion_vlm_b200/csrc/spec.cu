// Speculative verify + longest-prefix accept + in-place KV truncation
// [Fast-dVLM technical overview (ocdem.com), section 2.3.1: the causal pass
// checks the diffusion draft, the longest verified prefix is kept and the KV
// cache is truncated and updated].
#include "kernels.h"
#include "ptx.cuh"

namespace dvlm {

// Truncate sequence i from L0+B to L0+k and optionally poison the dropped
// slots of every layer with bf16 NaN.  Run by one CTA.
__device__ void spec_finish(int i, int b, int B, int k, int32_t* accept_len, int32_t* cache_len, int poison,
                            bf16* kc, bf16* vc, int n_layers, int Hkv, int D, int Lmax, int* status) {
  __shared__ int s_old;
  if (threadIdx.x == 0) {
    accept_len[i] = k;
    s_old = cache_len ? cache_len[i] : 0;
    if (cache_len) cache_len[i] = s_old - (B - k);
  }
  __syncthreads();
  if (!poison || !cache_len) return;
  const int lo = s_old - B + k, hi = s_old;
  if (lo < 0 || hi > Lmax) {
    if (threadIdx.x == 0) record_error(status, DVLM_ERR_BOUNDS);
    return;
  }
  const bf16 nan = __ushort_as_bfloat16(static_cast<unsigned short>(0x7FC0));
  const int n_slots = hi - lo;
  const long long total = static_cast<long long>(n_layers) * Hkv * n_slots * D;
  for (long long e = threadIdx.x; e < total; e += blockDim.x) {
    const int d = static_cast<int>(e % D);
    long long r = e / D;
    const int slot = lo + static_cast<int>(r % n_slots);
    r /= n_slots;
    const int h = static_cast<int>(r % Hkv);
    const int l = static_cast<int>(r / Hkv);
    const size_t head = (static_cast<size_t>(l) * b + i) * Hkv + h;
    kc[(head * Lmax + slot) * D + d] = nan;
    vc[(head * D + d) * Lmax + slot] = nan;
  }
}

// Grid (splits, B, b): each CTA takes the argmax of one slice of one row;
// the last CTA of a sequence merges the slices (lowest id on ties; NaN
// logits never win) and finishes the sequence.
__global__ void spec_logits_kernel(const bf16* __restrict__ logits, const int32_t* __restrict__ draft, int b,
                                   int B, int V, int32_t* accept_len, int32_t* cache_len, int poison, bf16* kc,
                                   bf16* vc, int n_layers, int Hkv, int D, int Lmax, float* part, int* cnt,
                                   int* status) {
  const int split = blockIdx.x, j = blockIdx.y, i = blockIdx.z;
  const int splits = gridDim.x;
  const int per = ((V + splits - 1) / splits + 7) / 8 * 8;
  const int v0 = split * per, v1 = min(V, v0 + per);
  const bf16* row = logits + (static_cast<size_t>(i) * B + j) * V;
  float best = -INFINITY;
  int bidx = 0x7fffffff;
  const bool vec = (V % 8) == 0;  // rows start 16-byte aligned only then
  // Four 16-byte loads in flight per thread, scanned in index order (a tie
  // keeps the earlier, lower id).
  const int step = blockDim.x * 8;
  int v = v0 + threadIdx.x * 8;
  if (vec) {
    for (; v + 3 * step + 8 <= v1; v += 4 * step) {
      uint4 w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) w[u] = *reinterpret_cast<const uint4*>(row + v + u * step);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bf16* e = reinterpret_cast<const bf16*>(&w[u]);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float x = __bfloat162float(e[q]);
          if (x > best) {
            best = x;
            bidx = v + u * step + q;
          }
        }
      }
    }
  }
  for (; v < v1; v += step) {
    if (vec && v + 8 <= v1) {
      const uint4 w = *reinterpret_cast<const uint4*>(row + v);
      const bf16* e = reinterpret_cast<const bf16*>(&w);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float x = __bfloat162float(e[q]);
        if (x > best) {
          best = x;
          bidx = v + q;
        }
      }
    } else {
      for (int q = v; q < v1; ++q) {
        const float x = __bfloat162float(row[q]);
        if (x > best) {
          best = x;
          bidx = q;
        }
      }
    }
  }
  __shared__ float sb[256];
  __shared__ int si[256];
  __shared__ int s_last;
  sb[threadIdx.x] = best;
  si[threadIdx.x] = bidx;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) {
      const float b2 = sb[threadIdx.x + o];
      const int i2 = si[threadIdx.x + o];
      if (b2 > sb[threadIdx.x] || (b2 == sb[threadIdx.x] && i2 < si[threadIdx.x])) {
        sb[threadIdx.x] = b2;
        si[threadIdx.x] = i2;
      }
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    float* p = part + ((static_cast<size_t>(i) * B + j) * splits + split) * 2;
    __stcg(&p[0], sb[0]);
    __stcg(&p[1], __int_as_float(si[0]));
    __threadfence();
    const int old = atomicAdd(&cnt[i], 1);
    s_last = (old == B * splits - 1) ? 1 : 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  __shared__ int s_v[64];
  if (threadIdx.x < B) {
    float bb = -INFINITY;
    int ii = 0x7fffffff;
    // the row's split results in split order, eight loads in flight
    const float2* p = reinterpret_cast<const float2*>(part) + (static_cast<size_t>(i) * B + threadIdx.x) * splits;
    for (int s0 = 0; s0 < splits; s0 += 8) {
      float2 r[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) r[q] = s0 + q < splits ? __ldcg(&p[s0 + q]) : make_float2(-INFINITY, 0.f);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (s0 + q >= splits) break;
        const float x = r[q].x;
        const int ix = __float_as_int(r[q].y);
        if (x > bb || (x == bb && ix < ii)) {
          bb = x;
          ii = ix;
        }
      }
    }
    s_v[threadIdx.x] = ii;
  }
  __syncthreads();
  __shared__ int s_k;
  if (threadIdx.x == 0) {
    int k = 0;
    while (k < B && s_v[k] == draft[static_cast<size_t>(i) * B + k]) ++k;
    s_k = k;
    cnt[i] = 0;
  }
  __syncthreads();
  spec_finish(i, b, B, s_k, accept_len, cache_len, poison, kc, vc, n_layers, Hkv, D, Lmax, status);
}

__global__ void spec_ids_kernel(const int32_t* vids, const int32_t* draft, int b, int B, int32_t* accept_len,
                                int32_t* cache_len, int poison, bf16* kc, bf16* vc, int n_layers, int Hkv, int D,
                                int Lmax, int* status) {
  const int i = blockIdx.x;
  __shared__ int s_k;
  if (threadIdx.x == 0) {
    int k = 0;
    while (k < B && vids[static_cast<size_t>(i) * B + k] == draft[static_cast<size_t>(i) * B + k]) ++k;
    s_k = k;
  }
  __syncthreads();
  spec_finish(i, b, B, s_k, accept_len, cache_len, poison, kc, vc, n_layers, Hkv, D, Lmax, status);
}

cudaError_t launch_spec_logits(const bf16* logits, const int32_t* draft, int b, int B, int V, int32_t* accept_len,
                               int32_t* cache_len, int poison, bf16* kc, bf16* vc, int n_layers, int Hkv, int D,
                               int Lmax, float* ws_part, int* ws_cnt, int splits, int* status, cudaStream_t s) {
  spec_logits_kernel<<<dim3(splits, B, b), 256, 0, s>>>(logits, draft, b, B, V, accept_len, cache_len, poison, kc,
                                                         vc, n_layers, Hkv, D, Lmax, ws_part, ws_cnt, status);
  return cudaGetLastError();
}

cudaError_t launch_spec_ids(const int32_t* vids, const int32_t* draft, int b, int B, int32_t* accept_len,
                            int32_t* cache_len, int poison, bf16* kc, bf16* vc, int n_layers, int Hkv, int D,
                            int Lmax, int* status, cudaStream_t s) {
  spec_ids_kernel<<<b, 256, 0, s>>>(vids, draft, b, B, accept_len, cache_len, poison, kc, vc, n_layers, Hkv, D,
                                    Lmax, status);
  return cudaGetLastError();
}

}  // namespace dvlm
