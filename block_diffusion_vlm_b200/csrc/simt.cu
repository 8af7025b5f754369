// fp32 CUDA-core path of the decode step, for the tiny fp32 model (hidden 32,
// head_dim 16, vocab 256).  fp32 storage and fp32 arithmetic throughout; the
// 1e-4 parity bound rules out TF32 tensor cores, and at these sizes the work
// is launch-latency bound anyway.  Same definitions as the bf16 path.
#include "finalize.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace dvlm {

__global__ void f32_embed_kernel(const float* E, const float* rows_in, int n_src, const int32_t* tokens,
                                 const uint8_t* masked, int mask_id, int H, int V, float* x, int* status) {
  const int t = blockIdx.x;
  const float* src;
  if (t < n_src) {
    src = rows_in + static_cast<size_t>(t) * H;
  } else {
    const int j = t - n_src;
    int id = (masked && masked[j]) ? mask_id : tokens[j];
    if (id < 0 || id >= V) {
      if (threadIdx.x == 0) record_error(status, DVLM_ERR_BOUNDS);
      id = 0;
    }
    src = E + static_cast<size_t>(id) * H;
  }
  for (int c = threadIdx.x; c < H; c += blockDim.x) x[static_cast<size_t>(t) * H + c] = src[c];
}

// r[t] = 1 / sqrt(mean(x[t]^2) + eps)
__global__ void f32_rowscale_kernel(const float* x, int ld, int n_rows, int H, float eps, float* r) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n_rows) return;
  float s = 0.f;
  for (int c = 0; c < H; ++c) {
    const float v = x[static_cast<size_t>(t) * ld + c];
    s += v * v;
  }
  r[t] = 1.0f / sqrtf(s / H + eps);
}

// y[t][n] = r[t] * sum_k x[t][k] W[n][k]   (r = 1 when NULL)
__global__ void f32_gemm_kernel(const float* x, int ld_x, const float* W, int n_out, int K, int n_rows,
                                const float* r, float* y, int ld_y) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int t = blockIdx.y;
  if (n >= n_out || t >= n_rows) return;
  const float* xr = x + static_cast<size_t>(t) * ld_x;
  const float* wr = W + static_cast<size_t>(n) * K;
  float acc = 0.f;
  for (int k = 0; k < K; ++k) acc += xr[k] * wr[k];
  y[static_cast<size_t>(t) * ld_y + n] = r ? acc * r[t] : acc;
}

// RoPE on query/key heads and scatter: q_out [n_rows][Hq*D], K [Hkv][Lmax][D],
// V^T [Hkv][D][Lmax] at slot L+t.  One thread per (t, head, pair).
__global__ void f32_rope_scatter_kernel(const float* y, int n_rows, int nq, int nkv, int D, const int* d_len,
                                        int L_static, double log2_base, float* q_out, float* kc, float* vc,
                                        int Lmax) {
  const int half = D / 2;
  const int heads = nq + 2 * nkv;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_rows * heads * half) return;
  const int j = idx % half;
  const int hh = (idx / half) % heads;
  const int t = idx / (half * heads);
  const int L = d_len ? *d_len : L_static;
  const int pos = L + t;
  const float* yr = y + static_cast<size_t>(t) * heads * D + static_cast<size_t>(hh) * D;
  const float x1 = yr[j], x2 = yr[j + half];
  if (hh < nq + nkv) {
    const double inv = exp2(-(2.0 * j / D) * log2_base);
    double sn, cs;
    sincos(static_cast<double>(pos) * inv, &sn, &cs);
    const float c = static_cast<float>(cs), s = static_cast<float>(sn);
    const float o1 = x1 * c - x2 * s, o2 = x2 * c + x1 * s;
    if (hh < nq) {
      float* q = q_out + static_cast<size_t>(t) * nq * D + static_cast<size_t>(hh) * D;
      q[j] = o1;
      q[j + half] = o2;
    } else {
      float* k = kc + (static_cast<size_t>(hh - nq) * Lmax + pos) * D;
      k[j] = o1;
      k[j + half] = o2;
    }
  } else {
    const int h = hh - nq - nkv;
    vc[(static_cast<size_t>(h) * D + j) * Lmax + pos] = x1;
    vc[(static_cast<size_t>(h) * D + j + half) * Lmax + pos] = x2;
  }
}

__global__ void f32_add_kernel(float* resid, int ld_r, const float* y, int ld_y, int n_rows, int H) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_rows * H) return;
  const int t = i / H, c = i % H;
  resid[static_cast<size_t>(t) * ld_r + c] += y[static_cast<size_t>(t) * ld_y + c];
}

__global__ void f32_swiglu_kernel(const float* g, const float* u, float* act, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float a = g[i];
  act[i] = a / (1.0f + expf(-a)) * u[i];
}

// One thread per (batch, row, query head): softmax over the visible slots
// (clean row t: 0..L+t; noisy row: 0..L+n_rows-1), online in fp32.
__global__ void f32_attn_kernel(const float* q, float* out, const float* kc, const float* vc, int n_batch,
                                int n_rows, int n_clean, int L_static, const int* d_len, int Lmax, int Hq, int Hkv,
                                int D, float scale) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_batch * n_rows * Hq) return;
  const int h = idx % Hq;
  const int t = (idx / Hq) % n_rows;
  const int b = idx / (Hq * n_rows);
  const int L = d_len ? *d_len : L_static;
  const int g = h / (Hq / Hkv);
  const int vis = (t < n_clean) ? (L + t + 1) : (L + n_rows);
  const float* qr = q + ((static_cast<size_t>(b) * n_rows + t) * Hq + h) * D;
  const float* K = kc + (static_cast<size_t>(b) * Hkv + g) * Lmax * D;
  const float* Vt = vc + (static_cast<size_t>(b) * Hkv + g) * D * Lmax;
  float o[128];
  for (int d = 0; d < D; ++d) o[d] = 0.f;
  float m = -INFINITY, l = 0.f;
  for (int j = 0; j < vis; ++j) {
    float s = 0.f;
    for (int d = 0; d < D; ++d) s += qr[d] * K[static_cast<size_t>(j) * D + d];
    s *= scale;
    const float mn = fmaxf(m, s);
    const float a = expf(m - mn), p = expf(s - mn);
    l = l * a + p;
    for (int d = 0; d < D; ++d) o[d] = o[d] * a + p * Vt[static_cast<size_t>(d) * Lmax + j];
    m = mn;
  }
  float* dst = out + ((static_cast<size_t>(b) * n_rows + t) * Hq + h) * D;
  for (int d = 0; d < D; ++d) dst[d] = o[d] / l;
}

// One CTA per row: logits over the vocabulary, (max, sum exp, argmax) per
// thread, merged in thread order.
__global__ void f32_lmhead_kernel(const float* hidden, const float* w, int R, int H, int V, const float* r,
                                  float* p1, int32_t* ids) {
  const int row = blockIdx.x;
  const float* h = hidden + static_cast<size_t>(row) * H;
  const float scale = r ? r[row] : 1.0f;
  float m = -INFINITY, s = 0.f;
  int idx = 0x7fffffff;
  for (int v = threadIdx.x; v < V; v += blockDim.x) {
    const float* wr = w + static_cast<size_t>(v) * H;
    float acc = 0.f;
    for (int k = 0; k < H; ++k) acc += h[k] * wr[k];
    const float l = acc * scale;
    if (l > m) {
      s = s * expf(m - l) + 1.0f;
      m = l;
      idx = v;
    } else {
      s += expf(l - m);
    }
  }
  __shared__ float sm[256], ss[256];
  __shared__ int si[256];
  sm[threadIdx.x] = m;
  ss[threadIdx.x] = s;
  si[threadIdx.x] = idx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float M = -INFINITY, S = 0.f;
    int I = 0x7fffffff;
    for (int k = 0; k < blockDim.x; ++k) {
      if (ss[k] == 0.f) continue;
      if (S == 0.f) {
        M = sm[k];
        S = ss[k];
        I = si[k];
      } else if (sm[k] > M) {
        S = S * expf(M - sm[k]) + ss[k];
        M = sm[k];
        I = si[k];
      } else if (sm[k] == M) {
        S += ss[k];
        I = si[k] < I ? si[k] : I;
      } else {
        S += ss[k] * expf(sm[k] - M);
      }
    }
    p1[row] = 1.0f / S;
    ids[row] = I;
  }
}

__global__ void f32_finalize_kernel(const float* p1, const int32_t* ids, LmArgs a) {
  __shared__ FinalizeSmem fs;
  const int r = threadIdx.x;
  if (r < a.R) {
    fs.p1[r] = p1[r];
    fs.id[r] = ids[r];
  }
  __syncthreads();
  finalize_rows(r, a, fs, [] { __syncthreads(); });
}

// ------------------------------------------------------------------ host
static inline int cdiv(int a, int b) { return (a + b - 1) / b; }

cudaError_t f32_embed(const float* E, const float* rows_in, int n_src, const int32_t* tokens,
                      const uint8_t* masked, int mask_id, int n_rows, int H, int V, float* x, int* status,
                      cudaStream_t s) {
  f32_embed_kernel<<<n_rows, 64, 0, s>>>(E, rows_in, n_src, tokens, masked, mask_id, H, V, x, status);
  return cudaGetLastError();
}

cudaError_t f32_rowscale(const float* x, int ld, int n_rows, int H, float eps, float* r, cudaStream_t s) {
  f32_rowscale_kernel<<<cdiv(n_rows, 64), 64, 0, s>>>(x, ld, n_rows, H, eps, r);
  return cudaGetLastError();
}

cudaError_t f32_gemm(const float* x, int ld_x, const float* W, int n_out, int K, int n_rows, const float* r,
                     float* y, int ld_y, cudaStream_t s) {
  f32_gemm_kernel<<<dim3(cdiv(n_out, 128), n_rows), 128, 0, s>>>(x, ld_x, W, n_out, K, n_rows, r, y, ld_y);
  return cudaGetLastError();
}

cudaError_t f32_rope_scatter(const float* y, int n_rows, int nq, int nkv, int D, const int* d_len, int L_static,
                             double log2_base, float* q_out, float* kc, float* vc, int Lmax, cudaStream_t s) {
  const int n = n_rows * (nq + 2 * nkv) * (D / 2);
  f32_rope_scatter_kernel<<<cdiv(n, 128), 128, 0, s>>>(y, n_rows, nq, nkv, D, d_len, L_static, log2_base, q_out,
                                                       kc, vc, Lmax);
  return cudaGetLastError();
}

cudaError_t f32_add(float* resid, int ld_r, const float* y, int ld_y, int n_rows, int H, cudaStream_t s) {
  f32_add_kernel<<<cdiv(n_rows * H, 128), 128, 0, s>>>(resid, ld_r, y, ld_y, n_rows, H);
  return cudaGetLastError();
}

cudaError_t f32_swiglu(const float* g, const float* u, float* act, int n, cudaStream_t s) {
  f32_swiglu_kernel<<<cdiv(n, 128), 128, 0, s>>>(g, u, act, n);
  return cudaGetLastError();
}

cudaError_t f32_attention(const float* q, float* out, const float* kc, const float* vc, int n_batch, int n_rows,
                          int n_clean, int L, const int* d_len, int Lmax, int Hq, int Hkv, int D, float scale,
                          cudaStream_t s) {
  const int n = n_batch * n_rows * Hq;
  f32_attn_kernel<<<cdiv(n, 64), 64, 0, s>>>(q, out, kc, vc, n_batch, n_rows, n_clean, L, d_len, Lmax, Hq, Hkv, D,
                                             scale);
  return cudaGetLastError();
}

cudaError_t f32_lmhead(const float* hidden, const float* w, int R, int H, int V, const float* r, float* p1_buf,
                       int32_t* id_buf, const LmArgs& a, cudaStream_t s) {
  f32_lmhead_kernel<<<R, 256, 0, s>>>(hidden, w, R, H, V, r, p1_buf, id_buf);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  f32_finalize_kernel<<<1, 128, 0, s>>>(p1_buf, id_buf, a);
  return cudaGetLastError();
}

}  // namespace dvlm
