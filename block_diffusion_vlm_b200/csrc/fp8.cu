// FP8 (E4M3) row quantisation of a bf16 matrix: the weight side of the W8A8
// projections [Fast-dVLM technical overview (ocdem.com), section 2.3.2: the
// served model is quantised to W8A8 FP8 (SmoothQuant)].  The pages fix no
// format or granularity; the reading taken here: E4M3 in its finite variant
// (largest value 448), one scale per row s_r = max_k |a_rk| / 448 (1 for an
// all-zero row), codes = round-to-nearest-even(a / s_r), so that
// a_rk ~ s_r * code_rk.
//
// The quotient a / s_r is formed in fp64 and rounded to E4M3 straight from
// fp64 (no detour through fp32, which could round twice), so the codes are
// exactly those of the definition.  Rows are output channels for weights.
#include "kernels.h"
#include "ptx.cuh"

namespace dvlm {

// E4M3 code (finite variant: 4 exponent bits with bias 7, 3 mantissa bits,
// subnormals 2^-9 apart, largest magnitude 448, no infinities) of the real x,
// round to nearest, ties to even; magnitudes beyond 448 saturate to 448.
__device__ __forceinline__ uint8_t e4m3_code_rne(double x) {
  const uint8_t sign = x < 0.0 ? 0x80 : 0x00;
  double a = fabs(x);
  if (!(a > 0.0)) return sign;  // zero (and NaN, which a finite input never gives) -> 0
  if (a >= 448.0) return sign | 0x7E;
  int ex;
  frexp(a, &ex);                // a = m 2^ex, 0.5 <= m < 1: the leading bit is 2^(ex-1)
  int E = ex - 1;
  if (E < -6) {                 // subnormal range: multiples of 2^-9
    const double q = rint(ldexp(a, 9));
    return sign | static_cast<uint8_t>(q);  // q = 8 is the smallest normal, code 0x08
  }
  double q = rint(ldexp(a, 3 - E));         // 8 <= q <= 16: 3 mantissa bits below the leading one
  if (q >= 16.0) {
    q = 8.0;
    ++E;
  }
  if (E > 8 || (E == 8 && q > 14.0)) return sign | 0x7E;  // rounded past 448
  return sign | static_cast<uint8_t>(((E + 7) << 3) | (static_cast<int>(q) - 8));
}

// One CTA (256 threads) per row: the row's largest magnitude, then its codes.
__global__ void quantize_rows_e4m3_kernel(const bf16* __restrict__ a, int K, uint8_t* __restrict__ codes,
                                          float* __restrict__ scales) {
  const size_t row = blockIdx.x;
  const bf16* src = a + row * K;
  float amax = 0.f;
  for (int k = threadIdx.x; k < K; k += blockDim.x) amax = fmaxf(amax, fabsf(__bfloat162float(src[k])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  __shared__ float red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
  for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) amax = fmaxf(amax, red[w]);
  const double s = amax > 0.f ? static_cast<double>(amax) / 448.0 : 1.0;
  if (threadIdx.x == 0) scales[row] = static_cast<float>(s);
  uint8_t* dst = codes + row * K;
  for (int k = threadIdx.x; k < K; k += blockDim.x)
    dst[k] = e4m3_code_rne(static_cast<double>(__bfloat162float(src[k])) / s);
}

cudaError_t launch_quantize_rows_e4m3(const bf16* a, int rows, int K, uint8_t* codes, float* scales, cudaStream_t s) {
  if (rows < 1 || K < 1) return cudaErrorInvalidValue;
  quantize_rows_e4m3_kernel<<<rows, 256, 0, s>>>(a, K, codes, scales);
  return cudaGetLastError();
}

}  // namespace dvlm
