// Weight-streaming mainloop shared by the decoder GEMMs and the fused LM head.
//
// Batch-1 decoding re-reads every weight once per forward while only 16 token
// rows flow through it, so these products are bound by HBM, not by the tensor
// cores.  The layout is "swap-AB": the weight tile (128 output features x 64
// k) is the 128-row UMMA A operand, the token rows (NT = 16..128) are the
// N side, and the fp32 accumulator lives in TMEM (128 lanes x NT columns).
//
// Work split (stream-K kernels): the (output tile, 64-wide k block) units are
// cut into P equal contiguous ranges, one per CTA.  A tile whose k range spans
// two or more CTAs is finished by the CTA that streams its first k blocks (the
// last segment of that CTA's range); the others stream their parts first,
// store fp32 partial tiles and count them on a per-tile counter, and the
// finisher adds them in CTA order, so the result is deterministic.  The
// cluster split-K kernels use the same producer and MMA roles with one tile
// per cluster.
//
// Roles (224 threads): warp 0 lane 0 issues TMA loads; warps 1 and 6 (lane 0)
// issue UMMAs for alternate k blocks of each segment into their own TMEM
// accumulators; warps 2..5 run the epilogue (warp w reads TMEM lanes
// 32*(w%4)..+31) and add the two accumulators.
#pragma once
#include "ptx.cuh"

namespace dvlm {

struct SkSched {
  int n_tiles;  // output tiles of 128 rows
  int kb;       // 64-wide k blocks per tile
  int P;        // CTAs
  __host__ __device__ long long units() const { return static_cast<long long>(n_tiles) * kb; }
  __host__ __device__ long long begin(int p) const { return units() * p / P; }
  // CTA whose range holds unit u (largest p with begin(p) <= u).
  __host__ __device__ int cta_of(long long u) const { return static_cast<int>(((u + 1) * P - 1) / units()); }
  __host__ __device__ int first_tile(int p) const { return static_cast<int>(begin(p) / kb); }
};

// Warp roles of the weight-streaming kernels: 0 TMA producer, 1 and 6 MMA
// issuers (alternate k blocks of a segment into their own accumulators: one
// issuing thread cannot keep a 16-column MMA fed at HBM speed), 2..5 epilogue.
constexpr int kWsThreads = 224;
constexpr int kMmaWarp2 = 6;
constexpr int kATileBytes = 128 * 128;  // 128 rows x 64 bf16

// TMEM columns: 2 segment buffers x 2 issuers x NT (a power of two >= 32).
template <int NT>
__host__ __device__ constexpr int tmem_cols_for() {
  return (4 * NT < 32) ? 32 : 4 * NT;
}

// A operand source: one 128-row box, or two 64-row boxes from two tensors
// (gate rows on top, up rows below) so the SwiGLU epilogue sees matching
// gate/up features in one tile.
//
// FP8 (W8A8): the weight tiles are E4M3 codes, 128 rows x 128 k (the same 16 KB
// per stage, twice the k of a bf16 stage), and the producer streams only
// them; the activation codes for the CTA's k range are written into shared
// memory once by the epilogue warps (fp8_quantize_activations).
template <int NT, int STAGES, bool SPLIT_A, bool FP8 = false>
__device__ __forceinline__ void ws_producer(const CUtensorMap* mapA, const CUtensorMap* mapA2,
                                            const CUtensorMap* mapB, uint8_t* sA, uint8_t* sB, uint64_t* full,
                                            uint64_t* empty, const SkSched& sc, long long u0, long long u1,
                                            int a_row_base, int b_row, int* status, volatile int* abort_flag) {
  constexpr int B_BYTES = FP8 ? 0 : NT * 128;
  constexpr int KW = FP8 ? 128 : 64;  // k elements of one stage
  const uint64_t pol_w = l2_policy_evict_first();
  const uint64_t pol_x = l2_policy_evict_last();
  const int n = static_cast<int>(u1 - u0);
  const int pre = n < STAGES ? n : STAGES;
  auto load_a = [&](int s, long long u) {
    const int T = static_cast<int>(u / sc.kb), kk = static_cast<int>(u % sc.kb);
    if (SPLIT_A) {
      tma_load_2d(sA + s * kATileBytes, mapA, &full[s], kk * KW, a_row_base + T * 64, pol_w);
      tma_load_2d(sA + s * kATileBytes + kATileBytes / 2, mapA2, &full[s], kk * KW, a_row_base + T * 64, pol_w);
    } else {
      tma_load_2d(sA + s * kATileBytes, mapA, &full[s], kk * KW, a_row_base + T * 128, pol_w);
    }
  };
  auto load_b = [&](int s, long long u) {
    if (FP8) return;
    const int kk = static_cast<int>(u % sc.kb);
    tma_load_2d(sB + s * B_BYTES, mapB, &full[s], kk * 64, b_row, pol_x);
  };
  // Weights do not depend on the previous kernel: start streaming them before
  // waiting for it (programmatic dependent launch).
  for (int i = 0; i < pre; ++i) {
    mbar_arrive_expect_tx(&full[i], kATileBytes + B_BYTES);
    load_a(i, u0 + i);
  }
  griddep_wait();
  for (int i = 0; i < pre; ++i) load_b(i, u0 + i);
  for (int i = pre; i < n; ++i) {
    const int s = i % STAGES;
    if (!mbar_wait(&empty[s], ((i / STAGES) & 1) ^ 1, status, abort_flag)) return;
    mbar_arrive_expect_tx(&full[s], kATileBytes + B_BYTES);
    load_a(s, u0 + i);
    load_b(s, u0 + i);
  }
}

// The MMA issuer's work for the stream-K units [u0, u1) of one GEMM.  i_base
// is the pipeline stage index of the first unit and seg the CTA's segment
// count (accumulator buffer and phase); both carry over to a following GEMM
// of the same kernel.  FP8: B is the activation code block of k block kk at
// sB + (kk - kb_lo) * NT * 128, written before the units start.  Returns
// false when a wait gave up.
template <int NT, int STAGES, bool FP8 = false>
__device__ __forceinline__ bool ws_mma_units(uint8_t* sA, uint8_t* sB, uint64_t* full, uint64_t* empty,
                                             uint64_t* accf, uint64_t* acce, uint32_t tmem, const SkSched& sc,
                                             long long u0, long long u1, int* status, volatile int* abort_flag,
                                             int issuer, int kb_lo, long long& i_base, int& seg) {
  // Issuer `issuer` (0 or 1) takes the k blocks j = issuer, issuer + 2, ... of
  // each segment into accumulator (b, issuer); both commit accf[b] (count 2).
  constexpr int B_BYTES = NT * 128;
  constexpr uint32_t IDESC = FP8 ? idesc_e4m3_f32(128, NT) : idesc_bf16_f32(128, NT);
  for (long long u = u0; u < u1; ++seg) {
    const int T = static_cast<int>(u / sc.kb);
    const long long seg_end = (static_cast<long long>(T) + 1) * sc.kb < u1 ? (static_cast<long long>(T) + 1) * sc.kb : u1;
    const int b = seg & 1;
    if (seg >= 2 && !mbar_wait(&acce[b], ((seg >> 1) - 1) & 1, status, abort_flag)) return false;
    tc_fence_after();
    const uint32_t d = tmem + static_cast<uint32_t>((b * 2 + issuer) * NT);
    const long long len = seg_end - u;
    for (long long jj = issuer; jj < len; jj += 2) {
      const long long i = i_base + jj;
      const int s = static_cast<int>(i % STAGES);
      if (!mbar_wait(&full[s], static_cast<uint32_t>((i / STAGES) & 1), status, abort_flag)) return false;
      tc_fence_after();
      const uint32_t a0 = smem_u32(sA + s * kATileBytes);
      const uint32_t b0 = FP8 ? smem_u32(sB + (static_cast<int>((u + jj) % sc.kb) - kb_lo) * B_BYTES)
                              : smem_u32(sB + s * B_BYTES);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (FP8)
          umma_e4m3_ss(d, sdesc_kmajor_sw128(a0 + 32 * k), sdesc_kmajor_sw128(b0 + 32 * k), IDESC,
                       (jj >= 2 || k > 0) ? 1u : 0u);
        else
          umma_bf16_ss(d, sdesc_kmajor_sw128(a0 + 32 * k), sdesc_kmajor_sw128(b0 + 32 * k), IDESC,
                       (jj >= 2 || k > 0) ? 1u : 0u);
      }
      umma_commit(&empty[s]);
    }
    umma_commit(&accf[b]);
    i_base += len;
    u = seg_end;
  }
  return true;
}

template <int NT, int STAGES, bool FP8 = false>
__device__ __forceinline__ void ws_mma(uint8_t* sA, uint8_t* sB, uint64_t* full, uint64_t* empty, uint64_t* accf,
                                       uint64_t* acce, uint32_t tmem, const SkSched& sc, long long u0, long long u1,
                                       int* status, volatile int* abort_flag, int issuer, uint64_t* b_ready = nullptr,
                                       int kb_lo = 0) {
  griddep_wait();
  if (FP8 && !mbar_wait(b_ready, 0, status, abort_flag)) return;
  long long i_base = 0;
  int seg = 0;
  ws_mma_units<NT, STAGES, FP8>(sA, sB, full, empty, accf, acce, tmem, sc, u0, u1, status, abort_flag, issuer, kb_lo,
                                i_base, seg);
}

// The NT accumulator columns of segment buffer b for this thread's lane: the
// first issuer's accumulator plus, when the segment had two or more k blocks,
// the second one's (fixed order).
template <int NT>
__device__ __forceinline__ void ws_load_acc(uint32_t tmem, int b, int quarter, float (&v)[NT], bool two) {
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll
  for (int c = 0; c < NT; c += 16) {
    float tmp[16], tmp2[16];
    tmem_ld16(lane_base + static_cast<uint32_t>(b * 2 * NT + c), tmp);
    if (two) {
      tmem_ld16(lane_base + static_cast<uint32_t>((b * 2 + 1) * NT + c), tmp2);
    } else {
#pragma unroll
      for (int k = 0; k < 16; ++k) tmp2[k] = 0.f;
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) v[c + k] = tmp[k] + tmp2[k];
  }
  tmem_wait_ld();
}

// Columns [c, c+16) of the same sum.
template <int NT>
__device__ __forceinline__ void ws_load_acc16(uint32_t tmem, int b, int quarter, int c, float (&v)[16], bool two) {
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
  float tmp2[16];
  tmem_ld16(lane_base + static_cast<uint32_t>(b * 2 * NT + c), v);
  if (two) {
    tmem_ld16(lane_base + static_cast<uint32_t>((b * 2 + 1) * NT + c), tmp2);
#pragma unroll
    for (int k = 0; k < 16; ++k) v[k] += tmp2[k];
  }
}

__device__ __forceinline__ float bf16_round_f(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

// W8A8 activations [Fast-dVLM technical overview (ocdem.com), section 2.3.2;
// per-token scale a_t = max_k |h_tk| / 448, codes E4M3(h_tk / a_t)]: run by
// the 128 epilogue threads (et = 0..127) of a weight-streaming CTA before its
// first UMMA.  The projection's input h is src (bf16 [NT rows][src_ld]) or,
// with rms != NULL, RMSNorm(src) = rms[t] * src (then a_t = rms[t] * amax /
// 448 and the codes need only src * 448 / amax: the factor cancels).  The
// per-token largest magnitude comes from amax_in ([n_amax][NT], written by
// the producing kernel) or from reading the rows.  Codes of the 128-wide k
// blocks [kb_lo, kb_hi) go to sB (block i at i * NT * 128, rows of 128 bytes,
// 128-byte swizzle); a_t to sAt[t] (0 for rows >= n_rows).  Then one arrival
// on b_ready.
template <int NT>
__device__ void fp8_quantize_activations(int et, const bf16* __restrict__ src, int src_ld, int K, int n_rows,
                                         const float* rms, const float* amax_in, int n_amax, int kb_lo, int kb_hi,
                                         uint8_t* sB, float* sAt, float* sQm, uint64_t* b_ready) {
  constexpr int TPT = 128 / NT;  // threads per token for the row scan
  constexpr int SCAN_UNROLL = 16, CODE_UNROLL = 8;  // independent loads in flight per thread
  if (amax_in) {
    if (et < NT) {
      float m = 0.f;
      for (int p = 0; p < n_amax; ++p) m = fmaxf(m, amax_in[p * NT + et]);
      sQm[et] = m;
    }
  } else {
    // the TPT threads of a token read consecutive 16-byte pieces of its row
    const int t = et / TPT, part = et % TPT;
    const int n16 = K / 8;
    float m = 0.f;
    if (t < n_rows) {
      const uint4* row = reinterpret_cast<const uint4*>(src + static_cast<size_t>(t) * src_ld);
      for (int i0 = part; i0 < n16; i0 += TPT * SCAN_UNROLL) {
        uint4 w[SCAN_UNROLL];
#pragma unroll
        for (int j = 0; j < SCAN_UNROLL; ++j) {
          const int i = i0 + j * TPT;
          w[j] = i < n16 ? row[i] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int j = 0; j < SCAN_UNROLL; ++j) {
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w[j]);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(h[q]);
            m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
          }
        }
      }
    }
#pragma unroll
    for (int o = TPT / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (part == 0) sQm[t] = m;
  }
  named_bar_sync(1, 128);
  if (et < NT) {
    const float m = sQm[et];
    const bool live = et < n_rows && m > 0.f;
    sAt[et] = live ? m / 448.0f * (rms ? rms[et] : 1.0f) : 0.f;
    sQm[et] = live ? 448.0f / m : 0.f;
  }
  named_bar_sync(1, 128);
  const int n_items = (kb_hi - kb_lo) * NT * 8;  // (k block, row, 16-byte chunk)
  for (int i0 = et; i0 < n_items; i0 += 128 * CODE_UNROLL) {
    uint4 w0[CODE_UNROLL], w1[CODE_UNROLL];
#pragma unroll
    for (int j = 0; j < CODE_UNROLL; ++j) {
      const int i = i0 + j * 128;
      const int c = i & 7, t = (i >> 3) % NT, b = i / (8 * NT);
      w0[j] = w1[j] = make_uint4(0u, 0u, 0u, 0u);
      if (i < n_items && sQm[t] != 0.f) {
        const uint4* p = reinterpret_cast<const uint4*>(src + static_cast<size_t>(t) * src_ld + (kb_lo + b) * 128 + c * 16);
        w0[j] = p[0];
        w1[j] = p[1];
      }
    }
#pragma unroll
    for (int j = 0; j < CODE_UNROLL; ++j) {
      const int i = i0 + j * 128;
      if (i >= n_items) continue;
      const int c = i & 7, t = (i >> 3) % NT, b = i / (8 * NT);
      const float q = sQm[t];
      const __nv_bfloat162* h0 = reinterpret_cast<const __nv_bfloat162*>(&w0[j]);
      const __nv_bfloat162* h1 = reinterpret_cast<const __nv_bfloat162*>(&w1[j]);
      uint32_t o[4];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const float2 a = __bfloat1622float2(h0[2 * k]), bb = __bfloat1622float2(h0[2 * k + 1]);
        o[k] = static_cast<uint32_t>(cvt_e4m3x2(a.y * q, a.x * q)) |
               (static_cast<uint32_t>(cvt_e4m3x2(bb.y * q, bb.x * q)) << 16);
        const float2 a2 = __bfloat1622float2(h1[2 * k]), b2 = __bfloat1622float2(h1[2 * k + 1]);
        o[2 + k] = static_cast<uint32_t>(cvt_e4m3x2(a2.y * q, a2.x * q)) |
                   (static_cast<uint32_t>(cvt_e4m3x2(b2.y * q, b2.x * q)) << 16);
      }
      *reinterpret_cast<uint4*>(sB + b * NT * 128 + (t >> 3) * 1024 + (t & 7) * 128 + ((c ^ (t & 7)) << 4)) =
          make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  fence_proxy_async_smem();
  named_bar_sync(1, 128);
  if (et == 0) mbar_arrive(b_ready);
}

}  // namespace dvlm
