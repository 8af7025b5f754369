// Compute-bound prefill: the whole context (vision rows and prompt ids) goes
// through each decoder layer as one set of large-M tcgen05 GEMMs and one
// causal attention launch, instead of 16-row weight-streaming forwards.
//
// A prefill of n context rows is the causal pass that fills the exact KV
// cache the block decode attends to [Fast-dVLM technical overview
// (ocdem.com), section 2.2.1: the cache of vision, prompt and committed
// tokens; section 1.2: decoding continues block by block on that cache].  It
// computes what n/16 chunked causal forwards compute, with the weights read
// once per layer (from HBM, then from L2 by the CTAs sharing a weight tile)
// rather than once per chunk.
//
// GEMM (gemm_tm_kernel): token-major tiles.  The 128 context rows of a tile
// are the UMMA A operand (M = 128), 256 weight rows the B operand (N = 256),
// the fp32 accumulator fills 256 TMEM columns, and the whole k range streams
// through one CTA (4-stage TMA pipeline, 48 KB a stage).  Each epilogue
// thread owns one context row, so the fused epilogues need no cross-thread
// exchange:
//   EPI_QKV    rmsnorm factor, rotate-half RoPE of the two heads of the tile,
//              q rows to the q buffer, K/V rows to the cache (V transposed);
//   EPI_RESID  residual add (bf16 stream) and the row's sum of squares over
//              the tile's 256 features (the next RMSNorm's input);
//   EPI_SWIGLU 128 gate rows over the matching 128 up rows:
//              silu(r*g) * (r*u) -> bf16 activation.
// The same definitions as the decode epilogues (gemm_ws.cu), in the same
// precision: sums in fp32, RoPE angles in fp64, bf16 at the same points.
//
// Attention (attn_prefill_kernel): one CTA per (128 query rows, query head);
// S = Q K^T over 128-key chunks and O += P V accumulate in TMEM, softmax runs
// in fp32 with one thread per query row (causal: row at slot p sees slots
// 0..p, the C2C rule of the same section), online rescaling of O in TMEM,
// P and the value tile in fp16 for the second product as in the decode
// attention.
#include <cuda_fp16.h>

#include "kernels.h"
#include "mainloop.cuh"

namespace dvlm {

namespace {
// ---------------------------------------------------------------- GEMM
constexpr int kTmThreads = 192;        // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int kTmStages = 4;
constexpr int kTmCntStride = 512;      // split-K counters: [0, 512) arrivals per tile, [512, 1024) past the wait
constexpr int kTmA = 128 * 128;        // 128 context rows x 64 k (bf16)
constexpr int kTmB = 256 * 128;        // 256 weight rows x 64 k
constexpr int kTmStage = kTmA + kTmB;
constexpr int kTmBar = kTmStages * kTmStage;
constexpr int kTmSmem = kTmBar + 256 + 1024;
constexpr uint32_t kTmIdesc = idesc_bf16_f32(128, 256);

// ---------------------------------------------------------------- attention
constexpr int kPaThreads = 192;        // warp 0 TMA, warp 1 MMA, warps 2..5 softmax (one row each)
constexpr int kPaKeys = 128;           // keys per chunk
constexpr int kPaAtom = 128 * 128;     // one 128-byte-swizzled 128-row operand atom (16 KB)
constexpr int oPaQ = 0;                              // Q: 2 atoms (d 0..63, 64..127)
constexpr int oPaK = oPaQ + 2 * kPaAtom;             // K: 2 stages x 2 atoms
constexpr int oPaV = oPaK + 4 * kPaAtom;             // V^T: 2 stages x 2 atoms (keys 0..63, 64..127)
constexpr int oPaP = oPaV + 4 * kPaAtom;             // P: 2 atoms
constexpr int oPaBar = oPaP + 2 * kPaAtom;
constexpr int kPaSmem = oPaBar + 256 + 1024;
constexpr uint32_t kPaIdescS = idesc_bf16_f32(128, kPaKeys);
constexpr uint32_t kPaIdescO = idesc_f16_f32(128, 128);
constexpr int kPaTmem = 512;                         // S: 2 x 128 columns, O: 128 columns

__device__ __forceinline__ uint64_t l2_policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Loads columns [c, c+16) of this warp's 32 accumulator lanes.
__device__ __forceinline__ void acc16(uint32_t tmem, int quarter, int c, float (&v)[16]) {
  tmem_ld16(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(c), v);
}

__device__ __forceinline__ void store_bf16x16(bf16* dst, const float (&v)[16]) {
  uint32_t w[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
    w[q] = *reinterpret_cast<const uint32_t*>(&b);
  }
  reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
  reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
}
}  // namespace

// (cos, sin) of the RoPE angle of row tok, frequency j (see launch_rope_table).
__global__ void rope_table_kernel(float2* __restrict__ cs, const TmArgs a) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= a.n_tok * 64) return;
  const int tok = idx >> 6, j = idx & 63;
  const int L0 = a.d_len ? *a.d_len : a.L0;
  const int Bq = a.quad_B;
  const bool cand = Bq > 0 && tok >= Bq;
  const int pos = cand ? L0 + (tok - Bq) / Bq + 1 + (tok - Bq) % Bq : L0 + tok;
  const double inv_freq = exp2(-(2.0 * j / 128.0) * a.log2_rope_base);
  double sn, c;
  sincos(static_cast<double>(pos) * inv_freq, &sn, &c);
  cs[idx] = make_float2(static_cast<float>(c), static_cast<float>(sn));
}

template <int EPI>
__global__ void __launch_bounds__(kTmThreads, 1)
    gemm_tm_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapW,
                   const __grid_constant__ CUtensorMap mapW2, const int kb, const int w_row_base, const TmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kTmBar);
  uint64_t* empty = full + kTmStages;
  uint64_t* accf = empty + kTmStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* sabort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tt = blockIdx.x;  // token tile (fastest: the CTAs of one weight tile run together, sharing it in L2)
  const int T = blockIdx.y;   // weight tile
  const int S = gridDim.z, z = blockIdx.z;
  const int k_lo = z * kb / S, k_hi = (z + 1) * kb / S;
  int* sflag = reinterpret_cast<int*>(tmem_slot + 2);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTmStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    *sabort = 0;
    fence_mbar_init();
    tma_prefetch_map(&mapX);
    tma_prefetch_map(&mapW);
    if (EPI == EPI_SWIGLU) tma_prefetch_map(&mapW2);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_normal();
      for (int i = 0; i < k_hi - k_lo; ++i) {
        const int s = i % kTmStages, kk = k_lo + i;
        if (i >= kTmStages && !mbar_wait(&empty[s], ((i / kTmStages) & 1) ^ 1, a.status, sabort)) break;
        uint8_t* sA = smem + s * kTmStage;
        uint8_t* sB = sA + kTmA;
        mbar_arrive_expect_tx(&full[s], kTmStage);
        tma_load_2d(sA, &mapX, &full[s], kk * 64, tt * 128, pol);
        if (EPI == EPI_SWIGLU) {
          tma_load_2d(sB, &mapW, &full[s], kk * 64, w_row_base + T * 128, pol);
          tma_load_2d(sB + kTmB / 2, &mapW2, &full[s], kk * 64, w_row_base + T * 128, pol);
        } else {
          tma_load_2d(sB, &mapW, &full[s], kk * 64, w_row_base + T * 256, pol);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = true;
      for (int i = 0; i < k_hi - k_lo; ++i) {
        const int s = i % kTmStages;
        if (!mbar_wait(&full[s], (i / kTmStages) & 1, a.status, sabort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + s * kTmStage), b0 = a0 + kTmA;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_bf16_ss(tmem, sdesc_kmajor_sw128(a0 + 32 * k), sdesc_kmajor_sw128(b0 + 32 * k), kTmIdesc,
                       (i > 0 || k > 0) ? 1u : 0u);
        umma_commit(&empty[s]);
      }
      if (ok) umma_commit(accf);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int tok = tt * 128 + row;
    const bool valid = tok < a.n_tok;
    float r = 1.f;
    if (EPI != EPI_RESID && valid) {
      float s2 = 0.f;
      for (int p = 0; p < a.n_ssq; ++p) s2 += a.ssq_in[static_cast<size_t>(p) * a.tok_stride + tok];
      r = 1.0f / sqrtf(s2 * a.inv_h + a.eps);
    }
    bool got = mbar_wait(accf, 0, a.status, sabort);
    __syncwarp();
    if (got) tc_fence_after();
    // Split-K: every CTA stores its fp32 partial tile and counts itself on
    // the tile's counter; once all S have arrived (the S CTAs of a tile are
    // resident together: the grid is at most one CTA per SM), CTA z adds the
    // partials in z order (deterministic) for its 1/S of the tile's epilogue
    // units and runs the epilogue on those sums.  A second counter, of CTAs
    // past the wait, lets the last of them zero both for the next launch.
    const int tile = tt * gridDim.y + T;
    constexpr int kUnits = EPI == EPI_RESID ? 16 : 8;  // 16-column groups (QKV: a head's quarter)
    int u_lo = 0, u_hi = kUnits;
    if (S > 1) {
      if (got) {
        // partial tile as [column group of 4][row] float4: a warp's 32 rows
        // of one group are 512 contiguous bytes (stores and loads coalesce)
        float4* mine = reinterpret_cast<float4*>(a.part + (static_cast<size_t>(tile) * S + z) * 128 * 256) + row;
#pragma unroll 1
        for (int c = 0; c < 256; c += 16) {
          float v[16];
          acc16(tmem, quarter, c, v);
#pragma unroll
          for (int q = 0; q < 16; q += 4) __stcg(mine + ((c + q) >> 2) * 128, make_float4(v[q], v[q + 1], v[q + 2], v[q + 3]));
        }
      }
      __threadfence();
      named_bar_sync(1, 128);
      if (threadIdx.x == 64) {
        atomicAdd(&a.cnt[tile], 1);
        *sflag = wait_counter(&a.cnt[tile], S, a.status, sabort) ? 1 : 0;
        if (atomicAdd(&a.cnt[kTmCntStride + tile], 1) == S - 1) {  // every CTA of the tile is past the wait
          a.cnt[tile] = 0;
          a.cnt[kTmCntStride + tile] = 0;
        }
      }
      named_bar_sync(1, 128);
      got = got && *sflag;
      __threadfence();
      u_lo = z * kUnits / S;
      u_hi = (z + 1) * kUnits / S;
    }
    // Columns [c, c+16) of this thread's row: the accumulator, or the sum of
    // the split partials.
    auto cols = [&](int c, float (&v)[16]) {
      if (S == 1) {
        acc16(tmem, quarter, c, v);
        return;
      }
#pragma unroll
      for (int q = 0; q < 16; ++q) v[q] = 0.f;
      for (int zz = 0; zz < S; ++zz) {
        const float4* src =
            reinterpret_cast<const float4*>(a.part + (static_cast<size_t>(tile) * S + zz) * 128 * 256) + row;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 f = __ldcg(src + ((c >> 2) + q) * 128);
          v[4 * q] += f.x;
          v[4 * q + 1] += f.y;
          v[4 * q + 2] += f.z;
          v[4 * q + 3] += f.w;
        }
      }
    };
    if (got) {
      if (EPI == EPI_RESID) {
        bf16* x = a.resid + static_cast<size_t>(tok) * a.resid_ld + T * 256;
        float sq = 0.f;
#pragma unroll 1
        for (int u = u_lo; u < u_hi; ++u) {
          const int c = u * 16;
          float v[16];
          cols(c, v);  // TMEM loads are warp-collective: every lane loads
          if (valid) {
            const uint4 xa = reinterpret_cast<const uint4*>(x + c)[0];
            const uint4 xb = reinterpret_cast<const uint4*>(x + c)[1];
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&xa);
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&xb);
            float o[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float2 f = __bfloat1622float2(h[q]), g = __bfloat1622float2(h2[q]);
              o[2 * q] = bf16_round_f(f.x + v[2 * q]);
              o[2 * q + 1] = bf16_round_f(f.y + v[2 * q + 1]);
              o[8 + 2 * q] = bf16_round_f(g.x + v[8 + 2 * q]);
              o[8 + 2 * q + 1] = bf16_round_f(g.y + v[8 + 2 * q + 1]);
            }
#pragma unroll
            for (int k = 0; k < 16; ++k) sq += o[k] * o[k];
            store_bf16x16(x + c, o);
          }
        }
        // sum of squares over this CTA's columns of the tile: entry T * S + z
        if (valid) a.ssq_out[(static_cast<size_t>(T) * S + z) * a.tok_stride + tok] = sq;
      } else if (EPI == EPI_SWIGLU) {
        bf16* out = a.out + static_cast<size_t>(tok) * a.out_ld + T * 128;
#pragma unroll 1
        for (int uu = u_lo; uu < u_hi; ++uu) {
          const int c = uu * 16;
          float g[16], u[16];
          cols(c, g);
          cols(128 + c, u);
          float o[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float gg = g[k] * r;
            o[k] = gg / (1.0f + expf(-gg)) * (u[k] * r);
          }
          if (valid) store_bf16x16(out + c, o);
        }
      } else {  // EPI_QKV: the tile holds heads 2T and 2T+1 of the [q | k | v] rows
        const int nq = a.n_q_heads, nkv = a.n_kv_heads;
        const int L0 = a.d_len ? *a.d_len : a.L0;
        // candidate rows of a fused draft+verify forward: block ci, row cr
        const int Bq = a.quad_B;
        const bool cand = Bq > 0 && tok >= Bq;
        const int ci = cand ? (tok - Bq) / Bq : 0, cr = cand ? (tok - Bq) % Bq : 0;
        const int pos = cand ? L0 + ci + 1 + cr : L0 + tok;
        const int side_n = a.side_n;  // keys per KV head in the side buffers
#pragma unroll 1
        for (int uu = u_lo; uu < u_hi; ++uu) {  // unit uu: quarter sub of head i of the tile
          const int i = uu >> 2, sub = uu & 3;
          const int hh = 2 * T + i;
          if (hh < nq + nkv) {
            bf16* dst = hh < nq ? a.out + static_cast<size_t>(tok) * a.out_ld + hh * 128
                        : cand ? a.kside + (static_cast<size_t>(hh - nq) * side_n + ci * 64 + cr) * 128
                               : a.kcache + (static_cast<size_t>(hh - nq) * a.Lmax + pos) * 128;
#pragma unroll 1
            for (int j0 = sub * 16; j0 < sub * 16 + 16; j0 += 16) {
              float x1[16], x2[16], y1[16], y2[16];
              cols(i * 128 + j0, x1);
              cols(i * 128 + 64 + j0, x2);
              const float4* cs4 = reinterpret_cast<const float4*>(a.rope_cs + static_cast<size_t>(valid ? tok : 0) * 64 + j0);
              float2 csj[16];
#pragma unroll
              for (int k = 0; k < 16; k += 2) {
                const float4 f = __ldg(cs4 + k / 2);
                csj[k] = make_float2(f.x, f.y);
                csj[k + 1] = make_float2(f.z, f.w);
              }
#pragma unroll
              for (int k = 0; k < 16; ++k) {
                const float c = csj[k].x, s = csj[k].y;
                const float u1 = x1[k] * r, u2 = x2[k] * r;
                y1[k] = u1 * c - u2 * s;
                y2[k] = u2 * c + u1 * s;
              }
              if (valid) {
                store_bf16x16(dst + j0, y1);
                store_bf16x16(dst + 64 + j0, y2);
              }
            }
          } else {
            const int h = hh - nq - nkv;
#pragma unroll 1
            for (int c = sub * 32; c < sub * 32 + 32; c += 16) {
              float v[16];
              cols(i * 128 + c, v);
              if (valid) {
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                  const bf16 vb = __float2bfloat16_rn(v[k] * r);
                  if (cand)
                    a.vside[(static_cast<size_t>(h) * 128 + c + k) * side_n + ci * 64 + cr] = vb;
                  else
                    a.vcache[(static_cast<size_t>(h) * 128 + c + k) * a.Lmax + pos] = vb;
                }
              }
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// Causal attention of n_tok prefill rows (slots L0..L0+n_tok-1, their K/V
// already in the cache) over the cache slots 0..L0+n_tok-1: one CTA per 128
// rows of one query head.
__global__ void __launch_bounds__(kPaThreads, 1)
    attn_tile_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                     const __grid_constant__ CUtensorMap mapV, const PrefillAttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem + oPaQ;
  uint8_t* sK = smem + oPaK;
  uint8_t* sV = smem + oPaV;
  uint8_t* sP = smem + oPaP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + oPaBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2] PV of the chunk in that stage done
  uint64_t* s_full = bars + 5;    // [2]
  uint64_t* s_empty = bars + 7;   // [2] the softmax warps have read S of that buffer
  uint64_t* p_full = bars + 9;    // P of the current chunk written, O rescaled (one phase per chunk)
  uint64_t* pv_done = bars + 10;  // PV of a chunk done (one phase per chunk)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);
  volatile int* sabort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x;                              // query tile
  const int h = blockIdx.y;                               // query head
  const int g = h / (a.Hq / a.Hkv);                       // KV head
  const int Ltot = a.L0 + a.n_tok;
  const int q_last = min(a.L0 + qt * 128 + 127, Ltot - 1);  // last query slot of a prefill tile
  const int nc = q_last / kPaKeys + 1;
  const int kv_row0 = a.kv_base * a.Hkv + g;  // (layer, KV head) entry of the cache

  if (threadIdx.x == 0) {
    for (int i = 0; i < 11; ++i) mbar_init(&bars[i], (i == 7 || i == 8 || i == 9) ? 4 : 1);
    *sabort = 0;
    fence_mbar_init();
    tma_prefetch_map(&mapQ);
    tma_prefetch_map(&mapK);
    tma_prefetch_map(&mapV);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kPaTmem);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_last();
      mbar_arrive_expect_tx(q_full, 2 * kPaAtom);
      for (int d = 0; d < 2; ++d) tma_load_2d(sQ + d * kPaAtom, &mapQ, q_full, h * 128 + d * 64, qt * 128, pol);
      for (int c = 0; c < nc; ++c) {
        const int st = c & 1;
        if (c >= 2 && !mbar_wait(&kv_empty[st], ((c >> 1) - 1) & 1, a.status, sabort)) break;
        mbar_arrive_expect_tx(&kv_full[st], 4 * kPaAtom);
        const int key0 = c * kPaKeys;
        for (int d = 0; d < 2; ++d)
          tma_load_2d(sK + (2 * st + d) * kPaAtom, &mapK, &kv_full[st], d * 64, kv_row0 * a.Lmax + key0, pol);
        for (int k = 0; k < 2; ++k)
          tma_load_2d(sV + (2 * st + k) * kPaAtom, &mapV, &kv_full[st], key0 + k * 64, kv_row0 * 128, pol);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, a.status, sabort);
      auto issue_pv = [&](int c) -> bool {
        if (!mbar_wait(p_full, c & 1, a.status, sabort)) return false;
        tc_fence_after();
        const uint32_t pa = smem_u32(sP), vb = smem_u32(sV + 2 * (c & 1) * kPaAtom);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kPaAtom + (kk & 3) * 32;
          umma_bf16_ss(tmem + 256, sdesc_kmajor_sw128(pa + off), sdesc_kmajor_sw128(vb + off), kPaIdescO,
                       (c > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&kv_empty[c & 1]);
        umma_commit(pv_done);
        return true;
      };
      // Issue whichever product is ready (PV of the oldest chunk with its P
      // written first: that frees its K/V stage for the load two chunks
      // ahead), so consecutive loads overlap instead of queueing behind S.
      int cs = 0, cp = 0;
      long long t0 = clock64();
      while (ok && cp < nc) {
        if (cp < cs && mbar_test_wait(p_full, cp & 1)) {
          ok = issue_pv(cp);
          ++cp;
          t0 = clock64();
          continue;
        }
        if (cs < nc && cs <= cp + 1) {
          const int st = cs & 1;
          if (mbar_test_wait(&kv_full[st], (cs >> 1) & 1) &&
              (cs < 2 || mbar_test_wait(&s_empty[st], ((cs >> 1) - 1) & 1))) {
            tc_fence_after();
            const uint32_t qa = smem_u32(sQ), kb = smem_u32(sK + 2 * st * kPaAtom);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t off = (kk >> 2) * kPaAtom + (kk & 3) * 32;
              umma_bf16_ss(tmem + st * kPaKeys, sdesc_kmajor_sw128(qa + off), sdesc_kmajor_sw128(kb + off),
                           kPaIdescS, kk > 0 ? 1u : 0u);
            }
            umma_commit(&s_full[st]);
            ++cs;
            t0 = clock64();
            continue;
          }
        }
        if (*sabort || clock64() - t0 > kWaitBudgetCycles) {
          record_error(a.status, DVLM_ERR_TIMEOUT);
          *sabort = 1;
          ok = false;
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int tok = qt * 128 + row;
    const bool valid = tok < a.n_tok;
    const int qslot = valid ? a.L0 + tok : Ltot - 1;  // prefill rows past the end: finite, never written
    // key j of chunk c is visible to this row
    auto visible = [&](int c, int j) -> bool {
      return c * kPaKeys + j <= qslot;
    };
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int c = 0; c < nc; ++c) {
      const int st = c & 1;
      const int key0 = c * kPaKeys;
      if (!mbar_wait(&s_full[st], (c >> 1) & 1, a.status, sabort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // pass 1: row maximum; pass 2: probabilities (scores re-read from TMEM)
      float mx = -INFINITY;
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {
        float sc[64];
        tmem_ld64(tmem + lane_off + static_cast<uint32_t>(st * kPaKeys + hf * 64), sc);
#pragma unroll
        for (int k = 0; k < 64; ++k)
          if (visible(c, hf * 64 + k)) mx = fmaxf(mx, sc[k] * a.scale_log2);
      }
      const float m_new = fmaxf(m, mx);
      const float alpha = (m == -INFINITY) ? (m_new == -INFINITY ? 1.f : 0.f) : exp2f(m - m_new);
      uint32_t packed[64];
      float psum = 0.f;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float sc[64];
        tmem_ld64(tmem + lane_off + static_cast<uint32_t>(st * kPaKeys + hf * 64), sc);
#pragma unroll
        for (int k = 0; k < 64; k += 2) {
          const bool v0 = visible(c, hf * 64 + k), v1 = visible(c, hf * 64 + k + 1);
          const float p0 = v0 ? ex2_approx(sc[k] * a.scale_log2 - m_new) : 0.f;
          const float p1 = v1 ? ex2_approx(sc[k + 1] * a.scale_log2 - m_new) : 0.f;
          psum += p0 + p1;
          const __half2 ph = __floats2half2_rn(p0, p1);
          packed[hf * 32 + k / 2] = *reinterpret_cast<const uint32_t*>(&ph);
        }
      }
      // S of this buffer is consumed
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[st]);
      // the previous chunk's PV is complete: O is stable and P is free
      if (c > 0) {
        if (!mbar_wait(pv_done, (c - 1) & 1, a.status, sabort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll 1
          for (int cc = 0; cc < 128; cc += 64) {
            float o[64];
            tmem_ld64(tmem + lane_off + 256u + cc, o);
#pragma unroll
            for (int k = 0; k < 64; ++k) o[k] *= alpha;
#pragma unroll
            for (int k = 0; k < 64; k += 16) tmem_st16_nowait(tmem + lane_off + 256u + cc + k, o + k);
            tmem_wait_st();
          }
        }
      }
      // P row (fp16) into the two 64-key atoms, 128-byte swizzle
#pragma unroll
      for (int at = 0; at < 2; ++at) {
        uint8_t* prow = sP + at * kPaAtom + row * 128;
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
          *reinterpret_cast<uint4*>(prow + ((cc ^ (row & 7)) << 4)) =
              make_uint4(packed[at * 32 + cc * 4], packed[at * 32 + cc * 4 + 1], packed[at * 32 + cc * 4 + 2],
                         packed[at * 32 + cc * 4 + 3]);
      }
      // value row `row` (feature d = row) of this chunk to fp16 in place;
      // keys past the cache's valid slots were zero-filled by the load
      // (prefill) or are zeroed here (candidate blocks: stale or poisoned
      // slots past L+i, padding of the side chunk)
      {
        const int n_valid = kPaKeys;
        if (!mbar_wait(&kv_full[st], (c >> 1) & 1, a.status, sabort)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int at = 0; at < 2; ++at) {
          uint8_t* vrow = sV + (2 * st + at) * kPaAtom + row * 128;
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            uint4* p16 = reinterpret_cast<uint4*>(vrow + ((cc ^ (row & 7)) << 4));
            uint4 w = *p16;
            uint32_t* wv = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[e]));
              // keys 8 cc + 2e, +1 sit in 16-byte chunk cc ^ (row & 7) of this 128-byte row
              const int kk = at * 64 + (cc << 3) + 2 * e;
              const __half2 hh = __floats2half2_rn(kk < n_valid ? f.x : 0.f, kk + 1 < n_valid ? f.y : 0.f);
              wv[e] = *reinterpret_cast<const uint32_t*>(&hh);
            }
            *p16 = w;
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      l = l * alpha + psum;
      m = m_new;
    }
    if (ok && mbar_wait(pv_done, (nc - 1) & 1, a.status, sabort)) {
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.0f / l : 0.f;
      bf16* dst = a.out + static_cast<size_t>(tok) * a.out_ld + h * 128;
#pragma unroll 1
      for (int cc = 0; cc < 128; cc += 64) {
        float o[64];
        tmem_ld64(tmem + lane_off + 256u + cc, o);
        if (valid) {
#pragma unroll
          for (int k = 0; k < 64; k += 16) {
            float v[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) v[q] = o[k + q] * inv_l;
            store_bf16x16(dst + cc + k, v);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kPaTmem);
  }
}

template <int EPI>
static cudaError_t tm_launch(const CUtensorMap& mapX, const CUtensorMap& mapW, const CUtensorMap& mapW2, int kb,
                             int w_row_base, int n_wtiles, const TmArgs& a, cudaStream_t s) {
  auto kern = gemm_tm_kernel<EPI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kTmSmem);
  if (e != cudaSuccess) return e;
  const int n_tt = (a.n_tok + 127) / 128;
  const int S = a.splits > 1 ? a.splits : 1;
  if (S > 1 && (!a.part || !a.cnt || S > kb)) return cudaErrorInvalidValue;
  // split-K: the S CTAs of a tile wait for one another, so the whole grid
  // must be resident (one CTA per SM); S <= the tile's epilogue units
  if (S > 1 && (n_tt * n_wtiles > kTmCntStride || n_tt * n_wtiles * S > device_sm_count() ||
                S > (EPI == EPI_RESID ? 16 : 8)))
    return cudaErrorInvalidValue;
  kern<<<dim3(n_tt, n_wtiles, S), kTmThreads, kTmSmem, s>>>(mapX, mapW, mapW2, kb, w_row_base, a);
  return cudaGetLastError();
}

cudaError_t launch_rope_table(float2* cs, const TmArgs& a, cudaStream_t s) {
  if (!cs || a.n_tok < 1) return cudaErrorInvalidValue;
  rope_table_kernel<<<(a.n_tok * 64 + 255) / 256, 256, 0, s>>>(cs, a);
  return cudaGetLastError();
}

cudaError_t launch_gemm_tm(const CUtensorMap& mapX, const CUtensorMap& mapW, const CUtensorMap& mapW2, int kb,
                           int w_row_base, int n_wtiles, const TmArgs& a, cudaStream_t s) {
  if (a.n_tok < 1 || kb < 1 || n_wtiles < 1) return cudaErrorInvalidValue;
  if (a.epi == EPI_QKV && !a.rope_cs) return cudaErrorInvalidValue;
  if (a.quad_B > 0 && (a.side_n < 64 * a.quad_B || !a.kside || !a.vside)) return cudaErrorInvalidValue;
  switch (a.epi) {
    case EPI_QKV: return tm_launch<EPI_QKV>(mapX, mapW, mapW2, kb, w_row_base, n_wtiles, a, s);
    case EPI_RESID: return tm_launch<EPI_RESID>(mapX, mapW, mapW2, kb, w_row_base, n_wtiles, a, s);
    case EPI_SWIGLU: return tm_launch<EPI_SWIGLU>(mapX, mapW, mapW2, kb, w_row_base, n_wtiles, a, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_prefill(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                                const PrefillAttnArgs& a, cudaStream_t s) {
  if (a.n_tok < 1 || a.Hq % a.Hkv) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(attn_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPaSmem);
  if (e != cudaSuccess) return e;
  attn_tile_kernel<<<dim3((a.n_tok + 127) / 128, a.Hq), kPaThreads, kPaSmem, s>>>(mapQ, mapK, mapV, a);
  return cudaGetLastError();
}


}  // namespace dvlm
