// Dense prefill: the prompt's tokens go through each layer together, so the
// int4 projections become matrix products (T tokens x K) . W~^T and run on the
// tcgen05 tensor cores; attention over the prompt is causal (with the sliding
// window on the SWA layers) and runs as a flash-attention kernel.
//
// Per layer (ATLAS-OLMo-3-32B-Think-v4 model card, "Architecture deep-dive";
// "Limitations & roadmap": batched / tiled prefill, GEMV -> GEMM):
//   Y  = X16 . Wqkv~^T                     (GEMM, fp32 out)
//   q, k <- RMSNorm over the whole projection, gains, RoPE / YaRN; K, V -> cache
//   O  = causal GQA attention              (fp16 out)
//   A  = O . Wo~^T;   X += RMSNorm(A) g_pa (fp32 residual), X16 = fp16(X)
//   H  = silu(G) * U, [G; U] = X16 . Wgu~^T (GEMM with the SwiGLU epilogue)
//   F  = H . Wd~^T;   X += RMSNorm(F) g_pf
//
// The int4 weights are expanded, one matrix at a time, to fp16 (q - z) * s
// rounded to nearest (the product of a 4-bit code and an fp16 scale needs up
// to 15 significant bits; fp16 keeps 11) in the rows' tiled order, so the
// gate / up rows alternate and the GEMM epilogue finds each pair side by
// side.  Activations are fp16 with a per-token power-of-two scale that keeps
// every row's magnitude below 2^15 (undone in the GEMM epilogue).
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ptx.cuh"
#include "tc.cuh"
#include "w4a_internal.h"

namespace w4a {

constexpr long long PF_WAIT = 4000000000LL;  // bound on any single wait (~2 s)

__device__ __forceinline__ void pf_error(uint32_t* err, uint32_t bits) {
  if (err) atomicOr(err, bits);
}
__device__ __forceinline__ uint16_t f16_checked(float v, uint32_t* err) {
  const uint16_t h = f32_to_f16(v);
  if ((h & 0x7c00u) == 0x7c00u) pf_error(err, EW_RANGE);
  return h;
}

// ---------------------------------------------------------------------------
// int4 tiled units -> fp16 [n, k] (tiled row order)
// ---------------------------------------------------------------------------
// One unit per warp: lane (g, t) holds, for every k-step s of the unit, the
// code word of rows g and g + 8 at columns 32 (s / 2) + 8 t + 4 (s % 2) ..
// + 3 (eight nibbles: row g + 8 when the nibble index is odd, column offset
// 2 [j & 2] + [j & 4]); its words are eight (four) 16-byte loads, coalesced
// across the warp.  Both formats: asymmetric group 128 (16 x 512 units, fp16
// scales, int4 zeros) and the symmetric group-32 checkpoint (16 x 256 units,
// bf16 scales, zero 8).  Streaming loads and stores: the int4 units are read
// once and the fp16 rows are read back by a later GEMM, not from L2.
__device__ __forceinline__ void dq_pair(uint32_t w0, uint32_t w1, float s_lo, float s_hi, int z_lo, int z_hi,
                                        uint16_t* __restrict__ dst, int64_t k) {
  uint16_t lo[8], hi[8];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const uint32_t w = e ? w1 : w0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int q = int((w >> (4 * j)) & 15u);
      const int c = 4 * e + ((j & 2) ? 2 : 0) + ((j & 4) ? 1 : 0);
      if (j & 1)
        hi[c] = f32_to_f16(float(q - z_hi) * s_hi);
      else
        lo[c] = f32_to_f16(float(q - z_lo) * s_lo);
    }
  }
  uint4 a, b;
  a.x = uint32_t(lo[0]) | (uint32_t(lo[1]) << 16);
  a.y = uint32_t(lo[2]) | (uint32_t(lo[3]) << 16);
  a.z = uint32_t(lo[4]) | (uint32_t(lo[5]) << 16);
  a.w = uint32_t(lo[6]) | (uint32_t(lo[7]) << 16);
  b.x = uint32_t(hi[0]) | (uint32_t(hi[1]) << 16);
  b.y = uint32_t(hi[2]) | (uint32_t(hi[3]) << 16);
  b.z = uint32_t(hi[4]) | (uint32_t(hi[5]) << 16);
  b.w = uint32_t(hi[6]) | (uint32_t(hi[7]) << 16);
  __stcs(reinterpret_cast<uint4*>(dst), a);
  __stcs(reinterpret_cast<uint4*>(dst + 8 * k), b);
}
__device__ __forceinline__ uint32_t u4c(const uint4& v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }

__device__ __forceinline__ void dq_unit(const uint8_t* __restrict__ tiled, int64_t k, int fmt, int unit, int lane,
                                        uint16_t* __restrict__ out) {
  const int g = lane >> 2, t = lane & 3;
  if (fmt == FMT_SYM32) {
    const int nkc = int(k / S32_KC), rb = unit / nkc, kc = unit - rb * nkc;
    const uint8_t* u = tiled + (size_t)unit * S32_UNIT;
    uint4 wv[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) wv[q] = __ldcs(reinterpret_cast<const uint4*>(u) + q * 32 + lane);
    const uint4 sa = __ldcs(reinterpret_cast<const uint4*>(u + 2048) + 2 * g);
    const uint4 sb = __ldcs(reinterpret_cast<const uint4*>(u + 2048) + 2 * g + 1);
    uint16_t* row = out + ((size_t)rb * RB + g) * k + (size_t)kc * S32_KC + 8 * t;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      // scales of group m: bf16 (row g, row g + 8) in word m of the row's 32 bytes
      const uint32_t sw = m < 4 ? u4c(sa, m) : u4c(sb, m - 4);
      dq_pair(u4c(wv[m >> 1], (2 * m) & 3), u4c(wv[m >> 1], (2 * m + 1) & 3), bf16_to_f32(uint16_t(sw & 0xffffu)),
              bf16_to_f32(uint16_t(sw >> 16)), 8, 8, row + 32 * m, k);
    }
  } else {
    const int nkc = int(k / W4_KC), rb = unit / nkc, kc = unit - rb * nkc;
    const uint8_t* u = tiled + (size_t)unit * W4_UNIT;
    uint4 wv[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) wv[q] = __ldcs(reinterpret_cast<const uint4*>(u) + q * 32 + lane);
    const uint4 sc = __ldcs(reinterpret_cast<const uint4*>(u + 4096) + g);  // fp16 (row g, row g + 8) per group
    const uint4 z0 = __ldcs(reinterpret_cast<const uint4*>(u + 4224));       // zero words: group, row half
    const uint4 z1 = __ldcs(reinterpret_cast<const uint4*>(u + 4224) + 1);
    uint16_t* row = out + ((size_t)rb * RB + g) * k + (size_t)kc * W4_KC + 8 * t;
#pragma unroll
    for (int grp = 0; grp < 4; ++grp) {
      const uint32_t sw = u4c(sc, grp);
      const float s_lo = half_bits_to_f32(uint16_t(sw & 0xffffu)), s_hi = half_bits_to_f32(uint16_t(sw >> 16));
      const uint32_t zl = grp < 2 ? u4c(z0, 2 * grp) : u4c(z1, 2 * grp - 4);
      const uint32_t zh = grp < 2 ? u4c(z0, 2 * grp + 1) : u4c(z1, 2 * grp - 3);
      const int z_lo = int((zl >> (4 * g)) & 15u), z_hi = int((zh >> (4 * g)) & 15u);
#pragma unroll
      for (int mm = 0; mm < 4; ++mm) {
        const int m = 4 * grp + mm;
        dq_pair(u4c(wv[m >> 1], (2 * m) & 3), u4c(wv[m >> 1], (2 * m + 1) & 3), s_lo, s_hi, z_lo, z_hi,
                row + 32 * m, k);
      }
    }
  }
}

// Units of a matrix.
__host__ __device__ __forceinline__ int dequant_units(int64_t n, int64_t k, int fmt) {
  return int((n / RB) * (k / (fmt == FMT_SYM32 ? S32_KC : W4_KC)));
}
__global__ void __launch_bounds__(256) dequant_f16_kernel(const uint8_t* __restrict__ tiled, int64_t n, int64_t k,
                                                          int fmt, uint16_t* __restrict__ out) {
  const int unit = int(blockIdx.x) * 8 + int(threadIdx.x >> 5);
  if (unit < dequant_units(n, k, fmt)) dq_unit(tiled, k, fmt, unit, threadIdx.x & 31, out);
}

// ---------------------------------------------------------------------------
// GEMM on the tcgen05 tensor cores: D[M, N] = A[M, K] . B[N, K]^T, fp16 in,
// fp32 accumulation in tensor memory
// ---------------------------------------------------------------------------
// Persistent: one CTA per SM walks output tiles of 128 x BN (groups of 16
// M-blocks, M-block-fastest, so the CTAs running together share the A and B
// panels in L2).  Warp 0 (one thread) issues the TMA loads of a ring of 64-column K
// slices, warp 1 (one thread) issues the MMAs (four of K = 16 per slice) and
// owns 2 BN tensor-memory columns (two accumulators, so the epilogue of a
// tile overlaps the MMAs of the next), warps 2..5 read an accumulator back
// (each its own 32 TMEM lanes = 32 rows) and write it, and warps 6..13 expand
// later matrices of the sequence from int4 to fp16 meanwhile.
constexpr int GM_BM = 128, GM_BK = 64;
constexpr double GM_NARROW_COST = 0.77;  // time of a 128-wide tile / a 256-wide one (measured)
constexpr double GM_SPLIT_COST = 1.1;    // time of a half-K tile / half a whole one (the reduction)
constexpr int GM_GROUP = 16;             // M-blocks per group of the tile order
constexpr int GM_A_BYTES = GM_BM * GM_BK * 2;
constexpr int GM_EXP = 256;  // threads expanding later matrices (warps 6 ..)
constexpr int GM_THREADS = 192 + GM_EXP;
// Tile widths: 256 columns (4 stages), or 128 (6 stages) where the wider
// tile would leave too much of the last wave of tiles idle.
template <int BN>
struct GmTile {
  static constexpr int ST = BN == 256 ? 4 : 6;
  static constexpr int B_BYTES = BN * GM_BK * 2;
  static constexpr int STAGE_BYTES = GM_A_BYTES + B_BYTES;
  static constexpr int SMEM = ST * STAGE_BYTES + 256 + 1024;  // ring, barriers, alignment slack
  static constexpr int TMEM_COLS = 2 * BN;                    // two accumulators
  static constexpr uint32_t IDESC = umma_idesc_f16(GM_BM, BN, false);
};
static_assert(GmTile<256>::SMEM <= 232448 && GmTile<128>::SMEM <= 232448, "GEMM shared memory");

enum GemmEpi : int { GE_F32 = 0, GE_SILU = 1 };

struct GemmArgs {
  int M, N, K;
  int epi;               // GE_F32: out fp32 [M, ldo]; GE_SILU: out fp16 [M, ldo], ldo >= N / 2
  int ldo;
  void* out;
  const float* row_scale;  // [M] or null: row m of the product is multiplied by it
  uint32_t* err;           // error word
  int ksplit;              // 1, or 2 (GE_F32 only): halves of K added into a zeroed out
  // matrices to expand to fp16 while this product runs (their int4 units,
  // shapes, fp16 destinations; nx_count of them, 0 .. 3)
  int nx_count, nx_fmt;
  const uint8_t* nx_blob[3];
  int64_t nx_n[3], nx_k[3];
  uint16_t* nx_out[3];
};

// Bounded wait on an mbarrier phase; gives up (setting the CTA's abort flag
// and the error word) after ~2 s or when another role has given up.
__device__ __forceinline__ bool gm_wait(uint64_t* bar, uint32_t par, volatile int* abort_flag, uint32_t* err) {
  if (mbar_try_wait(bar, par)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, par)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > PF_WAIT) {
      *abort_flag = 1;
      pf_error(err, EW_MBAR_TIMEOUT);
      return false;
    }
  }
  return true;
}

template <int BN>
__global__ void __launch_bounds__(GM_THREADS, 1)
    gemm_f16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const GemmArgs g) {
  using TL = GmTile<BN>;
  constexpr int GM_ST = TL::ST, GM_BN = BN, GM_B_BYTES = TL::B_BYTES, GM_STAGE_BYTES = TL::STAGE_BYTES;
  extern __shared__ uint8_t gm_raw[];
  // the ring at a 1,024-byte aligned shared address (the 128-byte swizzle's atom)
  uint8_t* sm = gm_raw + ((1024u - (smem_addr(gm_raw) & 1023u)) & 1023u);
  uint8_t* sA = sm;
  uint8_t* sB = sm + GM_ST * GM_A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + GM_ST * GM_STAGE_BYTES);
  uint64_t* empty = full + GM_ST;
  uint64_t* tfull = empty + GM_ST;   // accumulator b holds a finished tile
  uint64_t* tempty = tfull + 2;      // accumulator b has been read back
  uint64_t* done = tempty + 2;       // every MMA of this CTA has completed
  uint32_t* tbase = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tbase + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = (g.M + GM_BM - 1) / GM_BM, nt = (g.N + GM_BN - 1) / GM_BN;
  const int ntiles = mt * nt * g.ksplit, nkb = g.K / GM_BK;
  // tile t: K part t / (mt nt); within a part, groups of GM_GROUP M-blocks
  // walk their N-blocks M-block-fastest, so the ~148 tiles in flight cover a
  // block of about 16 x 9 tiles and read about half the operand bytes of a
  // whole column of M-blocks
  auto tile_mn = [&](int t, int& mb, int& nb) {
    const int r = t % (mt * nt);
    const int grp = r / (GM_GROUP * nt), first = grp * GM_GROUP;
    const int gm = min(GM_GROUP, mt - first);
    const int rr = r - first * nt;
    mb = first + rr % gm;
    nb = rr / gm;
  };
  auto krange = [&](int t, int& kb0, int& kb1) {
    const int ks = t / (mt * nt);
    kb0 = ks * nkb / g.ksplit;
    kb1 = (ks + 1) * nkb / g.ksplit;
  };

  if (threadIdx.x == 0) {
#pragma unroll 1
    for (int s = 0; s < GM_ST; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    mbar_init(tfull + 0, 1);
    mbar_init(tfull + 1, 1);
    mbar_init(tempty + 0, 4);
    mbar_init(tempty + 1, 4);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&tmA);
    tma_prefetch_map(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tbase, TL::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;

  if (warp == 0) {
    if (lane == 0) {
      // ---- producer: TMA loads into the ring ----
      uint32_t it = 0;
      bool ok = true;
#pragma unroll 1
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        int mb, nb, kb0, kb1;
        tile_mn(t, mb, nb);
        krange(t, kb0, kb1);
#pragma unroll 1
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = int(it % GM_ST);
          if (it >= GM_ST && !gm_wait(empty + s, ((it / GM_ST) & 1u) ^ 1u, abort_flag, g.err)) {
            ok = false;
            break;
          }
          mbar_expect_tx(full + s, GM_STAGE_BYTES);
          tma_load_2d(sA + s * GM_A_BYTES, &tmA, kb * GM_BK, mb * GM_BM, full + s);
          tma_load_2d(sB + s * GM_B_BYTES, &tmB, kb * GM_BK, nb * GM_BN, full + s);
        }
      }
      // the loads in flight land before the CTA may exit
      const uint32_t first = it > uint32_t(GM_ST) ? it - GM_ST : 0u;
#pragma unroll 1
      for (uint32_t j = first; j < it; ++j) {
        const long long t0 = clock64();
        while (!mbar_try_wait(full + (j % GM_ST), (j / GM_ST) & 1u)) {
          if (clock64() - t0 > PF_WAIT) {
            pf_error(g.err, EW_DRAIN_TIMEOUT);
            break;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer ----
      uint32_t it = 0;
      int local = 0;
      bool ok = true;
#pragma unroll 1
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++local) {
        const int buf = local & 1;
        const uint32_t use = uint32_t(local >> 1);
        if (local >= 2 && !gm_wait(tempty + buf, (use - 1u) & 1u, abort_flag, g.err)) break;
        tc_fence_after();
        const uint32_t d = tmem + uint32_t(buf * GM_BN);
        int kb0, kb1;
        krange(t, kb0, kb1);
#pragma unroll 1
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = int(it % GM_ST);
          if (!gm_wait(full + s, (it / GM_ST) & 1u, abort_flag, g.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < GM_BK / 16; ++k) {
            const uint64_t ad = umma_desc_sw128(sA + s * GM_A_BYTES, uint32_t(k * 32));
            const uint64_t bd = umma_desc_sw128(sB + s * GM_B_BYTES, uint32_t(k * 32));
            umma_f16(d, ad, bd, TL::IDESC, (kb != kb0 || k != 0) ? 1u : 0u);
          }
          umma_commit(empty + s);
        }
        if (ok) umma_commit(tfull + buf);
      }
      // every MMA issued has completed before the tensor memory is freed
      umma_commit(done);
      const long long t0 = clock64();
      while (!mbar_try_wait(done, 0u)) {
        if (clock64() - t0 > PF_WAIT) {
          pf_error(g.err, EW_DRAIN_TIMEOUT);
          break;
        }
      }
    }
  } else if (warp >= 6) {
    // ---- warps 6..13: later matrices' fp16 expansion, this CTA's share ----
    // (HBM-bound work under the tensor-bound product; the GEMMs that read
    // them run later on the same stream).  One unit per warp at a time.
    const int ew = int(blockIdx.x) * (GM_EXP / 32) + (warp - 6), nw = int(gridDim.x) * (GM_EXP / 32);
#pragma unroll 1
    for (int mi = 0; mi < g.nx_count; ++mi) {
      const int units = dequant_units(g.nx_n[mi], g.nx_k[mi], g.nx_fmt);
#pragma unroll 1
      for (int unit = ew; unit < units; unit += nw) dq_unit(g.nx_blob[mi], g.nx_k[mi], g.nx_fmt, unit, lane, g.nx_out[mi]);
    }
  } else {
    // ---- epilogue: warps 2..5, TMEM lanes 32 (warp % 4) .. + 31 ----
    const int q = warp & 3;
    int local = 0;
#pragma unroll 1
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++local) {
      int mb, nb;
      tile_mn(t, mb, nb);
      const int buf = local & 1;
      const uint32_t use = uint32_t(local >> 1);
      if (!gm_wait(tfull + buf, use & 1u, abort_flag, g.err)) break;
      tc_fence_after();
      const int row = mb * GM_BM + q * 32 + lane;
      const bool live = row < g.M;
      const float rs = (live && g.row_scale != nullptr) ? g.row_scale[row] : 1.f;
      const uint32_t ta = tmem + (uint32_t(q * 32) << 16) + uint32_t(buf * GM_BN);
#pragma unroll 1
      for (int c = 0; c < GM_BN; c += 16) {
        uint32_t r[16];
        tmem_ld16(ta + uint32_t(c), r);
        tmem_ld_wait();
        const int col = nb * GM_BN + c;
        if (!live || col >= g.N) continue;
        if (g.epi == GE_F32) {
          float* o = static_cast<float*>(g.out) + (size_t)row * g.ldo + col;
          if (g.ksplit > 1) {
            // this half of K's sum added into the zeroed output: with two
            // halves, 0 + a + b is the same in either order
#pragma unroll
            for (int i = 0; i < 4; ++i)
              asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(o + 4 * i),
                           "f"(__uint_as_float(r[4 * i]) * rs), "f"(__uint_as_float(r[4 * i + 1]) * rs),
                           "f"(__uint_as_float(r[4 * i + 2]) * rs), "f"(__uint_as_float(r[4 * i + 3]) * rs)
                           : "memory");
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              reinterpret_cast<float4*>(o)[i] =
                  make_float4(__uint_as_float(r[4 * i]) * rs, __uint_as_float(r[4 * i + 1]) * rs,
                              __uint_as_float(r[4 * i + 2]) * rs, __uint_as_float(r[4 * i + 3]) * rs);
          }
        } else {
          // columns alternate gate j, up j: eight SwiGLU outputs
          uint32_t h[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float g0 = __uint_as_float(r[4 * i]) * rs, u0 = __uint_as_float(r[4 * i + 1]) * rs;
            const float g1 = __uint_as_float(r[4 * i + 2]) * rs, u1 = __uint_as_float(r[4 * i + 3]) * rs;
            const float h0 = g0 / (1.f + expf(-g0)) * u0, h1 = g1 / (1.f + expf(-g1)) * u1;
            h[i] = uint32_t(f16_checked(h0, g.err)) | (uint32_t(f16_checked(h1, g.err)) << 16);
          }
          *reinterpret_cast<uint4*>(static_cast<uint16_t*>(g.out) + (size_t)row * g.ldo + col / 2) =
              make_uint4(h[0], h[1], h[2], h[3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty + buf);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TL::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Causal GQA flash attention over the prompt for head_dim 64 (mma.sync, bf16
// in, fp32 softmax; head_dim 128 runs on the tensor-memory kernel below)
// ---------------------------------------------------------------------------
// CTA = 64 consecutive query positions of one query head; 4 warps of 16
// queries.  Keys stream through shared memory in blocks of 64 positions
// (double buffered, cp.async).  Positions before the prompt come from the
// cache, whose rows keep their chunk permutation (16-byte chunk c of slot s at
// c ^ (s & 7); a block's row r has r = slot mod 8, since window and block
// start are multiples of 64, so a block never straddles the ring's wrap);
// the prompt's own keys come from a plain buffer and are permuted the same
// way on the way in.  The ldmatrix addressing undoes the permutation.  The
// prompt's keys are not in the cache yet: a ring of `window` slots cannot
// hold the windows of two consecutive queries, so they are appended after the
// attention (kv_append_kernel).
constexpr int FA_BQ = 64, FA_BK = 64, FA_THREADS = 128;

struct FaArgs {
  const uint16_t* q;    // bf16 [T][nq][hd]
  const uint16_t* kc;   // this layer's K region [batch][nkv][slots][hd]: positions before the prompt
  const uint16_t* vc;
  const uint16_t* kn;   // the prompt's own keys / values, bf16 [nkv][T][hd] in plain order
  const uint16_t* vn;
  uint16_t* out;        // fp16 [T][nq][hd]
  int T, nq, nkv, slots, window, start, seq;
  float scale_log2;     // log2(e) / sqrt(hd)
  uint32_t* err;
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int HD>
__global__ void __launch_bounds__(FA_THREADS, 3) flash_prefill_kernel(const FaArgs a) {
  constexpr int CH = HD / 8;            // 16-byte chunks per row
  constexpr int ROWB = HD * 2;          // bytes per key row
  extern __shared__ __align__(128) uint8_t fa_sm[];
  uint8_t* Ks = fa_sm;                  // [2][64][HD]
  uint8_t* Vs = fa_sm + 2 * FA_BK * ROWB;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int nqb = (a.T + FA_BQ - 1) / FA_BQ;
  const int qb = nqb - 1 - int(blockIdx.x);  // the longest rows first
  const int h = blockIdx.y;
  const int kvh = h / (a.nq / a.nkv);
  const int q0 = qb * FA_BQ;                 // first query of the CTA (prompt index)
  const int p_first = a.start + q0;
  const int p_last = a.start + min(q0 + FA_BQ, a.T) - 1;
  const int lo = a.window ? max(0, p_first - a.window + 1) : 0;
  const int jb0 = lo / FA_BK, jb1 = p_last / FA_BK;  // key blocks [jb0, jb1]
  const size_t head_base = ((size_t)a.seq * a.nkv + kvh) * a.slots;

  // Q fragments of this warp's 16 queries (rows beyond T are zero)
  uint32_t qf[HD / 16][4];
  {
    const int r0 = q0 + warp * 16 + g8, r1 = r0 + 8;
#pragma unroll
    for (int s = 0; s < HD / 16; ++s) {
      const int c = 16 * s + 2 * t4;
      auto ld = [&](int r, int cc) -> uint32_t {
        if (r >= a.T) return 0u;
        return *reinterpret_cast<const uint32_t*>(a.q + ((size_t)r * a.nq + h) * HD + cc);
      };
      qf[s][0] = ld(r0, c);
      qf[s][1] = ld(r1, c);
      qf[s][2] = ld(r0, c + 8);
      qf[s][3] = ld(r1, c + 8);
    }
  }
  const size_t new_base = (size_t)kvh * a.T;
  const int end = a.start + a.T;
  auto load_block = [&](int jb, int buf) {
    uint8_t* kd = Ks + buf * FA_BK * ROWB;
    uint8_t* vd = Vs + buf * FA_BK * ROWB;
#pragma unroll 1
    for (int i = threadIdx.x; i < FA_BK * CH; i += FA_THREADS) {
      const int r = i / CH, c = i % CH;
      const int j = jb * FA_BK + r;  // key position
      if (j >= end) {
        // beyond the prompt (masked keys): zeros, since a masked key's
        // weight 0 times a NaN would still poison the sum
        *reinterpret_cast<uint4*>(kd + r * ROWB + c * 16) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(vd + r * ROWB + c * 16) = make_uint4(0u, 0u, 0u, 0u);
      } else if (j >= a.start) {
        const size_t off = (new_base + (j - a.start)) * HD + c * 8;
        const int pc = (c ^ (r & 7)) * 16;
        cp_async16(kd + r * ROWB + pc, a.kn + off);
        cp_async16(vd + r * ROWB + pc, a.vn + off);
      } else {
        const int slot = a.window ? j % a.window : j;
        const size_t off = ((head_base + slot) * HD) + c * 8;  // stored order = shared-memory order
        cp_async16(kd + r * ROWB + c * 16, a.kc + off);
        cp_async16(vd + r * ROWB + c * 16, a.vc + off);
      }
    }
    cp_async_commit();
  };

  float o[HD / 8][4];
#pragma unroll
  for (int j = 0; j < HD / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const int pq0 = a.start + q0 + warp * 16 + g8, pq1 = pq0 + 8;  // positions of this thread's two rows

  load_block(jb0, 0);
#pragma unroll 1
  for (int jb = jb0; jb <= jb1; ++jb) {
    const int buf = (jb - jb0) & 1;
    if (jb < jb1) {
      load_block(jb + 1, buf ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint8_t* kb = Ks + buf * FA_BK * ROWB;
    const uint8_t* vb = Vs + buf * FA_BK * ROWB;
    // S = Q K^T: 16 queries x 64 keys (8 n-tiles of 8 keys)
    float sc[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
    const int lr = lane & 7, lm = lane >> 3;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const int row = 8 * n + lr;
#pragma unroll
      for (int s = 0; s < HD / 16; s += 2) {
        uint32_t k0, k1, k2, k3;
        ldsm_x4(k0, k1, k2, k3, kb + row * ROWB + (((2 * s + lm) ^ (row & 7)) << 4));
        mma_16816(sc[n], qf[s][0], qf[s][1], qf[s][2], qf[s][3], k0, k1);
        mma_16816(sc[n], qf[s + 1][0], qf[s + 1][1], qf[s + 1][2], qf[s + 1][3], k2, k3);
      }
    }
    // mask (causal, window) and online softmax in base 2; a block that every
    // row of the warp sees whole needs no mask (warp-uniform test)
    const int j0 = jb * FA_BK;
    const int wq_lo = a.start + q0 + warp * 16, wq_hi = wq_lo + 15;
    const bool whole = j0 + FA_BK - 1 <= wq_lo && (a.window == 0 || wq_hi - j0 < a.window);
    float mx0 = -INFINITY, mx1 = -INFINITY;
    if (whole) {
#pragma unroll
      for (int n = 0; n < 8; ++n) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          sc[n][e] *= a.scale_log2;
          sc[n][2 + e] *= a.scale_log2;
          mx0 = fmaxf(mx0, sc[n][e]);
          mx1 = fmaxf(mx1, sc[n][2 + e]);
        }
      }
    } else {
#pragma unroll
      for (int n = 0; n < 8; ++n) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int j = j0 + 8 * n + 2 * t4 + e;
          const bool v0 = j <= pq0 && (a.window == 0 || pq0 - j < a.window);
          const bool v1 = j <= pq1 && (a.window == 0 || pq1 - j < a.window);
          sc[n][e] = v0 ? sc[n][e] * a.scale_log2 : -INFINITY;
          sc[n][2 + e] = v1 ? sc[n][2 + e] * a.scale_log2 : -INFINITY;
          mx0 = fmaxf(mx0, sc[n][e]);
          mx1 = fmaxf(mx1, sc[n][2 + e]);
        }
      }
    }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float ref0 = (mn0 == -INFINITY) ? 0.f : mn0, ref1 = (mn1 == -INFINITY) ? 0.f : mn1;
    const float al0 = exp2f(m0 - ref0), al1 = exp2f(m1 - ref1);
    m0 = mn0;
    m1 = mn1;
    float s0 = 0.f, s1 = 0.f;
    uint32_t pf[4][4];  // P as A fragments of the 4 key k-steps
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const float p00 = exp2f(sc[n][0] - ref0), p01 = exp2f(sc[n][1] - ref0);
      const float p10 = exp2f(sc[n][2] - ref1), p11 = exp2f(sc[n][3] - ref1);
      s0 += p00 + p01;
      s1 += p10 + p11;
      const uint32_t w0 = pack_bf16x2(p00, p01), w1 = pack_bf16x2(p10, p11);
      pf[n >> 1][(n & 1) ? 2 : 0] = w0;
      pf[n >> 1][(n & 1) ? 3 : 1] = w1;
    }
    l0 = l0 * al0 + s0;
    l1 = l1 * al1 + s1;
#pragma unroll
    for (int j = 0; j < HD / 8; ++j) {
      o[j][0] *= al0;
      o[j][1] *= al0;
      o[j][2] *= al1;
      o[j][3] *= al1;
    }
    // O += P V: 4 k-steps of 16 keys, HD / 8 n-tiles of 8 dims (two per ldmatrix)
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int row = 16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
      for (int d2 = 0; d2 < HD / 16; ++d2) {
        uint32_t v0, v1, v2, v3;
        const int ch = 2 * d2 + (lane >> 4);
        ldsm_x4_t(v0, v1, v2, v3, vb + row * ROWB + ((ch ^ (row & 7)) << 4));
        mma_16816(o[2 * d2], pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3], v0, v1);
        mma_16816(o[2 * d2 + 1], pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3], v2, v3);
      }
    }
    __syncthreads();  // the buffer is refilled by the next iteration's load
  }
#pragma unroll
  for (int off = 1; off <= 2; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
  const int r0 = q0 + warp * 16 + g8, r1 = r0 + 8;
#pragma unroll
  for (int j = 0; j < HD / 8; ++j) {
    const int c = 8 * j + 2 * t4;
    if (r0 < a.T)
      *reinterpret_cast<uint32_t*>(a.out + ((size_t)r0 * a.nq + h) * HD + c) =
          uint32_t(f16_checked(o[j][0] * i0, a.err)) | (uint32_t(f16_checked(o[j][1] * i0, a.err)) << 16);
    if (r1 < a.T)
      *reinterpret_cast<uint32_t*>(a.out + ((size_t)r1 * a.nq + h) * HD + c) =
          uint32_t(f16_checked(o[j][2] * i1, a.err)) | (uint32_t(f16_checked(o[j][3] * i1, a.err)) << 16);
  }
}

// ---------------------------------------------------------------------------
// Causal GQA flash attention on the tcgen05 tensor cores (head_dim 128)
// ---------------------------------------------------------------------------
// CTA = two tiles of 128 consecutive queries of one query head (tile 0 the
// earlier); they share every key / value block of 128 positions.  Per block:
// S_i = Q_i K^T into tensor memory, the softmax warps of tile i turn their
// rows of S_i into bf16 P_i in shared memory, O_i += P_i V accumulates in
// tensor memory.  The two tiles alternate on the tensor core, so one tile's
// softmax runs under the other's MMAs.  Warp roles: warps 0-3 the softmax of
// tile 0 and 4-7 of tile 1 (thread = query row = TMEM lane), warp 8 the
// loads (Q, K and V by tensor copies, from the prompt's buffers or from the
// cache; the one block that straddles the prompt's start, or a ring's wrap,
// is gathered row by row by the whole warp), warp 9 the MMAs (one thread)
// and the 512 TMEM columns (S_0, S_1, O_0, O_1).  K and V tiles are stored
// alike (rows = keys, 128-byte swizzle, two 64-column panels): S reads K as
// a K-major operand, O reads V as an MN-major one.  The online softmax keeps
// a row's reference maximum until a block raises it by more than 2^8, so O is
// rescaled (read, scaled, written back in TMEM) only on those rare blocks;
// P <= 2^8 meanwhile, exact enough in bf16 and fp32.
constexpr int FT_BQ = 128, FT_BK = 128, FT_HD = 128;
constexpr int FT_PANEL = 128 * 128;       // 128 rows x 64 bf16
constexpr int FT_TILE = 2 * FT_PANEL;     // 128 x 128 bf16
constexpr int FT_NS = 3;                  // K / V ring slots (K_j, V_j, K_j+1, ... in load order)
constexpr int FT_THREADS = 320;
constexpr int FT_SMEM = (4 + FT_NS) * FT_TILE + 128 + 1024;
constexpr float FT_RESCALE = 8.f;
static_assert(FT_SMEM <= 232448, "flash shared memory");

struct FtArgs {
  const uint16_t* kc;   // this layer's cache region [batch][nkv][slots][hd] (rows chunk-permuted)
  const uint16_t* vc;
  const uint16_t* kn;   // the prompt's keys / values, bf16 [nkv][T][hd]
  const uint16_t* vn;
  uint16_t* out;        // fp16 [T][nq][hd]
  int T, nq, nkv, slots, window, start, seq;
  float scale_log2;
  uint32_t* err;
};

// Bounded wait by every lane of a warp; false (the abort flag and the error
// word set) on a timeout or when another role has given up.
__device__ __forceinline__ bool ft_wait(uint64_t* bar, uint32_t par, volatile int* abort_flag, uint32_t* err) {
  if (mbar_wait_sleep(bar, par)) return true;
  const long long t0 = clock64();
  while (!mbar_wait_sleep(bar, par)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > PF_WAIT) {
      *abort_flag = 1;
      pf_error(err, EW_MBAR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Rows of a key / value block that reaches back into the cache, gathered by
// the 32 lanes into the tile layout (row r = position pb + r): cache rows
// verbatim but for their chunk order, prompt rows, zeros past the prompt.
__device__ __forceinline__ void ft_gather(uint8_t* dst, const uint16_t* cache, const uint16_t* prompt, int pb, int kvh,
                                          const FtArgs& a, int lane) {
#pragma unroll 1
  for (int idx = lane; idx < FT_BK * 16; idx += 32) {
    const int r = idx >> 4, c = idx & 15;
    uint8_t* d = dst + (c >> 3) * FT_PANEL + r * 128 + (((c & 7) ^ (r & 7)) << 4);
    const int p = pb + r;
    if (p < a.start) {
      const int slot = a.window ? p % a.window : p;
      const size_t row = ((size_t)a.seq * a.nkv + kvh) * a.slots + slot;
      cp_async16(d, cache + row * FT_HD + ((c ^ (slot & 7)) << 3));
    } else if (p < a.start + a.T) {
      cp_async16(d, prompt + ((size_t)kvh * a.T + (p - a.start)) * FT_HD + (c << 3));
    } else {
      *reinterpret_cast<uint4*>(d) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  cp_async_commit();
}

// 2^x on the special-function unit (results below 2^-126 flush to zero)
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Two floats rounded to bf16 in one conversion (lo in the low half).
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

__global__ void __launch_bounds__(FT_THREADS, 1)
    flash_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKc,
                    const __grid_constant__ CUtensorMap tmVc, const FtArgs a) {
  extern __shared__ uint8_t ft_raw[];
  uint8_t* sm = ft_raw + ((1024u - (smem_addr(ft_raw) & 1023u)) & 1023u);
  uint8_t* sQ = sm;                  // Q_0, Q_1
  uint8_t* sP = sm + 2 * FT_TILE;    // P_0, P_1
  uint8_t* sR = sm + 4 * FT_TILE;    // ring
  uint64_t* q_full = reinterpret_cast<uint64_t*>(sm + (4 + FT_NS) * FT_TILE);
  uint64_t* kv_full = q_full + 1;          // [FT_NS]
  uint64_t* kv_empty = kv_full + FT_NS;    // [FT_NS]
  uint64_t* s_full = kv_empty + FT_NS;     // [2]: S_i computed (and every earlier MMA done)
  uint64_t* p_full = s_full + 2;           // [2]: P_i written, O_i rescaled (4 warps arrive)
  uint64_t* o_done = p_full + 2;           // every MMA of the CTA done
  uint32_t* tbase = reinterpret_cast<uint32_t*>(o_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tbase + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int npair = (a.T + 2 * FT_BQ - 1) / (2 * FT_BQ);
  const int q0 = (npair - 1 - int(blockIdx.x)) * 2 * FT_BQ;  // the longest rows first
  const int h = blockIdx.y, kvh = h / (a.nq / a.nkv);
  const int p_first = a.start + q0;
  const int p_last = a.start + min(q0 + 2 * FT_BQ, a.T) - 1;
  const int lo = a.window ? max(0, p_first - a.window + 1) : 0;
  const int b0 = lo / FT_BK, nb = p_last / FT_BK - b0 + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
#pragma unroll 1
    for (int s = 0; s < FT_NS; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    mbar_init(s_full + 0, 1);
    mbar_init(s_full + 1, 1);
    mbar_init(p_full + 0, 4);
    mbar_init(p_full + 1, 4);
    mbar_init(o_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
    tma_prefetch_map(&tmKc);
    tma_prefetch_map(&tmVc);
  }
  if (warp == 9) {
    tmem_alloc(tbase, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;

  if (warp == 8) {
    // ---- loads ----
    if (lane == 0) {
      mbar_expect_tx(q_full, 2 * FT_TILE);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        tma_load_3d(sQ + i * FT_TILE, &tmQ, 0, h, q0 + i * FT_BQ, q_full);
        tma_load_3d(sQ + i * FT_TILE + FT_PANEL, &tmQ, 64, h, q0 + i * FT_BQ, q_full);
      }
    }
    uint32_t it = 0;
    bool ok = true;
#pragma unroll 1
    for (int j = 0; j < nb && ok; ++j) {
      const int pb = (b0 + j) * FT_BK;
#pragma unroll 1
      for (int kv = 0; kv < 2; ++kv, ++it) {
        const int s = int(it % FT_NS);
        if (it >= FT_NS) {
          int good = 1;
          if (lane == 0) good = ft_wait(kv_empty + s, ((it / FT_NS) - 1u) & 1u, abort_flag, a.err) ? 1 : 0;
          if (!__shfl_sync(0xffffffffu, good, 0)) {
            ok = false;
            break;
          }
        }
        uint8_t* dst = sR + s * FT_TILE;
        if (pb >= a.start) {
          if (lane == 0) {
            const CUtensorMap* m = kv ? &tmV : &tmK;
            mbar_expect_tx(kv_full + s, FT_TILE);
            tma_load_3d(dst, m, 0, pb - a.start, kvh, kv_full + s);
            tma_load_3d(dst + FT_PANEL, m, 64, pb - a.start, kvh, kv_full + s);
          }
        } else if (pb + FT_BK <= a.start && (a.window == 0 || pb % a.window + FT_BK <= a.window)) {
          // history only, in consecutive slots: the cache rows already carry
          // the tile's chunk order (chunk c of slot s at c ^ (s & 7), and
          // s = pb + r mod 8), so a plain tensor copy lays the tile out
          if (lane == 0) {
            const CUtensorMap* m = kv ? &tmVc : &tmKc;
            const int slot0 = a.window ? pb % a.window : pb;
            mbar_expect_tx(kv_full + s, FT_TILE);
            tma_load_3d(dst, m, 0, slot0, a.seq * a.nkv + kvh, kv_full + s);
            tma_load_3d(dst + FT_PANEL, m, 64, slot0, a.seq * a.nkv + kvh, kv_full + s);
          }
        } else {
          ft_gather(dst, kv ? a.vc : a.kc, kv ? a.vn : a.kn, pb, kvh, a, lane);
          cp_async_wait<0>();
          fence_proxy_async();  // the rows are read by the tensor core
          __syncwarp();
          if (lane == 0) mbar_arrive(kv_full + s);
        }
      }
    }
    // tensor copies still in flight land before the CTA may exit
    if (lane == 0) {
      const uint32_t first = it > uint32_t(FT_NS) ? it - FT_NS : 0u;
#pragma unroll 1
      for (uint32_t j = first; j < it; ++j) {
        const long long t0 = clock64();
        while (!mbar_try_wait(kv_full + (j % FT_NS), (j / FT_NS) & 1u)) {
          if (clock64() - t0 > PF_WAIT) {
            pf_error(a.err, EW_DRAIN_TIMEOUT);
            break;
          }
        }
      }
    }
  } else if (warp == 9) {
    // ---- MMAs (one thread) ----
    if (lane == 0) {
      const uint32_t idS = umma_idesc_f16(128, 128, true);
      const uint32_t idO = idS | UMMA_B_MN;
      auto tile_ready = [&](uint32_t i) {
        return ft_wait(kv_full + i % FT_NS, (i / FT_NS) & 1u, abort_flag, a.err);
      };
      // S_qi = Q_qi K^T, K = ring tile ki
      auto issue_s = [&](int qi, uint32_t ki) {
        const uint8_t* q = sQ + qi * FT_TILE;
        const uint8_t* k = sR + (ki % FT_NS) * FT_TILE;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = uint32_t((ks >> 2) * FT_PANEL + (ks & 3) * 32);
          umma_f16(tmem + uint32_t(qi * 128), umma_desc_sw128(q, off), umma_desc_sw128(k, off), idS,
                   ks > 0 ? 1u : 0u);
        }
        umma_commit(s_full + qi);
      };
      // O_qi (+)= P_qi V, V = ring tile vi (MN-major: 64-column atoms a panel apart, 8-key groups 1 KB apart)
      auto issue_pv = [&](int qi, uint32_t vi, bool first) {
        const uint8_t* pm = sP + qi * FT_TILE;
        const uint8_t* v = sR + (vi % FT_NS) * FT_TILE;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = uint32_t((ks >> 2) * FT_PANEL + (ks & 3) * 32);
          umma_f16(tmem + uint32_t(256 + qi * 128), umma_desc_sw128(pm, off),
                   umma_desc_mn_sw128(v + ks * 16 * 128, FT_PANEL, 1024), idO, (first && ks == 0) ? 0u : 1u);
        }
      };
      bool ok = ft_wait(q_full, 0u, abort_flag, a.err) && tile_ready(0);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        umma_commit(kv_empty + 0);
      }
#pragma unroll 1
      for (int j = 0; j < nb && ok; ++j) {
        const uint32_t vt = 2u * j + 1u, kn = 2u * j + 2u;
        const bool more = j + 1 < nb;
        if (!tile_ready(vt) || !ft_wait(p_full + 0, uint32_t(j) & 1u, abort_flag, a.err)) break;
        tc_fence_after();
        issue_pv(0, vt, j == 0);
        if (more) {
          if (!tile_ready(kn)) break;
          tc_fence_after();
          issue_s(0, kn);
        }
        if (!ft_wait(p_full + 1, uint32_t(j) & 1u, abort_flag, a.err)) break;
        tc_fence_after();
        issue_pv(1, vt, j == 0);
        umma_commit(kv_empty + vt % FT_NS);
        if (more) {
          issue_s(1, kn);
          umma_commit(kv_empty + kn % FT_NS);
        }
      }
      umma_commit(o_done);
      // every MMA issued has completed before the tensor memory is freed
      const long long t0 = clock64();
      while (!mbar_try_wait(o_done, 0u)) {
        if (clock64() - t0 > PF_WAIT) {
          pf_error(a.err, EW_DRAIN_TIMEOUT);
          break;
        }
      }
    }
  } else {
    // ---- softmax of tile qi: thread = query row = TMEM lane ----
    const int qi = warp >> 2, r = (warp & 3) * 32 + lane;
    const int t = q0 + qi * FT_BQ + r;
    const int p = a.start + t;
    const uint32_t tl = tmem + (uint32_t((warp & 3) * 32) << 16);
    const uint32_t tS = tl + uint32_t(qi * 128), tO = tl + uint32_t(256 + qi * 128);
    uint8_t* prow = sP + qi * FT_TILE + r * 128;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
#pragma unroll 1
    for (int j = 0; j < nb; ++j) {
      if (!__all_sync(0xffffffffu, ft_wait(s_full + qi, uint32_t(j) & 1u, abort_flag, a.err))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // the row of S in four 32-column register groups, one wait; keys pb + i
      // visible to this row: i in [ilo, ihi] (the whole block on most blocks;
      // the others get -inf where hidden)
      const int pb = (b0 + j) * FT_BK;
      const int ilo = a.window ? max(0, p - a.window + 1 - pb) : 0;
      const int ihi = min(FT_BK - 1, p - pb);
      uint32_t v0[32], v1[32], v2[32], v3[32];
      tmem_ld32(tS + 0u, v0);
      tmem_ld32(tS + 32u, v1);
      tmem_ld32(tS + 64u, v2);
      tmem_ld32(tS + 96u, v3);
      tmem_ld_wait();
      if (ilo > 0 || ihi < FT_BK - 1) {
        auto hide = [&](uint32_t (&v)[32], int c0) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c0 + i < ilo || c0 + i > ihi) v[i] = 0xff800000u;  // -inf
        };
        hide(v0, 0);
        hide(v1, 32);
        hide(v2, 64);
        hide(v3, 96);
      }
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; ++i)
        mx = fmaxf(fmaxf(mx, fmaxf(__uint_as_float(v0[i]), __uint_as_float(v1[i]))),
                   fmaxf(__uint_as_float(v2[i]), __uint_as_float(v3[i])));
      mx *= a.scale_log2;  // a positive scale commutes with the maximum
      float alpha = 1.f;
      if (mx > m_run + FT_RESCALE) {  // also the first finite maximum of the row
        alpha = exp2f(m_run - mx);    // 0 while the reference was -inf
        m_run = mx;
      }
      const float nref = m_run == -INFINITY ? 0.f : -m_run;
      float sum = 0.f;
      // P = 2^(s scale - m) rounded to bf16, 16 bytes (8 keys) per store
      auto emit = [&](const uint32_t (&v)[32], int c0) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float p0 = ex2_fast(fmaf(__uint_as_float(v[8 * k + 2 * e]), a.scale_log2, nref));
            const float p1 = ex2_fast(fmaf(__uint_as_float(v[8 * k + 2 * e + 1]), a.scale_log2, nref));
            sum += p0 + p1;
            w[e] = cvt_bf16x2(p0, p1);
          }
          const int c8 = (c0 >> 3) + k;
          *reinterpret_cast<uint4*>(prow + (c8 >> 3) * FT_PANEL + (((c8 & 7) ^ (r & 7)) << 4)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      };
      emit(v0, 0);
      emit(v1, 32);
      emit(v2, 64);
      emit(v3, 96);
      l_run = l_run * alpha + sum;
      // O rows whose reference moved (the previous block's P V has completed:
      // S_qi's barrier follows it)
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t o[32];
          tmem_ld32(tO + uint32_t(c), o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tO + uint32_t(c), o);
        }
        tmem_st_wait();
      }
      fence_proxy_async();  // P is read by the tensor core
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full + qi);
    }
    if (ok && __all_sync(0xffffffffu, ft_wait(o_done, 0u, abort_flag, a.err))) {
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      uint16_t* orow = a.out + ((size_t)t * a.nq + h) * FT_HD;
#pragma unroll 1
      for (int c = 0; c < 128; c += 32) {
        uint32_t o[32];
        tmem_ld32(tO + uint32_t(c), o);
        tmem_ld_wait();
        if (t < a.T) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w[e] = uint32_t(f16_checked(__uint_as_float(o[i + 2 * e]) * inv, a.err)) |
                     (uint32_t(f16_checked(__uint_as_float(o[i + 2 * e + 1]) * inv, a.err)) << 16);
            *reinterpret_cast<uint4*>(orow + c + i) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Per-token row kernels (one CTA of 256 threads per token)
// ---------------------------------------------------------------------------
constexpr int RT = 256;

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < RT / 32; ++i) s += red[i];
  return s;
}
__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < RT / 32; ++i) s = fmaxf(s, red[i]);
  return s;
}

// fp16 copy of a residual row with the range guard: rows whose max |x|
// reaches 2^15 are scaled by a power of two first; scale[t] undoes it.
__device__ __forceinline__ void row_to_f16(const float* x, int d, uint16_t* x16, float* scale, float* red) {
  float mx = 0.f;
  for (int i = threadIdx.x; i < d; i += RT) mx = fmaxf(mx, fabsf(x[i]));
  mx = block_max(mx, red);
  float s = 1.f, inv = 1.f;
  if (mx >= 32768.f) {
    int ex;
    frexpf(mx, &ex);
    s = ldexpf(1.f, 15 - ex);
    inv = ldexpf(1.f, ex - 15);
  }
  for (int i = threadIdx.x; i < d; i += RT) x16[i] = f32_to_f16(x[i] * s);
  if (threadIdx.x == 0) *scale = inv;
}

__global__ void __launch_bounds__(RT) embed_rows_kernel(const int32_t* __restrict__ tokens, const uint16_t* embed,
                                                        int vocab, int d, float* X, uint16_t* X16, float* scale,
                                                        uint32_t* err) {
  __shared__ float red[RT / 32];
  const int t = blockIdx.x;
  int tok = tokens[t];
  if (tok < 0 || tok >= vocab) {
    if (threadIdx.x == 0) pf_error(err, EW_BAD_SHAPE);
    tok = tok < 0 ? 0 : vocab - 1;
  }
  float* x = X + (size_t)t * d;
  for (int i = threadIdx.x; i < d; i += RT) x[i] = bf16_to_f32(embed[(size_t)tok * d + i]);
  __syncthreads();
  row_to_f16(x, d, X16 + (size_t)t * d, scale + t, red);
}

// X[t] += RMSNorm(V[t]) * gain, then the fp16 copy for the next GEMM.
__global__ void __launch_bounds__(RT) resid_rows_kernel(const float* __restrict__ V, const float* __restrict__ gain,
                                                        int d, float eps, float* X, uint16_t* X16, float* scale) {
  __shared__ float red[RT / 32];
  const int t = blockIdx.x;
  const float* v = V + (size_t)t * d;
  float ss = 0.f;
  for (int i = threadIdx.x; i < d; i += RT) ss += v[i] * v[i];
  ss = block_sum(ss, red);
  const float r = rsqrtf(ss / float(d) + eps);
  float* x = X + (size_t)t * d;
  for (int i = threadIdx.x; i < d; i += RT) x[i] += v[i] * r * gain[i];
  __syncthreads();
  row_to_f16(x, d, X16 + (size_t)t * d, scale + t, red);
}

// The last prompt token's input to the lm_head: RMSNorm with the final gains
// (none when `gain` is null), rounded to bf16.  One CTA.
__global__ void __launch_bounds__(RT) final_row_kernel(const float* __restrict__ x, const float* __restrict__ gain,
                                                       int d, float eps, uint16_t* __restrict__ xb) {
  __shared__ float red[RT / 32];
  float r = 1.f;
  if (gain != nullptr) {
    float ss = 0.f;
    for (int i = threadIdx.x; i < d; i += RT) ss += x[i] * x[i];
    ss = block_sum(ss, red);
    r = rsqrtf(ss / float(d) + eps);
  }
  for (int i = threadIdx.x; i < d; i += RT) xb[i] = f32_to_bf16(gain != nullptr ? x[i] * r * gain[i] : x[i]);
}

// logits = W . x for one bf16 row x and the bf16 lm_head W in 16-row x
// 128-column units of mma A fragments (the decode layout).  HBM-bound: each
// warp takes whole 16-row blocks from a counter (so every row's sum runs in
// one fixed order) and streams the block's units with two in flight; x sits
// in shared memory and enters the mma as the n = 0 column (the other seven
// columns are zero).
constexpr int HG_THREADS = 256;
__global__ void __launch_bounds__(HG_THREADS) head_gemv_kernel(const uint8_t* __restrict__ W, int n, int k,
                                                               const uint16_t* __restrict__ xb, float* __restrict__ out,
                                                               int* __restrict__ counter) {
  extern __shared__ __align__(16) uint16_t hg_x[];
  for (int i = threadIdx.x * 8; i < k; i += HG_THREADS * 8)
    *reinterpret_cast<uint4*>(hg_x + i) = *reinterpret_cast<const uint4*>(xb + i);
  __syncthreads();
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int nrb = (n + RB - 1) / RB, nkc = k / BF_KC;
#pragma unroll 1
  for (;;) {
    int rb = 0;
    if (lane == 0) rb = atomicAdd(counter, 1);
    rb = __shfl_sync(0xffffffffu, rb, 0);
    if (rb >= nrb) break;
    const uint4* u = reinterpret_cast<const uint4*>(W + (size_t)rb * nkc * BF_UNIT) + lane;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    auto math = [&](const uint4 (&av)[8], int kc) {
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        // k-step s holds columns 32 m + 8 t + 4 e + (0..3), m = s / 2, e = s % 2
        const int c = kc * BF_KC + 32 * (s >> 1) + 8 * t + 4 * (s & 1);
        const uint2 xv = g == 0 ? *reinterpret_cast<const uint2*>(hg_x + c) : make_uint2(0u, 0u);
        mma_16816(acc, av[s].x, av[s].y, av[s].z, av[s].w, xv.x, xv.y);
      }
    };
    auto load = [&](uint4 (&av)[8], int kc) {
      const uint4* un = u + (size_t)kc * (BF_UNIT / 16);
#pragma unroll
      for (int i = 0; i < 8; ++i) av[i] = __ldcs(un + i * 32);
    };
    uint4 a0[8], a1[8];
    load(a0, 0);
#pragma unroll 1
    for (int kc = 0; kc < nkc; kc += 2) {
      if (kc + 1 < nkc) load(a1, kc + 1);
      math(a0, kc);
      if (kc + 2 < nkc) load(a0, kc + 2);
      if (kc + 1 < nkc) math(a1, kc + 1);
    }
    if (t == 0) {
      const int r0 = rb * RB + g, r1 = r0 + 8;
      if (r0 < n) out[r0] = acc[0];
      if (r1 < n) out[r1] = acc[2];
    }
  }
}

struct QkArgs {
  const float* Y;         // [T][q_dim + 2 kv_dim]
  const float* qg;        // q gains [q_dim]
  const float* kg;        // k gains [kv_dim]
  uint16_t* q16;          // bf16 [T][nq][hd]
  uint16_t* kn;           // the prompt's keys / values, bf16 [nkv][T][hd]
  uint16_t* vn;
  double f[64];           // inverse frequencies of the layer type
  float ms;               // attention factor
  float eps;
  int T, nq, nkv, hd, start;
};

// QK-norm over the whole projections, gains, rotation (pairs i, i + hd / 2),
// the query, key and value as bf16.
__global__ void __launch_bounds__(RT) qk_rows_kernel(const __grid_constant__ QkArgs a) {
  __shared__ float red[RT / 32];
  const int t = blockIdx.x;
  const int qd = a.nq * a.hd, kd = a.nkv * a.hd, H2 = a.hd / 2;
  const float* y = a.Y + (size_t)t * (qd + 2 * kd);
  float sq = 0.f, sk = 0.f;
  for (int i = threadIdx.x; i < qd; i += RT) sq += y[i] * y[i];
  for (int i = threadIdx.x; i < kd; i += RT) sk += y[qd + i] * y[qd + i];
  sq = block_sum(sq, red);
  sk = block_sum(sk, red);
  const float rq = rsqrtf(sq / float(qd) + a.eps), rk = rsqrtf(sk / float(kd) + a.eps);
  const int pos = a.start + t;
  // the rotation of pair i at this position, shared by every head
  __shared__ float2 rot[64];
  for (int i = threadIdx.x; i < H2; i += RT) {
    const double ang = double(pos) * a.f[i];
    const double rr = ang - 6.283185307179586 * rint(ang * 0.15915494309189535);
    float sn, cs;
    sincosf(float(rr), &sn, &cs);
    rot[i] = make_float2(cs * a.ms, sn * a.ms);
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < (a.nq + a.nkv) * H2; idx += RT) {
    const bool isq = idx < a.nq * H2;
    const int j = isq ? idx : idx - a.nq * H2;
    const int hh = j / H2, i = j - hh * H2;
    const float cs = rot[i].x, sn = rot[i].y;
    if (isq) {
      const int c = hh * a.hd + i;
      const float x1 = y[c] * rq * a.qg[c], x2 = y[c + H2] * rq * a.qg[c + H2];
      a.q16[(size_t)t * qd + c] = f32_to_bf16(x1 * cs - x2 * sn);
      a.q16[(size_t)t * qd + c + H2] = f32_to_bf16(x2 * cs + x1 * sn);
    } else {
      const int c = hh * a.hd + i;
      const float x1 = y[qd + c] * rk * a.kg[c], x2 = y[qd + c + H2] * rk * a.kg[c + H2];
      const size_t row = ((size_t)hh * a.T + t) * a.hd;
      a.kn[row + i] = f32_to_bf16(x1 * cs - x2 * sn);
      a.kn[row + i + H2] = f32_to_bf16(x2 * cs + x1 * sn);
      a.vn[row + i] = f32_to_bf16(y[qd + kd + c]);
      a.vn[row + i + H2] = f32_to_bf16(y[qd + kd + c + H2]);
    }
  }
}

// The prompt's keys and values of positions start + t, t in [t0, T), into
// the cache (slot = position, or position % window on a ring), with the
// cache's chunk permutation; one thread per 16-byte chunk.
__global__ void kv_append_kernel(uint16_t* __restrict__ kc, uint16_t* __restrict__ vc, const uint16_t* __restrict__ kn,
                                 const uint16_t* __restrict__ vn, int nkv, int hd, int slots, int window, int seq,
                                 int start, int T, int t0) {
  const int ch = hd / 8;
  const int64_t total = (int64_t)nkv * (T - t0) * ch;
  const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= total) return;
  const int c = int(id % ch);
  const int64_t rest = id / ch;
  const int t = t0 + int(rest % (T - t0));
  const int h = int(rest / (T - t0));
  const int pos = start + t;
  const int slot = window ? pos % window : pos;
  const size_t src = ((size_t)h * T + t) * hd + c * 8;
  const size_t dst = (((size_t)seq * nkv + h) * slots + slot) * hd + ((c ^ (slot & 7)) * 8);
  *reinterpret_cast<uint4*>(kc + dst) = *reinterpret_cast<const uint4*>(kn + src);
  *reinterpret_cast<uint4*>(vc + dst) = *reinterpret_cast<const uint4*>(vn + src);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// K-major fp16 matrix [rows, k] (row stride k), box of box_rows x 64 with the 128-byte swizzle.
static cudaError_t make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t k, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {cuuint64_t(k), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(k * 2)};
  const cuuint32_t box[2] = {cuuint32_t(GM_BK), cuuint32_t(box_rows)};
  const cuuint32_t es[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// bf16 3-D tensor [d2][d1][d0] (d0 contiguous; row strides in bytes), box of
// 64 x b1 x b2 with the 128-byte swizzle.
static cudaError_t make_map3(CUtensorMap* m, const void* base, int64_t d0, int64_t d1, int64_t d2, int64_t s1,
                             int64_t s2, int b1, int b2, bool swizzle = true) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {cuuint64_t(d0), cuuint64_t(d1), cuuint64_t(d2)};
  const cuuint64_t strides[2] = {cuuint64_t(s1), cuuint64_t(s2)};
  const cuuint32_t box[3] = {64u, cuuint32_t(b1), cuuint32_t(b2)};
  const cuuint32_t es[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

static cudaError_t launch_flash_tc(const uint16_t* q, const uint16_t* kc, const uint16_t* vc, const uint16_t* kn,
                                   const uint16_t* vn, uint16_t* out, int T, int nq, int nkv, int slots, int window,
                                   int start, int seq, uint32_t* err, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    const cudaError_t e = cudaFuncSetAttribute(flash_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, FT_SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  CUtensorMap mq, mk, mv;
  // q [T][nq][128]: boxes of 64 dims x 1 head x 128 tokens
  cudaError_t e = make_map3(&mq, q, FT_HD, nq, T, (int64_t)FT_HD * 2, (int64_t)nq * FT_HD * 2, 1, FT_BQ);
  if (e != cudaSuccess) return e;
  // the prompt's K / V [nkv][T][128]: boxes of 64 dims x 128 keys x 1 head
  e = make_map3(&mk, kn, FT_HD, T, nkv, (int64_t)FT_HD * 2, (int64_t)T * FT_HD * 2, FT_BK, 1);
  if (e != cudaSuccess) return e;
  e = make_map3(&mv, vn, FT_HD, T, nkv, (int64_t)FT_HD * 2, (int64_t)T * FT_HD * 2, FT_BK, 1);
  if (e != cudaSuccess) return e;
  // the cache regions [.. seq][nkv][slots][128], rows as stored (no swizzle)
  CUtensorMap mkc, mvc;
  e = make_map3(&mkc, kc, FT_HD, slots, (int64_t)(seq + 1) * nkv, (int64_t)FT_HD * 2, (int64_t)slots * FT_HD * 2, FT_BK,
                1, false);
  if (e != cudaSuccess) return e;
  e = make_map3(&mvc, vc, FT_HD, slots, (int64_t)(seq + 1) * nkv, (int64_t)FT_HD * 2, (int64_t)slots * FT_HD * 2, FT_BK,
                1, false);
  if (e != cudaSuccess) return e;
  FtArgs a;
  a.kc = kc;
  a.vc = vc;
  a.kn = kn;
  a.vn = vn;
  a.out = out;
  a.T = T;
  a.nq = nq;
  a.nkv = nkv;
  a.slots = slots;
  a.window = window;
  a.start = start;
  a.seq = seq;
  a.scale_log2 = float(1.4426950408889634 / sqrt(double(FT_HD)));
  a.err = err;
  const dim3 grid((T + 2 * FT_BQ - 1) / (2 * FT_BQ), nq);
  flash_tc_kernel<<<grid, FT_THREADS, FT_SMEM, st>>>(mq, mk, mv, mkc, mvc, a);
  return cudaGetLastError();
}

cudaError_t launch_dequant_f16(const uint8_t* tiled, int64_t n, int64_t k, int fmt, uint16_t* out, cudaStream_t st) {
  const int units = dequant_units(n, k, fmt);
  dequant_f16_kernel<<<(unsigned)((units + 7) / 8), 256, 0, st>>>(tiled, n, k, fmt, out);
  return cudaGetLastError();
}

template <int BN>
static cudaError_t launch_gemm_tile(const CUtensorMap& ma, const uint16_t* B, int M, int N, int K, const GemmArgs& g,
                                   int n_sms, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    const cudaError_t e =
        cudaFuncSetAttribute(gemm_f16_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, GmTile<BN>::SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  CUtensorMap mb;
  const cudaError_t e = make_map(&mb, B, N, K, BN);
  if (e != cudaSuccess) return e;
  const int tiles = ((M + GM_BM - 1) / GM_BM) * ((N + BN - 1) / BN);
  const int grid = tiles < n_sms ? tiles : n_sms;
  gemm_f16_kernel<BN><<<grid, GM_THREADS, GmTile<BN>::SMEM, st>>>(ma, mb, g);
  return cudaGetLastError();
}

// Tile width of a GEMM: the persistent CTAs take tiles round-robin, so the
// time goes as the number of waves of tiles times a tile's time.  A 128-wide
// tile takes about 0.77 of a 256-wide one (its A slice is read from shared
// memory for half the columns); it is chosen when its waves cost less, which
// happens for short prompts whose tiles do not fill one wave.
int gemm_tile_width(int M, int N, int n_sms) {
  const int64_t mt = (M + GM_BM - 1) / GM_BM;
  const int64_t w256 = (mt * ((N + 255) / 256) + n_sms - 1) / n_sms;
  const int64_t w128 = (mt * ((N + 127) / 128) + n_sms - 1) / n_sms;
  return double(w128) * GM_NARROW_COST < double(w256) ? 128 : 256;
}

// K in two halves (the tile count doubles, each tile does half the work) when
// that fills the last wave of tiles better: long K, few tiles (short prompts
// through O and down).  Only the plain fp32 output sums partial products.
int gemm_ksplit(int M, int N, int K, int bn, int epi, int n_sms) {
  if (epi != GE_F32 || K / GM_BK < 16) return 1;
  const int64_t tiles = (int64_t)((M + GM_BM - 1) / GM_BM) * ((N + bn - 1) / bn);
  const int64_t w1 = (tiles + n_sms - 1) / n_sms, w2 = (2 * tiles + n_sms - 1) / n_sms;
  return double(w2) * 0.5 * GM_SPLIT_COST < double(w1) ? 2 : 1;
}

// C = A[M, K] . B[N, K]^T; A, B fp16 K-major (16-byte aligned, K % 64 == 0).
cudaError_t launch_gemm_f16(const uint16_t* A, const uint16_t* B, int M, int N, int K, int epi, void* out, int ldo,
                            const float* row_scale, uint32_t* err, int n_sms, cudaStream_t st, int nx_count,
                            const uint8_t* const* nx_blob, const int64_t* nx_n, const int64_t* nx_k, int nx_fmt,
                            uint16_t* const* nx_out) {
  CUtensorMap ma;
  const cudaError_t e = make_map(&ma, A, M, K, GM_BM);
  if (e != cudaSuccess) return e;
  GemmArgs g;
  g.M = M;
  g.N = N;
  g.K = K;
  g.epi = epi;
  g.ldo = ldo;
  g.out = out;
  g.row_scale = row_scale;
  g.err = err;
  if (nx_count < 0 || nx_count > 3) return cudaErrorInvalidValue;
  g.nx_count = nx_count;
  g.nx_fmt = nx_fmt;
  for (int i = 0; i < 3; ++i) {
    g.nx_blob[i] = i < nx_count ? nx_blob[i] : nullptr;
    g.nx_n[i] = i < nx_count ? nx_n[i] : 0;
    g.nx_k[i] = i < nx_count ? nx_k[i] : 0;
    g.nx_out[i] = i < nx_count ? nx_out[i] : nullptr;
  }
  const int bn = gemm_tile_width(M, N, n_sms);
  g.ksplit = gemm_ksplit(M, N, K, bn, epi, n_sms);
  if (g.ksplit > 1) {
    const cudaError_t z = cudaMemset2DAsync(out, (size_t)ldo * 4, 0, (size_t)N * 4, (size_t)M, st);
    if (z != cudaSuccess) return z;
  }
  if (bn == 128) return launch_gemm_tile<128>(ma, B, M, N, K, g, n_sms, st);
  return launch_gemm_tile<256>(ma, B, M, N, K, g, n_sms, st);
}

cudaError_t launch_flash_prefill(const uint16_t* q, const uint16_t* kc, const uint16_t* vc, const uint16_t* kn,
                                 const uint16_t* vn, uint16_t* out, int T, int nq, int nkv, int hd, int slots,
                                 int window, int start, int seq, uint32_t* err, cudaStream_t st) {
  FaArgs a;
  a.q = q;
  a.kc = kc;
  a.vc = vc;
  a.kn = kn;
  a.vn = vn;
  a.out = out;
  a.T = T;
  a.nq = nq;
  a.nkv = nkv;
  a.slots = slots;
  a.window = window;
  a.start = start;
  a.seq = seq;
  a.scale_log2 = float(1.4426950408889634 / sqrt(double(hd)));
  a.err = err;
  if (hd == 128) return launch_flash_tc(q, kc, vc, kn, vn, out, T, nq, nkv, slots, window, start, seq, err, st);
  const dim3 grid((T + FA_BQ - 1) / FA_BQ, nq);
  const int smem = 4 * FA_BK * hd * 2;
  flash_prefill_kernel<64><<<grid, FA_THREADS, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_embed_rows(const int32_t* tokens, int T, const uint16_t* embed, int vocab, int d, float* X,
                              uint16_t* X16, float* scale, uint32_t* err, cudaStream_t st) {
  embed_rows_kernel<<<T, RT, 0, st>>>(tokens, embed, vocab, d, X, X16, scale, err);
  return cudaGetLastError();
}

cudaError_t launch_resid_rows(const float* V, const float* gain, int T, int d, float eps, float* X, uint16_t* X16,
                              float* scale, cudaStream_t st) {
  resid_rows_kernel<<<T, RT, 0, st>>>(V, gain, d, eps, X, X16, scale);
  return cudaGetLastError();
}

cudaError_t launch_final_row(const float* x, const float* gain, int d, float eps, uint16_t* xb, cudaStream_t st) {
  final_row_kernel<<<1, RT, 0, st>>>(x, gain, d, eps, xb);
  return cudaGetLastError();
}

// counter: one int of device memory, reset here.
cudaError_t launch_head_gemv(const uint8_t* W, int n, int k, const uint16_t* xb, float* out, int* counter, int n_sms,
                             cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(counter, 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)k * 2;
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(head_gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
  }
  head_gemv_kernel<<<2 * n_sms, HG_THREADS, smem, st>>>(W, n, k, xb, out, counter);
  return cudaGetLastError();
}

cudaError_t launch_qk_rows(const float* Y, const float* qg, const float* kg, uint16_t* q16, uint16_t* kn,
                           uint16_t* vn, const double* f, float ms, float eps, int T, int nq, int nkv, int hd,
                           int start, cudaStream_t st) {
  QkArgs a;
  a.Y = Y;
  a.qg = qg;
  a.kg = kg;
  a.q16 = q16;
  a.kn = kn;
  a.vn = vn;
  for (int i = 0; i < 64; ++i) a.f[i] = f[i];
  a.ms = ms;
  a.eps = eps;
  a.T = T;
  a.nq = nq;
  a.nkv = nkv;
  a.hd = hd;
  a.start = start;
  qk_rows_kernel<<<T, RT, 0, st>>>(a);
  return cudaGetLastError();
}

// Append the prompt's last rows to the cache: all of them on a full layer,
// the last `window` on a ring (the ones it keeps).
cudaError_t launch_kv_append(uint16_t* kc, uint16_t* vc, const uint16_t* kn, const uint16_t* vn, int nkv, int hd,
                             int slots, int window, int seq, int start, int T, cudaStream_t st) {
  const int t0 = (window && T > window) ? T - window : 0;
  const int64_t total = (int64_t)nkv * (T - t0) * (hd / 8);
  kv_append_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(kc, vc, kn, vn, nkv, hd, slots, window, seq,
                                                                     start, T, t0);
  return cudaGetLastError();
}

}  // namespace w4a
