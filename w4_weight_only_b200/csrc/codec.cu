// int4 codec (quantize + pack, unpack), kernel-layout tiling, KV-cache row
// copies and the standalone QK-norm/rotation/append step.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "ptx.cuh"
#include "w4a_internal.h"

namespace w4a {

// ---- quantize + canonical pack: one warp per (row, 128-group) --------------
// Source: ATLAS-OLMo-3-32B-Think-v4 model card, "Quantization recipe" (packing
// order); round-to-nearest asymmetric min/max in IEEE fp32 (see include/w4a.h).
__global__ void pack_kernel(const void* __restrict__ W, int w_dtype, int64_t n, int64_t k,
                            uint32_t* __restrict__ qweight, uint16_t* __restrict__ scales,
                            uint32_t* __restrict__ qzeros) {
  const int64_t ngroups = k / GROUP;
  const int64_t gw = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (gw >= n * ngroups) return;
  const int64_t row = gw / ngroups, gi = gw - row * ngroups;
  const int64_t base = row * k + gi * GROUP + lane * 4;
  float v[4];
  if (w_dtype == W4A_F32) {
    const float4 f = *reinterpret_cast<const float4*>(static_cast<const float*>(W) + base);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
  } else {
    const uint2 h = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(W) + base);
    v[0] = bf16_to_f32(uint16_t(h.x & 0xffffu));
    v[1] = bf16_to_f32(uint16_t(h.x >> 16));
    v[2] = bf16_to_f32(uint16_t(h.y & 0xffffu));
    v[3] = bf16_to_f32(uint16_t(h.y >> 16));
  }
  float mn = fminf(fminf(v[0], v[1]), fminf(v[2], v[3]));
  float mx = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const float s32 = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
  __half sh = __float2half_rn(s32);
  uint16_t sbits = __half_as_ushort(sh);
  if ((sbits & 0x7fffu) == 0x7c00u) sbits = 0x7bffu;   // overflow -> 65504
  if ((sbits & 0x7fffu) == 0u) sbits = 0x0001u;       // zero -> 2^-24
  const float s = __half2float(__ushort_as_half(sbits));
  const float zf = fminf(fmaxf(rintf(__fdiv_rn(-mn, s)), 0.f), 15.f);
  const int z = int(zf);
  uint32_t nib = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float q = rintf(__fdiv_rn(v[e], s)) + zf;
    q = fminf(fmaxf(q, 0.f), 15.f);
    nib |= uint32_t(q) << (4 * e);
  }
  // lanes 2j and 2j+1 share word j of the group (k = 8j .. 8j+7)
  const uint32_t other = __shfl_down_sync(0xffffffffu, nib, 1);
  if ((lane & 1) == 0) qweight[row * (k / 8) + gi * 16 + lane / 2] = nib | (other << 16);
  if (lane == 0) {
    scales[gi * n + row] = sbits;
    atomicOr(qzeros + gi * (n / 8) + row / 8, uint32_t(z) << (4 * (row % 8)));
  }
}

// ---- tiled layout helpers ------------------------------------------------------
// Tiled row r -> canonical row (row_interleave: even rows from the first half,
// odd rows from the second half).
__host__ __device__ inline int64_t canon_row(int64_t r, int64_t n, int interleave) {
  if (!interleave) return r;
  return (r & 1) ? (n / 2 + r / 2) : (r / 2);
}

__device__ inline uint32_t canon_code(const uint32_t* qw, int64_t k, int64_t row, int64_t col) {
  return (qw[row * (k / 8) + col / 8] >> (4 * (col % 8))) & 15u;
}

// Column order inside a unit.  Each 32-column slice is split in four runs of
// eight, one per thread-in-quad t; the run of quad t feeds k-steps 2m (first
// four columns) and 2m+1 (last four) of the m16n8k16 products, so the
// activation fragments of a thread are 16 contiguous bytes of x.  Fragment
// register a0 holds (row g, columns c, c+1), a1 (row g+8, c, c+1), a2 (row g,
// c+2, c+3), a3 (row g+8, c+2, c+3) with c = 32m + 8t + 4e for k-step 2m+e.
__host__ __device__ inline int64_t unit_col(int s, int t, int j) {
  const int m = s >> 1, e = s & 1;
  return 32 * m + 8 * t + 4 * e + j;  // j = 0..3: columns of a0/a1 (j < 2) and a2/a3 (j >= 2)
}

// One thread per 32-bit word of int4 codes in the tiled layout.
__global__ void tile_codes_kernel(const uint32_t* __restrict__ qw, int64_t n, int64_t k, int interleave,
                                  uint8_t* __restrict__ out) {
  const int64_t nkc = k / W4_KC;
  const int64_t total = (n / RB) * nkc * (W4_KC / 16) * 32;
  const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= total) return;
  const int lane = int(id % 32);
  const int s = int((id / 32) % (W4_KC / 16));
  const int64_t unit = id / (32 * (W4_KC / 16));
  const int64_t rb = unit / nkc, kc = unit % nkc;
  const int g = lane >> 2, t = lane & 3;
  const int64_t r0 = canon_row(rb * RB + g, n, interleave), r1 = canon_row(rb * RB + g + 8, n, interleave);
  // nibble j of the word: row (j & 1 ? g + 8 : g), column unit_col(.., (j & 2 ? 2 : 0) + (j & 4 ? 1 : 0))
  uint32_t w = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int64_t row = (j & 1) ? r1 : r0;
    const int64_t col = kc * W4_KC + unit_col(s, t, ((j & 2) ? 2 : 0) + ((j & 4) ? 1 : 0));
    w |= canon_code(qw, k, row, col) << (4 * j);
  }
  uint8_t* u = out + unit * W4_UNIT;
  reinterpret_cast<uint32_t*>(u + ((s >> 2) * 32 + lane) * 16)[s & 3] = w;
}

// One thread per (unit, group, tiled row in the 16-row block): scale and zero.
__global__ void tile_meta_kernel(const uint16_t* __restrict__ sc, const uint32_t* __restrict__ qz, int64_t n,
                                 int64_t k, int interleave, uint8_t* __restrict__ out) {
  const int64_t nkc = k / W4_KC;
  const int64_t total = (n / RB) * nkc * 4 * RB;
  const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= total) return;
  const int i = int(id % RB);
  const int grp = int((id / RB) % 4);
  const int64_t unit = id / (4 * RB);
  const int64_t rb = unit / nkc, kc = unit % nkc;
  const int64_t gi = kc * 4 + grp;
  const int64_t row = canon_row(rb * RB + i, n, interleave);
  uint8_t* u = out + unit * W4_UNIT;
  // scales ordered [row % 8][group][row / 8]: a thread's eight scales are 16 contiguous bytes
  reinterpret_cast<uint16_t*>(u + 4096)[(i & 7) * 8 + grp * 2 + (i >> 3)] = sc[gi * n + row];
  if ((i & 7) == 0) {
    uint32_t zw = 0;
    for (int j = 0; j < 8; ++j) {
      const int64_t rj = canon_row(rb * RB + i + j, n, interleave);
      zw |= ((qz[gi * (n / 8) + rj / 8] >> (4 * (rj % 8))) & 15u) << (4 * j);
    }
    reinterpret_cast<uint32_t*>(u + 4224)[grp * 2 + (i >> 3)] = zw;
  }
}

// bf16 [n, k] -> 16-row x 128-column units of mma A fragments (rows >= n are zero).
__global__ void tile_bf16_kernel(const uint16_t* __restrict__ W, int64_t n, int64_t k, uint8_t* __restrict__ out) {
  const int64_t nkc = k / BF_KC;
  const int64_t nrb = (n + RB - 1) / RB;
  const int64_t total = nrb * nkc * 8 * 32;
  const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= total) return;
  const int lane = int(id % 32);
  const int64_t s = (id / 32) % 8;
  const int64_t unit = id / 256;
  const int64_t rb = unit / nkc, kc = unit % nkc;
  const int g = lane >> 2, t = lane & 3;
  const int64_t r0 = rb * RB + g, r1 = r0 + 8;
  const int64_t k0 = kc * BF_KC + unit_col(int(s), t, 0);
  auto pair = [&](int64_t r, int64_t c) -> uint32_t {
    if (r >= n) return 0u;
    return uint32_t(W[r * k + c]) | (uint32_t(W[r * k + c + 1]) << 16);
  };
  uint4 v;
  v.x = pair(r0, k0);
  v.y = pair(r1, k0);
  v.z = pair(r0, k0 + 2);
  v.w = pair(r1, k0 + 2);
  reinterpret_cast<uint4*>(out + unit * BF_UNIT)[s * 32 + lane] = v;
}

// Exact dequantization to fp32 [n, k], canonical or tiled.
__global__ void unpack_kernel(const uint32_t* __restrict__ qw, const uint16_t* __restrict__ sc,
                              const uint32_t* __restrict__ qz, const uint8_t* __restrict__ tiled, int64_t n,
                              int64_t k, int interleave, float* __restrict__ out) {
  const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= n * k) return;
  const int64_t row = id / k, col = id - row * k;
  uint32_t q, z;
  uint16_t sb;
  if (tiled == nullptr) {
    q = canon_code(qw, k, row, col);
    sb = sc[(col / GROUP) * n + row];
    z = (qz[(col / GROUP) * (n / 8) + row / 8] >> (4 * (row % 8))) & 15u;
  } else {
    int64_t r = row;
    if (interleave) r = (row < n / 2) ? 2 * row : 2 * (row - n / 2) + 1;
    const int64_t rb = r / RB;
    const int i = int(r % RB), g = i & 7, hi = i >> 3;
    const int64_t nkc = k / W4_KC, kc = col / W4_KC;
    const int kk = int(col % W4_KC);
    // inverse of unit_col: column kk = 32 m + 8 t + 4 e + j
    const int m = kk / 32, t = (kk % 32) / 8, e = (kk % 8) / 4, j = kk % 4;
    const int s = 2 * m + e;
    const int lane = g * 4 + t;
    const int nib = ((j & 1) ? 4 : 0) + ((j & 2) ? 2 : 0) + hi;
    const uint8_t* u = tiled + (rb * nkc + kc) * W4_UNIT;
    const uint32_t w = reinterpret_cast<const uint32_t*>(u + ((s >> 2) * 32 + lane) * 16)[s & 3];
    q = (w >> (4 * nib)) & 15u;
    const int grp = kk / GROUP;
    sb = reinterpret_cast<const uint16_t*>(u + 4096)[g * 8 + grp * 2 + hi];
    z = (reinterpret_cast<const uint32_t*>(u + 4224)[grp * 2 + hi] >> (4 * g)) & 15u;
  }
  out[id] = float(int(q) - int(z)) * half_bits_to_f32(sb);
}

// ---- KV rows: logical [n_kv, n, hd] <-> chunk-permuted cache slots ------------
__global__ void kv_copy_kernel(uint16_t* __restrict__ cache, const uint16_t* __restrict__ src, int nkv, int hd,
                               int slots, int b, int slot0, int n, int to_cache) {
  const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= (int64_t)nkv * n * hd) return;
  const int d = int(id % hd);
  const int i = int((id / hd) % n);
  const int h = int(id / ((int64_t)hd * n));
  const int slot = slot0 + i;
  const int sw = (((d >> 3) ^ (slot & 7)) << 3) | (d & 7);
  const int64_t ci = (((int64_t)b * nkv + h) * slots + slot) * hd + sw;
  if (to_cache)
    cache[ci] = src[id];
  else
    const_cast<uint16_t*>(src)[id] = cache[ci];
}

// ---- standalone QK-norm + rotation + KV append: one CTA per sequence --------
struct RopeTab {
  double f[64];
  float ms;
};

__global__ void qk_prep_kernel(int nq, int nkv, int hd, float eps, const RopeTab rt,
                               const float* __restrict__ q_raw, const float* __restrict__ k_raw,
                               const float* __restrict__ v_raw, const float* __restrict__ q_gain,
                               const float* __restrict__ k_gain, const int32_t* __restrict__ pos,
                               uint16_t* __restrict__ q_out, uint16_t* __restrict__ k_cache,
                               uint16_t* __restrict__ v_cache, int slots) {
  __shared__ float red[2][32];
  const int b = blockIdx.x, tid = threadIdx.x;
  const int qd = nq * hd, kd = nkv * hd;
  const float* q = q_raw + (int64_t)b * qd;
  const float* kk = k_raw + (int64_t)b * kd;
  float sq = 0.f, sk = 0.f;
  for (int i = tid; i < qd; i += blockDim.x) sq = fmaf(q[i], q[i], sq);
  for (int i = tid; i < kd; i += blockDim.x) sk = fmaf(kk[i], kk[i], sk);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sq += __shfl_xor_sync(0xffffffffu, sq, o);
    sk += __shfl_xor_sync(0xffffffffu, sk, o);
  }
  if ((tid & 31) == 0) {
    red[0][tid >> 5] = sq;
    red[1][tid >> 5] = sk;
  }
  __syncthreads();
  if (tid == 0) {
    float a = 0.f, c = 0.f;
    for (int w = 0; w < int(blockDim.x / 32); ++w) {
      a += red[0][w];
      c += red[1][w];
    }
    red[0][0] = rsqrtf(a / float(qd) + eps);
    red[1][0] = rsqrtf(c / float(kd) + eps);
  }
  __syncthreads();
  const float rq = red[0][0], rk = red[1][0];
  const int p = pos[b];
  const int slot = p % slots;
  const int h2 = hd / 2;
  for (int idx = tid; idx < (nq + nkv) * h2; idx += blockDim.x) {
    const int head = idx / h2, i = idx - head * h2;
    double sn, cs;
    sincos(double(p) * rt.f[i], &sn, &cs);
    const float c = float(cs) * rt.ms, s = float(sn) * rt.ms;
    if (head < nq) {
      const int r = head * hd;
      const float x1 = q[r + i] * rq * q_gain[r + i], x2 = q[r + i + h2] * rq * q_gain[r + i + h2];
      q_out[(int64_t)b * qd + r + i] = f32_to_bf16(x1 * c - x2 * s);
      q_out[(int64_t)b * qd + r + i + h2] = f32_to_bf16(x2 * c + x1 * s);
    } else if (p >= 0) {
      const int g = head - nq, r = g * hd;
      const float x1 = kk[r + i] * rk * k_gain[r + i], x2 = kk[r + i + h2] * rk * k_gain[r + i + h2];
      const int64_t base = (((int64_t)b * nkv + g) * slots + slot) * hd;
      const int sw1 = (((i >> 3) ^ (slot & 7)) << 3) | (i & 7);
      const int sw2 = ((((i + h2) >> 3) ^ (slot & 7)) << 3) | ((i + h2) & 7);
      k_cache[base + sw1] = f32_to_bf16(x1 * c - x2 * s);
      k_cache[base + sw2] = f32_to_bf16(x2 * c + x1 * s);
      const float* vv = v_raw + (int64_t)b * kd + r;
      v_cache[base + sw1] = f32_to_bf16(vv[i]);
      v_cache[base + sw2] = f32_to_bf16(vv[i + h2]);
    }
  }
}

// ---- the symmetric group-32 checkpoint format ----------------------------------
// Canonical: qweight uint32 [n, k/8] with column j in word j/8, nibble j % 8
// holding q + 8; scales bf16 [n, k/32] (row-major, one per output row and
// 32-column group).  w = (nibble - 8) * s.  Tiled: 16-row x 256-column units
// of S32_UNIT bytes, codes as in the int4 unit (fragment order, the same
// in-unit column permutation), then the scales [row % 8][group 8][row / 8].

// One thread per 32-bit word of codes in the tiled layout.
__global__ void tile_s32_codes_kernel(const uint32_t* __restrict__ qw, int64_t n, int64_t k, int interleave,
                                      uint8_t* __restrict__ out) {
  const int64_t nkc = k / S32_KC;
  const int64_t total = (n / RB) * nkc * (S32_KC / 16) * 32;
  const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= total) return;
  const int lane = int(id % 32);
  const int s = int((id / 32) % (S32_KC / 16));
  const int64_t unit = id / (32 * (S32_KC / 16));
  const int64_t rb = unit / nkc, kc = unit % nkc;
  const int g = lane >> 2, t = lane & 3;
  const int64_t r0 = canon_row(rb * RB + g, n, interleave), r1 = canon_row(rb * RB + g + 8, n, interleave);
  uint32_t w = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int64_t row = (j & 1) ? r1 : r0;
    const int64_t col = kc * S32_KC + unit_col(s, t, ((j & 2) ? 2 : 0) + ((j & 4) ? 1 : 0));
    w |= canon_code(qw, k, row, col) << (4 * j);
  }
  uint8_t* u = out + unit * S32_UNIT;
  reinterpret_cast<uint32_t*>(u + ((s >> 2) * 32 + lane) * 16)[s & 3] = w;
}

// One thread per (unit, 32-column group, tiled row of the block): its scale.
__global__ void tile_s32_meta_kernel(const uint16_t* __restrict__ sc, int64_t n, int64_t k, int interleave,
                                     uint8_t* __restrict__ out) {
  const int64_t nkc = k / S32_KC;
  const int64_t total = (n / RB) * nkc * 8 * RB;
  const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= total) return;
  const int i = int(id % RB);
  const int grp = int((id / RB) % 8);
  const int64_t unit = id / (8 * RB);
  const int64_t rb = unit / nkc, kc = unit % nkc;
  const int64_t row = canon_row(rb * RB + i, n, interleave);
  const int64_t gi = kc * 8 + grp;  // 32-column group along k
  reinterpret_cast<uint16_t*>(out + unit * S32_UNIT + 2048)[(i & 7) * 16 + grp * 2 + (i >> 3)] =
      sc[row * (k / S32_GROUP) + gi];
}

// Exact dequantization of the symmetric group-32 format to fp32 [n, k],
// canonical (tiled == nullptr) or tiled.
__global__ void unpack_s32_kernel(const uint32_t* __restrict__ qw, const uint16_t* __restrict__ sc,
                                  const uint8_t* __restrict__ tiled, int64_t n, int64_t k, int interleave,
                                  float* __restrict__ out) {
  const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= n * k) return;
  const int64_t row = id / k, col = id - row * k;
  uint32_t q;
  uint16_t sb;
  if (tiled == nullptr) {
    q = canon_code(qw, k, row, col);
    sb = sc[row * (k / S32_GROUP) + col / S32_GROUP];
  } else {
    int64_t r = row;
    if (interleave) r = (row < n / 2) ? 2 * row : 2 * (row - n / 2) + 1;
    const int64_t rb = r / RB;
    const int i = int(r % RB), g = i & 7, hi = i >> 3;
    const int64_t nkc = k / S32_KC, kc = col / S32_KC;
    const int kk = int(col % S32_KC);
    const int m = kk / 32, t = (kk % 32) / 8, e = (kk % 8) / 4, j = kk % 4;
    const int s = 2 * m + e;
    const int lane = g * 4 + t;
    const int nib = ((j & 1) ? 4 : 0) + ((j & 2) ? 2 : 0) + hi;
    const uint8_t* u = tiled + (rb * nkc + kc) * S32_UNIT;
    const uint32_t w = reinterpret_cast<const uint32_t*>(u + ((s >> 2) * 32 + lane) * 16)[s & 3];
    q = (w >> (4 * nib)) & 15u;
    sb = reinterpret_cast<const uint16_t*>(u + 2048)[g * 16 + m * 2 + hi];
  }
  out[id] = float(int(q) - 8) * bf16_to_f32(sb);
}

// ---- launchers (called from api.cu) ------------------------------------------
cudaError_t launch_tile_s32(const uint32_t* qw, const uint16_t* sc, int64_t n, int64_t k, int interleave,
                            uint8_t* out, cudaStream_t st) {
  const int64_t nw = (n / RB) * (k / S32_KC) * (S32_KC / 16) * 32;
  tile_s32_codes_kernel<<<(unsigned)((nw + 255) / 256), 256, 0, st>>>(qw, n, k, interleave, out);
  const int64_t nm = (n / RB) * (k / S32_KC) * 8 * RB;
  tile_s32_meta_kernel<<<(unsigned)((nm + 255) / 256), 256, 0, st>>>(sc, n, k, interleave, out);
  return cudaGetLastError();
}

cudaError_t launch_unpack_s32(const uint32_t* qw, const uint16_t* sc, const uint8_t* tiled, int64_t n, int64_t k,
                              int interleave, float* out, cudaStream_t st) {
  const int64_t total = n * k;
  unpack_s32_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(qw, sc, tiled, n, k, interleave, out);
  return cudaGetLastError();
}

// ---- launchers (called from api.cu) ------------------------------------------
cudaError_t launch_pack(const void* W, int w_dtype, int64_t n, int64_t k, uint32_t* qw, uint16_t* sc, uint32_t* qz,
                        cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(qz, 0, (size_t)(k / GROUP) * (n / 8) * 4, st);
  if (e != cudaSuccess) return e;
  const int64_t warps = n * (k / GROUP);
  const int per = 8;
  pack_kernel<<<(unsigned)((warps + per - 1) / per), per * 32, 0, st>>>(W, w_dtype, n, k, qw, sc, qz);
  return cudaGetLastError();
}

cudaError_t launch_tile(const uint32_t* qw, const uint16_t* sc, const uint32_t* qz, int64_t n, int64_t k,
                        int interleave, uint8_t* out, cudaStream_t st) {
  const int64_t nw = (n / RB) * (k / W4_KC) * (W4_KC / 16) * 32;
  tile_codes_kernel<<<(unsigned)((nw + 255) / 256), 256, 0, st>>>(qw, n, k, interleave, out);
  const int64_t nm = (n / RB) * (k / W4_KC) * 4 * RB;
  tile_meta_kernel<<<(unsigned)((nm + 255) / 256), 256, 0, st>>>(sc, qz, n, k, interleave, out);
  return cudaGetLastError();
}

cudaError_t launch_tile_bf16(const uint16_t* W, int64_t n, int64_t k, uint8_t* out, cudaStream_t st) {
  const int64_t total = ((n + RB - 1) / RB) * (k / BF_KC) * 256;
  tile_bf16_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(W, n, k, out);
  return cudaGetLastError();
}

cudaError_t launch_unpack(const uint32_t* qw, const uint16_t* sc, const uint32_t* qz, const uint8_t* tiled, int64_t n,
                          int64_t k, int interleave, float* out, cudaStream_t st) {
  const int64_t total = n * k;
  unpack_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(qw, sc, qz, tiled, n, k, interleave, out);
  return cudaGetLastError();
}

cudaError_t launch_kv_copy(uint16_t* cache, const uint16_t* src, int nkv, int hd, int slots, int b, int slot0, int n,
                           int to_cache, cudaStream_t st) {
  const int64_t total = (int64_t)nkv * n * hd;
  if (total == 0) return cudaSuccess;
  kv_copy_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(cache, src, nkv, hd, slots, b, slot0, n, to_cache);
  return cudaGetLastError();
}

cudaError_t launch_qk_prep(int batch, int nq, int nkv, int hd, float eps, const double* inv_freq, float ms,
                           const float* q_raw, const float* k_raw, const float* v_raw, const float* q_gain,
                           const float* k_gain, const int32_t* pos, uint16_t* q_out, uint16_t* k_cache,
                           uint16_t* v_cache, int slots, cudaStream_t st) {
  RopeTab rt;
  for (int i = 0; i < 64; ++i) rt.f[i] = (i < hd / 2) ? inv_freq[i] : 0.0;
  rt.ms = ms;
  qk_prep_kernel<<<batch, 256, 0, st>>>(nq, nkv, hd, eps, rt, q_raw, k_raw, v_raw, q_gain, k_gain, pos, q_out,
                                         k_cache, v_cache, slots);
  return cudaGetLastError();
}

}  // namespace w4a
