// Temperature / top-p (nucleus) sampling of one token per row of logits, with
// the uniform draw u of each row given (ATLAS-OLMo-3-32B-Think-v4 model card,
// "Benchmarks" and "Prompting guide for Think models": temperature 0.6,
// top-p 0.95; nucleus sampling as published by Holtzman et al., 2019).
//
// One CTA per row.  Tokens are ordered by logit, largest first, equal logits
// by the lower index (the order of their probabilities).  With
// e_i = exp((z_i - max z) / T) in fp64 and Z = sum e_i:
//  1. the nucleus is the shortest prefix of that order whose mass reaches
//     top_p * Z: the largest logit key t with mass(key >= t) >= top_p Z is
//     found by bisection over the 32-bit order-preserving keys of the fp32
//     logits, and the first k tokens of key t (by index) complete the prefix;
//  2. the drawn token is the first of the nucleus whose cumulative mass
//     exceeds u * M (M = the nucleus mass): again the largest key s whose
//     nucleus mass from the top through s exceeds u M, then the j-th token of
//     key s by index.
// Every mass is a fixed-order sum (per thread, then a shuffle tree, then the
// warps in order), so the result does not depend on scheduling.
#include <math.h>
#include <stdint.h>

#include "w4a_internal.h"

namespace w4a {

namespace {

constexpr int ST = 1024;  // threads per row
constexpr int SW = ST / 32;

__device__ __forceinline__ uint32_t zkey(float z) {
  const uint32_t u = __float_as_uint(z + 0.0f);  // -0 and +0 are one logit
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // ascending with z
}
__device__ __forceinline__ float key_z(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Block-wide sum of one double per thread in a fixed order.
__device__ double block_sum(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();  // red is free again
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double s = lane < SW ? red[lane] : 0.0;
  if (warp == 0) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) red[SW] = s;
  }
  __syncthreads();
  return red[SW];
}

__device__ int block_sum_int(int v, int* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  int s = lane < SW ? red[lane] : 0;
  if (warp == 0) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) red[SW] = s;
  }
  __syncthreads();
  return red[SW];
}

// mass of the tokens whose key is at least x
__device__ double mass_ge(const float* z, const double* e, int V, uint32_t x, double* red) {
  double s = 0.0;
  for (int i = threadIdx.x; i < V; i += ST)
    if (zkey(z[i]) >= x) s += e[i];
  return block_sum(s, red);
}

// index of the j-th (1-based) token of key x, by index
__device__ int nth_of_key(const float* z, int V, uint32_t x, int j, int* ired, int* out) {
  const int chunk = (V + ST - 1) / ST, i0 = threadIdx.x * chunk, i1 = min(V, i0 + chunk);
  int c = 0;
  for (int i = i0; i < i1; ++i) c += zkey(z[i]) == x;
  // exclusive prefix over threads, in thread order
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  __syncthreads();
  if (lane == 31) ired[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < SW ? ired[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += t;
    }
    if (lane < SW) ired[lane] = w;  // inclusive totals per warp
  }
  __syncthreads();
  const int before = (warp ? ired[warp - 1] : 0) + incl - c;
  if (j > before && j <= before + c) {
    int seen = before;
    for (int i = i0; i < i1; ++i)
      if (zkey(z[i]) == x && ++seen == j) {
        *out = i;
        break;
      }
  }
  __syncthreads();
  return *out;
}

__global__ void __launch_bounds__(ST, 1) sample_kernel(const float* __restrict__ logits, int V, float temperature,
                                                        float top_p, const float* __restrict__ u,
                                                        int32_t* __restrict__ tokens, double* __restrict__ ebuf) {
  __shared__ double red[SW + 1];
  __shared__ int ired[SW + 1];
  __shared__ float fred[SW];
  __shared__ int found;
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* z = logits + (size_t)row * V;
  double* e = ebuf + (size_t)row * V;
  if (tid == 0) found = 0;
  // the largest and smallest logits (their keys bound the searches)
  float mx = -INFINITY, mn = INFINITY;
  for (int i = tid; i < V; i += ST) {
    mx = fmaxf(mx, z[i]);
    mn = fminf(mn, z[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  if (lane == 0) fred[warp] = mx;
  __syncthreads();
  float m = -INFINITY;
  for (int w = 0; w < SW; ++w) m = fmaxf(m, fred[w]);
  __syncthreads();
  if (lane == 0) fred[warp] = mn;
  __syncthreads();
  float lo_z = INFINITY;
  for (int w = 0; w < SW; ++w) lo_z = fminf(lo_z, fred[w]);
  // unnormalized probabilities
  const double invT = 1.0 / double(temperature);
  double zs = 0.0;
  for (int i = tid; i < V; i += ST) {
    const double v = exp((double(z[i]) - double(m)) * invT);
    e[i] = v;
    zs += v;
  }
  __syncthreads();
  const double Z = block_sum(zs, red);
  // 1. the nucleus: largest key t with mass(key >= t) >= top_p Z
  const double need = double(top_p) * Z;
  uint64_t lo = zkey(lo_z), hi = uint64_t(zkey(m)) + 1;  // mass_ge(lo) = Z >= need; mass_ge(hi) = 0
  while (hi - lo > 1) {
    const uint64_t mid = lo + (hi - lo) / 2;
    if (mass_ge(z, e, V, uint32_t(mid), red) >= need) lo = mid;
    else hi = mid;
  }
  const uint32_t t = uint32_t(lo);
  const double A = t == 0xffffffffu ? 0.0 : mass_ge(z, e, V, t + 1, red);
  int nt_local = 0;
  for (int i = tid; i < V; i += ST) nt_local += zkey(z[i]) == t;
  const int nt = block_sum_int(nt_local, ired);
  // the tokens of key t share one logit, hence one e (the same expression)
  const double et = exp((double(key_z(t)) - double(m)) * invT);
  int k = nt;
  if (et > 0.0) {
    const double kk = ceil((need - A) / et);
    k = kk < 1.0 ? 1 : (kk > double(nt) ? nt : int(kk));
  }
  const double M = A + double(k) * et;
  // 2. the draw: largest key s whose nucleus mass from the top through s
  // exceeds u M (every key above t: mass_ge; t itself: M)
  const double target = double(u[row]) * M;
  lo = t;
  hi = uint64_t(zkey(m)) + 1;
  while (hi - lo > 1) {
    const uint64_t mid = lo + (hi - lo) / 2;
    if (mass_ge(z, e, V, uint32_t(mid), red) > target) lo = mid;
    else hi = mid;
  }
  const uint32_t s = uint32_t(lo);
  const double above = s == 0xffffffffu ? 0.0 : mass_ge(z, e, V, s + 1, red);
  int ns_local = 0;
  for (int i = tid; i < V; i += ST) ns_local += zkey(z[i]) == s;
  int ns = block_sum_int(ns_local, ired);
  const double es = exp((double(key_z(s)) - double(m)) * invT);
  if (s == t) ns = k;  // only the first k tokens of key t are in the nucleus
  int j = 1;
  if (es > 0.0) {
    const double jj = floor((target - above) / es) + 1.0;
    j = jj < 1.0 ? 1 : (jj > double(ns) ? ns : int(jj));
  }
  const int tok = nth_of_key(z, V, s, j, ired, &found);
  if (tid == 0) tokens[row] = tok;
}

}  // namespace

cudaError_t launch_sample(const float* logits, int batch, int vocab, float temperature, float top_p, const float* u,
                          int32_t* tokens, double* ebuf, cudaStream_t st) {
  sample_kernel<<<batch, ST, 0, st>>>(logits, vocab, temperature, top_p, u, tokens, ebuf);
  return cudaGetLastError();
}

}  // namespace w4a
