// Temperature / top-p (nucleus) sampling of one token per row of logits, with
// the uniform draw u of each row given (ATLAS-OLMo-3-32B-Think-v4 model card,
// "Benchmarks" and "Prompting guide for Think models": temperature 0.6,
// top-p 0.95; nucleus sampling as published by Holtzman et al., 2019).
//
// Tokens are ordered by logit, largest first, equal logits by the lower index
// (the order of their probabilities).  Each token's weight
// e_i = exp((z_i - max z) / T) is evaluated in fp64 and held as a 64-bit
// fixed-point integer E_i = round(e_i 2^F), F = 63 - ceil(log2 V), so that
// any sum of them fits 64 bits and is exact: sums in any order give the same
// bits.  With Z = sum E_i:
//  1. the nucleus is the shortest prefix of that order whose mass reaches
//     need = top_p Z: the largest 32-bit order-preserving logit key t with
//     mass(key >= t) >= need, found by radix selection, eight bits of the key
//     per pass (a 256-bin histogram of masses per pass, bins taken from the
//     top until the mass reaches need); then the first k tokens of key t (by
//     index) complete the prefix, k = ceil((need - mass(key > t)) / E_t);
//  2. the drawn token is the first of the nucleus whose cumulative mass
//     exceeds target = floor(u M) (M = the nucleus mass): the largest key s
//     whose nucleus mass from the top through s exceeds target (again radix
//     selection, over the keys above t, or s = t), then the j-th token of key
//     s by index.
// A row is spread over a cluster of CL CTAs, each holding a contiguous slice
// of the vocabulary; every per-row quantity (the maximum, Z, each pass's
// histogram, the count of a key before a slice) is exchanged through
// distributed shared memory, so every CTA takes the same decisions.
#include <cooperative_groups.h>
#include <math.h>
#include <stdint.h>

#include "w4a_internal.h"

namespace cg = cooperative_groups;

namespace w4a {

namespace {

constexpr int CL = 8;      // CTAs per row (one thread-block cluster)
constexpr int ST = 512;    // threads per CTA
constexpr int SW = ST / 32;
constexpr int DYN = SW * 256 * (8 + 4);  // per-warp histograms (dynamic shared memory)

__device__ __forceinline__ uint32_t zkey(float z) {
  const uint32_t u = __float_as_uint(z + 0.0f);  // -0 and +0 are one logit
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // ascending with z
}

struct Shared {
  // read by the other CTAs of the cluster; two slots, by exchange parity
  unsigned long long xmass[2][256];
  unsigned int xcount[2][256];
  unsigned long long xsum[2];
  float xmax[2];
  unsigned int xcnt[2];
  // this CTA's
  unsigned long long mass[256];  // the row's histogram of the current pass
  unsigned int count[256];
  unsigned long long red[SW];
  float fred[SW];
  int ired[SW + 1];
  unsigned long long above;      // mass of the keys above the current prefix range
  unsigned long long bin_mass;   // mass of the chosen bin
  unsigned int bin_count;
  uint32_t prefix;
  int found;
};

struct Row {
  const float* z;          // the row's logits
  unsigned long long* E;   // the row's fixed-point weights
  int v0, v1;              // this CTA's slice
  int ph;                  // exchanges so far (slot parity)
};

__device__ float block_max(float v, Shared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) sh.fred[warp] = v;
  __syncthreads();
  float m = -INFINITY;
#pragma unroll 1
  for (int w = 0; w < SW; ++w) m = fmaxf(m, sh.fred[w]);
  return m;
}

__device__ unsigned long long block_sum_u64(unsigned long long v, Shared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) sh.red[warp] = v;
  __syncthreads();
  unsigned long long s = 0;
#pragma unroll 1
  for (int w = 0; w < SW; ++w) s += sh.red[w];
  return s;
}

// One radix pass: the row's histogram (mass, count) by key byte `shift` of
// the tokens whose key bits above that byte equal `hi` (all tokens at the top
// byte) and whose key exceeds `floor_key` (all when floor_key < 0).  Lanes of
// a warp that hit one bin are added up first (match.any groups; the 64-bit
// weights in three 23-bit parts, so the 32-bit group sums cannot overflow),
// into the warp's own histogram (no atomics); the warps' histograms are
// summed into this CTA's exchange slot, the CTAs' slots into the row's
// histogram.  Then warp 0 takes bins from the top down: the first bin at
// which (above + masses so far) reaches `need` is chosen; the masses of the
// bins above it join `above`.
__device__ void radix_pass(cg::cluster_group& cl, Row& r, int shift, uint32_t hi, long long floor_key,
                           unsigned long long need, Shared& sh) {
  extern __shared__ unsigned long long wh[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long* hm = wh + warp * 256;
  unsigned int* hc = reinterpret_cast<unsigned int*>(wh + SW * 256) + warp * 256;
#pragma unroll
  for (int b = lane; b < 256; b += 32) {
    hm[b] = 0ull;
    hc[b] = 0u;
  }
  __syncwarp();
  const bool top = shift == 24;
#pragma unroll 1
  for (int i0 = r.v0 + warp * 32; i0 < r.v1; i0 += ST) {  // warp-uniform
    const int i = i0 + lane;
    bool ok = i < r.v1;
    const uint32_t k = ok ? zkey(r.z[i]) : 0u;
    if (ok && !top && (k >> (shift + 8)) != hi) ok = false;
    if (ok && (long long)k <= floor_key) ok = false;
    if (__ballot_sync(0xffffffffu, ok) == 0u) continue;
    const int b = ok ? int((k >> shift) & 255u) : 256;
    const unsigned long long e = ok ? r.E[i] : 0ull;
    const unsigned peers = __match_any_sync(0xffffffffu, b);
    const uint32_t p0 = __reduce_add_sync(peers, uint32_t(e & 0x7FFFFFull));
    const uint32_t p1 = __reduce_add_sync(peers, uint32_t((e >> 23) & 0x7FFFFFull));
    const uint32_t p2 = __reduce_add_sync(peers, uint32_t(e >> 46));
    if (ok && lane == __ffs(peers) - 1) {
      hm[b] += (unsigned long long)p0 + ((unsigned long long)p1 << 23) + ((unsigned long long)p2 << 46);
      hc[b] += (unsigned)__popc(peers);
    }
    __syncwarp();
  }
  __syncthreads();
  const int slot = r.ph & 1;
  if (threadIdx.x < 256) {
    const int b = threadIdx.x;
    unsigned long long m = 0;
    unsigned int c = 0;
#pragma unroll 4
    for (int w = 0; w < SW; ++w) {
      m += wh[w * 256 + b];
      c += reinterpret_cast<const unsigned int*>(wh + SW * 256)[w * 256 + b];
    }
    sh.xmass[slot][b] = m;
    sh.xcount[slot][b] = c;
  }
  cl.sync();
  if (threadIdx.x < 256) {
    const int b = threadIdx.x;
    unsigned long long m = 0;
    unsigned int c = 0;
#pragma unroll 1
    for (int q = 0; q < CL; ++q) {
      const Shared* o = cl.map_shared_rank(&sh, q);
      m += o->xmass[slot][b];
      c += o->xcount[slot][b];
    }
    sh.mass[b] = m;
    sh.count[b] = c;
  }
  ++r.ph;
  __syncthreads();
  if (threadIdx.x < 32) {
    // lane l holds bins 255 - 8 l .. 248 - 8 l (from the top)
    unsigned long long local = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) local += sh.mass[255 - 8 * lane - j];
    // inclusive sum over the lanes from the top (lower lane = higher bins)
    unsigned long long incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const unsigned long long base = sh.above, excl = incl - local;
    const unsigned mask = __ballot_sync(0xffffffffu, base + incl >= need);
    // the lane whose range reaches need (callers guarantee one does; else the
    // lowest non-empty bin is taken)
    const int first = mask ? __ffs(mask) - 1 : 31;
    if (lane == first) {
      unsigned long long cum = base + excl;
      int pick = -1;
#pragma unroll 1
      for (int j = 0; j < 8; ++j) {
        const int b = 255 - 8 * lane - j;
        if (sh.count[b] == 0u) continue;
        if (cum + sh.mass[b] >= need) {
          pick = b;
          break;
        }
        cum += sh.mass[b];
        pick = b;
      }
      if (pick < 0) {
        pick = 255 - 8 * lane;
      } else if (cum + sh.mass[pick] < need) {
        cum -= sh.mass[pick];  // not reached: the picked bin's mass is not above it
      }
      sh.above = cum;
      sh.bin_mass = sh.mass[pick];
      sh.bin_count = sh.count[pick];
      sh.prefix = (top ? 0u : (hi << 8)) | uint32_t(pick);
    }
  }
  __syncthreads();
}

// Largest key x (over the keys above floor_key) with mass(key >= x) >= need;
// returns x, and mass(key > x), the mass and count of key x in sh.
__device__ uint32_t radix_select(cg::cluster_group& cl, Row& r, long long floor_key, unsigned long long need,
                                 Shared& sh) {
  if (threadIdx.x == 0) sh.above = 0ull;
  __syncthreads();
  uint32_t hi = 0;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    radix_pass(cl, r, shift, hi, floor_key, need, sh);
    hi = sh.prefix;
  }
  return hi;
}

// The row's j-th (1-based) token of key x, by index: counts of the key in
// the slices before this one come from the other CTAs; the CTA holding the
// token finds it in its slice and returns it (-1 elsewhere).
__device__ int nth_of_key(cg::cluster_group& cl, Row& r, uint32_t x, int j, Shared& sh) {
  const int n = r.v1 - r.v0;
  const int chunk = (n + ST - 1) / ST;
  const int i0 = r.v0 + threadIdx.x * chunk, i1 = min(r.v1, i0 + chunk);
  int c = 0;
  for (int i = i0; i < i1; ++i) c += zkey(r.z[i]) == x;
  // exclusive prefix over threads, in thread order
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  __syncthreads();
  if (lane == 31) sh.ired[warp] = incl;
  if (threadIdx.x == 0) sh.found = -1;
  __syncthreads();
  if (warp == 0) {
    int w = lane < SW ? sh.ired[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += t;
    }
    if (lane < SW) sh.ired[lane] = w;  // inclusive totals per warp
  }
  __syncthreads();
  const int slot = r.ph & 1;
  if (threadIdx.x == 0) sh.xcnt[slot] = unsigned(sh.ired[SW - 1]);
  cl.sync();
  int before_cta = 0;
  const int rank = int(cl.block_rank());
#pragma unroll 1
  for (int q = 0; q < rank; ++q) before_cta += int(cl.map_shared_rank(&sh, q)->xcnt[slot]);
  ++r.ph;
  const int before = before_cta + (warp ? sh.ired[warp - 1] : 0) + incl - c;
  if (j > before && j <= before + c) {
    int seen = before;
    for (int i = i0; i < i1; ++i)
      if (zkey(r.z[i]) == x && ++seen == j) {
        sh.found = i;
        break;
      }
  }
  __syncthreads();
  return sh.found;
}

__global__ void __cluster_dims__(CL, 1, 1) __launch_bounds__(ST, 1)
    sample_kernel(const float* __restrict__ logits, int V, float temperature, float top_p,
                  const float* __restrict__ u, int32_t* __restrict__ tokens, unsigned long long* __restrict__ ebuf,
                  int fbits) {
  __shared__ Shared sh;
  cg::cluster_group cl = cg::this_cluster();
  const int row = int(blockIdx.x) / CL, rank = int(cl.block_rank());
  const int per = (V + CL - 1) / CL;
  Row r;
  r.z = logits + (size_t)row * V;
  r.E = ebuf + (size_t)row * V;
  r.v0 = min(V, rank * per);
  r.v1 = min(V, r.v0 + per);
  r.ph = 0;
  const int tid = threadIdx.x;
  // the largest logit of the row
  float mx = -INFINITY;
  for (int i = r.v0 + tid; i < r.v1; i += ST) mx = fmaxf(mx, r.z[i]);
  mx = block_max(mx, sh);
  if (tid == 0) sh.xmax[r.ph & 1] = mx;
  cl.sync();
  float m = -INFINITY;
#pragma unroll 1
  for (int q = 0; q < CL; ++q) m = fmaxf(m, cl.map_shared_rank(&sh, q)->xmax[r.ph & 1]);
  ++r.ph;
  // fixed-point weights of the slice, and Z
  const double invT = 1.0 / double(temperature);
  const double scale = ldexp(1.0, fbits);
  unsigned long long zs = 0;
  for (int i = r.v0 + tid; i < r.v1; i += ST) {
    const double e = exp((double(r.z[i]) - double(m)) * invT);
    const unsigned long long q = (unsigned long long)(e * scale + 0.5);
    r.E[i] = q;
    zs += q;
  }
  zs = block_sum_u64(zs, sh);
  if (tid == 0) sh.xsum[r.ph & 1] = zs;
  cl.sync();  // also orders this CTA's weights before its own reads below
  unsigned long long Z = 0;
#pragma unroll 1
  for (int q = 0; q < CL; ++q) Z += cl.map_shared_rank(&sh, q)->xsum[r.ph & 1];
  ++r.ph;
  // 1. the nucleus
  unsigned long long need = (unsigned long long)ceil(double(top_p) * double(Z));
  if (need > Z) need = Z;
  if (need < 1) need = 1;
  const uint32_t t = radix_select(cl, r, -1, need, sh);
  const unsigned long long A = sh.above;  // mass of the keys above t
  const unsigned long long mt = sh.bin_mass;
  const unsigned int nt = sh.bin_count;
  const unsigned long long et = nt ? mt / nt : 0ull;  // one logit, one weight
  unsigned long long k = nt;
  if (et > 0 && need > A) {
    k = (need - A + et - 1) / et;
    if (k < 1) k = 1;
    if (k > nt) k = nt;
  } else if (et > 0) {
    k = 1;
  }
  const unsigned long long M = A + k * et;
  // 2. the draw: first nucleus token whose cumulative mass exceeds target
  unsigned long long target = (unsigned long long)floor(double(u[row]) * double(M));
  if (M > 0 && target >= M) target = M - 1;
  uint32_t s = t;
  unsigned long long above_s = A, es = et, ns = k;
  if (target < A) {  // the same decision in every CTA of the cluster
    __syncthreads();
    s = radix_select(cl, r, (long long)t, target + 1, sh);
    above_s = sh.above;
    ns = sh.bin_count;
    es = ns ? sh.bin_mass / ns : 0ull;
  }
  unsigned long long j = 1;
  if (es > 0) {
    j = (target - above_s) / es + 1;
    if (j < 1) j = 1;
    if (j > ns) j = ns;
  }
  __syncthreads();
  const int tok = nth_of_key(cl, r, s, int(j), sh);
  if (tid == 0 && tok >= 0) tokens[row] = tok;
  cl.sync();  // no CTA leaves while another may still read its shared memory
}

}  // namespace

// Bits of the fixed-point weights for a row of V tokens: V e_i <= V < 2^63.
int sample_fbits(int vocab) {
  int lg = 0;
  while ((1ll << lg) < (long long)vocab) ++lg;
  return 63 - lg;
}

cudaError_t launch_sample(const float* logits, int batch, int vocab, float temperature, float top_p, const float* u,
                          int32_t* tokens, double* ebuf, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    const cudaError_t e = cudaFuncSetAttribute(sample_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DYN);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  sample_kernel<<<batch * CL, ST, DYN, st>>>(logits, vocab, temperature, top_p, u, tokens,
                                             reinterpret_cast<unsigned long long*>(ebuf), sample_fbits(vocab));
  return cudaGetLastError();
}

}  // namespace w4a
