// The persistent decode engine.
//
// One CTA per SM, 16 warps.  A launch runs a list of phases (decode: per layer
// QKV GEMV, GQA attention, O GEMV, gate/up GEMV, down GEMV; then lm_head and
// argmax) separated by grid-wide barriers.  Every warp streams its own
// contiguous range of 4 KB "units" (16 weight rows x 512 int4 columns, 16 rows
// x 128 bf16 columns, or 8 keys of K and V) from HBM into a two-slot ring of
// shared memory with bulk asynchronous copies completing on mbarriers.  The
// loader runs ahead across phase boundaries: weights and old KV entries do not
// depend on the activations, so the copies for phase p+1 are in flight while
// the CTA waits at the barrier that ends phase p.
//
// GEMV math: the int4 codes of a unit are laid out as mma.sync A fragments
// (16 rows x 16 k per warp-wide word).  A LOP3 turns each nibble q into the
// fp16 value 1024 + q (exact), the tensor core accumulates sum_k (1024+q) x_k
// in fp32 per 128-group, and the group is closed in fp32 with
// s * (acc - (1024 + z) * sum_k x_k).  x is the mma B operand (batch = n),
// held in fp16 (11-bit significand) after an exact power-of-two range
// scaling that is undone when a partial leaves the warp.  The bf16 lm_head
// takes bf16 x.
//
// Split-K is deterministic: pieces of one 16-row block computed by different
// warps are summed in warp order in shared memory, pieces from different
// CTAs are summed in CTA order by the last CTA to arrive (an atomic counter
// per row block, no waiting).
#pragma once
#include <float.h>
#include <math.h>

#include "ptx.cuh"
#include "w4a_internal.h"

namespace w4a {

constexpr long long WAIT_CYCLES = 4000000000LL;  // bound on any single wait (~2 s)
constexpr int MAX_SEG = MAX_B * 16;              // attention segments (batch x kv heads)

__host__ __device__ inline long long rstart(long long U, int n, int i) { return (U * i) / n; }
// CTA (of n) whose range [rstart(c), rstart(c+1)) contains unit u.
__host__ __device__ inline int owner(long long U, int n, long long u) {
  return int(((u + 1) * n + U - 1) / U) - 1;
}

// Units per slab (k-chunks) so that the x fragments a CTA needs fit in shared
// memory.  Returns 0 when no split fits.
__host__ __device__ inline int choose_kps(int nkc, int kcw, int B, int nb) {
  const int cap = xs_cap(nb);
  if (B * (nkc * kcw * 2 + 64) <= cap) return nkc;
  for (int dv = nkc - 1; dv >= 1; --dv)
    if (nkc % dv == 0 && 2 * B * (dv * kcw * 2 + 64) <= cap) return dv;
  return 0;
}

struct PD {
  int kind, layer;
  // GEMV
  const uint8_t* blob;
  int n, k, kcw, ub, nrb, nkc, kps, ns, nca;
  long long U;
  int xsrc;
  const uint16_t* xbf;
  int xbf_stride;
  const float* xres;
  const float* vres;
  const float* vss;
  int vnrb;
  const float* gain;
  const float* gain2;
  float* xdst;
  float* dump;
  int epi;
  float* yout;
  int ystride;
  uint16_t* hout;
  int hstride;
  float* ssout;
  int rows_valid;
  // attention
  int type, newkv, slots, seqoff;
  int out_f16;   // SiLU / attention outputs in fp16 (decode workspace) rather than bf16
  const uint8_t* kc;
  const uint8_t* vc;
  uint16_t* aout;
};

template <int NB>
struct Lay {
  static constexpr int RING = 0;
  static constexpr int MBAR = RING + NW * NSLOT * SLOT_BYTES;
  static constexpr int XS = MBAR + NW * NSLOT * 8;
  static constexpr int XSUM = XS + xs_cap(NB);
  static constexpr int WSP = XSUM + XSUM_BYTES;
  static constexpr int QS = WSP + wsp_bytes(NB);
  static constexpr int KNV = QS + MAX_GQ * 128 * 4;
  static constexpr int RED = KNV + 512;
  static constexpr int POSB = RED + 64 * 4;
  static constexpr int LB = POSB + MAX_B * 4;
  static constexpr int SNEW = LB + 2 * MAX_B * 4;
  static constexpr int SST = SNEW + 2 * MAX_B * 4;
  static constexpr int FLAGS = SST + 2 * (MAX_SEG + 1) * 4;
  static constexpr int TOTAL = FLAGS + 64;
  static constexpr int APW_BYTES = xs_cap(NB) + XSUM_BYTES + wsp_bytes(NB);  // attention warp partials
  static constexpr int QF = XS + NW * MAX_GQ * (128 + 2) * 4;                 // q fragments (after the partials)
};
static_assert(Lay<1>::TOTAL <= 232448 && Lay<2>::TOTAL <= 232448, "shared memory budget");
static_assert(Lay<1>::QF + 4096 <= Lay<1>::XS + Lay<1>::APW_BYTES, "q fragments overlap");
static_assert(Lay<2>::QF + 4096 <= Lay<2>::XS + Lay<2>::APW_BYTES, "q fragments overlap");

__device__ __forceinline__ uint32_t u4_word(const uint4& v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// Position (in bf16 halves) of x[b][kl] in the fragment-ordered x buffer.
__device__ __forceinline__ int xfrag_half(int b, int kl, int xrow) {
  const int ks = kl >> 4, j = kl & 15;
  const int t = (j & 7) >> 1, hi = j >> 3, e = j & 1;
  const int word = b * xrow + ((ks >> 1) * 4 + t) * 4 + (ks & 1) * 2 + hi;
  return word * 2 + e;
}

// ---------------------------------------------------------------------------
// Unit kernels (one warp, one unit)
// ---------------------------------------------------------------------------
template <int NB>
__device__ __forceinline__ void w4_unit(const uint8_t* slot, const uint4* xs4, int xrow4, int ks0,
                                        const float* xsum, int grp0, float (&acc)[NB][4], int B, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const uint4* qw = reinterpret_cast<const uint4*>(slot);
  const uint16_t* sc = reinterpret_cast<const uint16_t*>(slot + 4096);
  const uint32_t* zw = reinterpret_cast<const uint32_t*>(slot + 4224);
#pragma unroll
  for (int grp = 0; grp < 4; ++grp) {
    const uint4 w0 = qw[(grp * 2) * 32 + lane];
    const uint4 w1 = qw[(grp * 2 + 1) * 32 + lane];
    uint4 xv[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const int bb = g + 8 * nb;
#pragma unroll
      for (int pr = 0; pr < 4; ++pr) {
        const int ks = ks0 + grp * 8 + pr * 2;
        xv[nb][pr] = (bb < B) ? xs4[bb * xrow4 + (ks >> 1) * 4 + t] : make_uint4(0u, 0u, 0u, 0u);
      }
    }
    float c[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) c[nb][0] = c[nb][1] = c[nb][2] = c[nb][3] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t w = u4_word(i < 4 ? w0 : w1, i & 3);
      const uint32_t a0 = lop3_and_or(w, 0x000F000Fu, 0x64006400u);
      const uint32_t a1 = lop3_and_or(w >> 4, 0x000F000Fu, 0x64006400u);
      const uint32_t a2 = lop3_and_or(w >> 8, 0x000F000Fu, 0x64006400u);
      const uint32_t a3 = lop3_and_or(w >> 12, 0x000F000Fu, 0x64006400u);
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const uint4& x = xv[nb][i >> 1];
        mma_16816_f16(c[nb], a0, a1, a2, a3, (i & 1) ? x.z : x.x, (i & 1) ? x.w : x.y);
      }
    }
    const float sl = half_bits_to_f32(sc[grp * 16 + g]);
    const float sh = half_bits_to_f32(sc[grp * 16 + g + 8]);
    const float zl = 1024.f + float((zw[grp * 2] >> (4 * g)) & 15u);
    const float zh = 1024.f + float((zw[grp * 2 + 1] >> (4 * g)) & 15u);
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const float* xsr = xsum + (grp0 + grp) * (8 * NB) + nb * 8 + 2 * t;
      const float x0 = xsr[0], x1 = xsr[1];
      acc[nb][0] = fmaf(sl, c[nb][0] - zl * x0, acc[nb][0]);
      acc[nb][1] = fmaf(sl, c[nb][1] - zl * x1, acc[nb][1]);
      acc[nb][2] = fmaf(sh, c[nb][2] - zh * x0, acc[nb][2]);
      acc[nb][3] = fmaf(sh, c[nb][3] - zh * x1, acc[nb][3]);
    }
  }
}

template <int NB>
__device__ __forceinline__ void bf_unit(const uint8_t* slot, const uint4* xs4, int xrow4, int ks0,
                                        float (&acc)[NB][4], int B, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const uint4* aw = reinterpret_cast<const uint4*>(slot);
  uint4 xv[NB][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    const int bb = g + 8 * nb;
#pragma unroll
    for (int pr = 0; pr < 4; ++pr) {
      const int ks = ks0 + pr * 2;
      xv[nb][pr] = (bb < B) ? xs4[bb * xrow4 + (ks >> 1) * 4 + t] : make_uint4(0u, 0u, 0u, 0u);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 a = aw[i * 32 + lane];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const uint4& x = xv[nb][i >> 1];
      mma_16816(acc[nb], a.x, a.y, a.z, a.w, (i & 1) ? x.z : x.x, (i & 1) ? x.w : x.y);
    }
  }
}

// ---------------------------------------------------------------------------
// The engine
// ---------------------------------------------------------------------------
template <int NB, int HD>
struct Engine {
  using L = Lay<NB>;
  const EngineParams& P;
  uint8_t* sm;
  int tid, warp, lane, cta;
  uint32_t consumed, issued;
  bool bad;  // this warp saw a timeout: stop waiting and issuing
  // loader cursor
  int lp;
  PD lpd;
  long long li, lend;
  int lseg;
  bool lvalid;

  __device__ Engine(const EngineParams& p, uint8_t* s) : P(p), sm(s) {
    tid = threadIdx.x;
    warp = tid >> 5;
    lane = tid & 31;
    cta = blockIdx.x;
    consumed = issued = 0;
    bad = false;
  }

  // ---- shared-memory views ----
  __device__ uint8_t* ring(int sl) const { return sm + L::RING + (warp * NSLOT + sl) * SLOT_BYTES; }
  __device__ uint64_t* mbar(int sl) const {
    return reinterpret_cast<uint64_t*>(sm + L::MBAR) + warp * NSLOT + sl;
  }
  __device__ uint32_t* xs() const { return reinterpret_cast<uint32_t*>(sm + L::XS); }
  __device__ float* xsum() const { return reinterpret_cast<float*>(sm + L::XSUM); }
  __device__ float* wsp() const { return reinterpret_cast<float*>(sm + L::WSP); }
  __device__ float* apw() const { return reinterpret_cast<float*>(sm + L::XS); }
  __device__ float* qs() const { return reinterpret_cast<float*>(sm + L::QS); }
  __device__ uint4* qf() const { return reinterpret_cast<uint4*>(sm + L::QF); }
  __device__ uint16_t* kn() const { return reinterpret_cast<uint16_t*>(sm + L::KNV); }
  __device__ uint16_t* vn() const { return reinterpret_cast<uint16_t*>(sm + L::KNV) + 128; }
  __device__ float* red() const { return reinterpret_cast<float*>(sm + L::RED); }
  __device__ int* posb() const { return reinterpret_cast<int*>(sm + L::POSB); }
  __device__ int* Lb(int type) const { return reinterpret_cast<int*>(sm + L::LB) + type * MAX_B; }
  __device__ int* snew(int type) const { return reinterpret_cast<int*>(sm + L::SNEW) + type * MAX_B; }
  __device__ int* sst(int type) const { return reinterpret_cast<int*>(sm + L::SST) + type * (MAX_SEG + 1); }
  __device__ int* flags() const { return reinterpret_cast<int*>(sm + L::FLAGS); }

  __device__ void set_error(uint32_t bits) { atomicOr(P.ws.ctl + 2, bits); }

  // ---- phase descriptors ----
  __device__ void gemv_geom(PD& d) const {
    d.nrb = d.n / RB;
    d.nkc = d.k / d.kcw;
    d.kps = choose_kps(d.nkc, d.kcw, P.B, NB);
    if (d.kps <= 0) d.kps = 1;  // host rejects such shapes; keep indices sane
    d.ns = d.nkc / d.kps;
    d.U = (long long)d.nrb * d.nkc;
    long long per = d.U / d.kps;
    d.nca = int(per < 1 ? 1 : (per < P.nc ? per : P.nc));
  }

  __device__ PD get_phase(int p) const {
    PD d;
    memset(&d, 0, sizeof(PD));
    const int B = P.B;
    if (P.mode == MODE_GEMV) {
      d.kind = PK_GEMV_W4;
      d.blob = P.g_blob;
      d.n = P.g_n;
      d.k = P.g_k;
      d.kcw = W4_KC;
      d.ub = W4_UNIT;
      d.xsrc = XS_BF16;
      d.xbf = P.g_x;
      d.xbf_stride = P.g_k;
      d.rows_valid = P.g_n;
      if (P.g_epi == W4A_EPI_SILU_MUL) {
        d.epi = EPI_SILU;
        d.hout = reinterpret_cast<uint16_t*>(P.g_out);
        d.hstride = P.g_n / 2;
      } else {
        d.epi = (P.g_epi == W4A_EPI_SUMSQ) ? EPI_Y_SUMSQ : EPI_Y;
        d.yout = reinterpret_cast<float*>(P.g_out);
        d.ystride = P.g_n;
        d.ssout = P.g_aux;
      }
      gemv_geom(d);
      return d;
    }
    if (P.mode == MODE_ATTN) {
      d.kind = PK_ATTN;
      d.type = 0;
      d.newkv = 0;
      d.seqoff = 0;
      d.slots = P.a_slots;
      d.kc = reinterpret_cast<const uint8_t*>(P.a_k);
      d.vc = reinterpret_cast<const uint8_t*>(P.a_v);
      d.aout = P.a_out;
      return d;
    }
    const int nl = P.n_layers, dm = P.d;
    if (p == 5 * nl) {
      d.kind = PK_GEMV_BF16;
      d.blob = P.lm_head;
      d.n = (P.vocab + RB - 1) / RB * RB;
      d.k = dm;
      d.kcw = BF_KC;
      d.ub = BF_UNIT;
      d.xsrc = XS_FINAL;
      d.xres = P.ws.xB;
      d.vres = P.ws.f;
      d.vss = P.ws.ss_f;
      d.vnrb = dm / RB;
      d.gain = P.layers[nl - 1].ffn_norm;
      d.gain2 = P.final_norm ? P.final_gain : nullptr;
      d.dump = P.dump ? P.dump + (size_t)nl * B * dm : nullptr;
      d.epi = EPI_LOGITS;
      d.yout = P.logits;
      d.ystride = P.vocab;
      d.rows_valid = P.vocab;
      gemv_geom(d);
      return d;
    }
    if (p == 5 * nl + 1) {
      d.kind = PK_ARGMAX;
      return d;
    }
    const int l = p / 5, sub = p % 5;
    const LayerPtrs& lw = P.layers[l];
    d.layer = l;
    const int qkv_dim = (P.nq + 2 * P.nkv) * P.hd;
    if (sub == 1) {
      d.kind = PK_ATTN;
      d.type = P.full[l] ? 1 : 0;
      d.newkv = 1;
      d.seqoff = P.seq0;
      d.slots = P.kv_slots[l];
      d.kc = P.kv_base + P.kv_off[l];
      d.vc = d.kc + (size_t)P.kv_batch * P.nkv * d.slots * HD * 2;
      d.aout = P.ws.o;
      d.out_f16 = 1;
      return d;
    }
    d.kind = PK_GEMV_W4;
    d.kcw = W4_KC;
    d.ub = W4_UNIT;
    d.rows_valid = 1 << 30;
    if (sub == 0) {
      d.blob = lw.qkv;
      d.n = qkv_dim;
      d.k = dm;
      if (l == 0) {
        d.xsrc = XS_EMBED;
      } else {
        d.xsrc = XS_RESID;
        d.xres = P.ws.xB;
        d.vres = P.ws.f;
        d.vss = P.ws.ss_f;
        d.vnrb = dm / RB;
        d.gain = P.layers[l - 1].ffn_norm;
      }
      d.xdst = P.ws.xA;
      d.dump = P.dump ? P.dump + (size_t)l * B * dm : nullptr;
      d.epi = EPI_Y_SUMSQ;
      d.yout = P.ws.y_qkv;
      d.ystride = qkv_dim;
      d.ssout = P.ws.ss_qkv;
    } else if (sub == 2) {
      d.blob = lw.o;
      d.n = dm;
      d.k = P.nq * P.hd;
      d.xsrc = XS_F16;
      d.xbf = P.ws.o;
      d.xbf_stride = P.nq * P.hd;
      d.epi = EPI_Y_SUMSQ;
      d.yout = P.ws.a;
      d.ystride = dm;
      d.ssout = P.ws.ss_a;
    } else if (sub == 3) {
      d.blob = lw.gu;
      d.n = 2 * P.ffn;
      d.k = dm;
      d.xsrc = XS_RESID;
      d.xres = P.ws.xA;
      d.vres = P.ws.a;
      d.vss = P.ws.ss_a;
      d.vnrb = dm / RB;
      d.gain = lw.attn_norm;
      d.xdst = P.ws.xB;
      d.epi = EPI_SILU;
      d.hout = P.ws.h;
      d.hstride = P.ffn;
      d.out_f16 = 1;
    } else {
      d.blob = lw.down;
      d.n = dm;
      d.k = P.ffn;
      d.xsrc = XS_F16;
      d.xbf = P.ws.h;
      d.xbf_stride = P.ffn;
      d.epi = EPI_Y_SUMSQ;
      d.yout = P.ws.f;
      d.ystride = dm;
      d.ssout = P.ws.ss_f;
    }
    gemv_geom(d);
    return d;
  }

  // ---- ranges ----
  __device__ void gemv_cta_range(const PD& d, long long& a, long long& b) const {
    if (cta < d.nca) {
      a = rstart(d.U, d.nca, cta);
      b = rstart(d.U, d.nca, cta + 1);
    } else {
      a = b = 0;
    }
  }
  __device__ static void warp_range(long long a, long long b, int w, long long& wa, long long& wb) {
    wa = a + (b - a) * w / NW;
    wb = a + (b - a) * (w + 1) / NW;
  }
  __device__ void attn_cta_range(const PD& d, long long& a, long long& b, int& nca) const {
    const long long total = sst(d.type)[P.B * P.nkv];
    nca = int(total < P.nc ? total : P.nc);
    if (nca > 0 && cta < nca) {
      a = rstart(total, nca, cta);
      b = rstart(total, nca, cta + 1);
    } else {
      a = b = 0;
    }
  }

  // ---- the loader ----
  __device__ void loader_enter(int p) {
    lp = p;
    if (p >= P.phase_end) {
      lvalid = false;
      return;
    }
    lpd = get_phase(p);
    long long a = 0, b = 0;
    if (lpd.kind == PK_GEMV_W4 || lpd.kind == PK_GEMV_BF16) {
      gemv_cta_range(lpd, a, b);
      warp_range(a, b, warp, li, lend);
    } else if (lpd.kind == PK_ATTN) {
      int nca;
      attn_cta_range(lpd, a, b, nca);
      li = a;
      lend = b;
      lseg = 0;
    } else {
      li = lend = 0;
    }
  }
  __device__ void loader_normalize() {
    for (;;) {
      if (lp >= P.phase_end) {
        lvalid = false;
        return;
      }
      if (lpd.kind == PK_GEMV_W4 || lpd.kind == PK_GEMV_BF16) {
        if (li < lend) {
          lvalid = true;
          return;
        }
      } else if (lpd.kind == PK_ATTN) {
        const int* st = sst(lpd.type);
        while (li < lend) {
          while (st[lseg + 1] <= li) ++lseg;
          const int key0 = int(li - st[lseg]) * ATT_CTA_KEYS + warp * ATT_KEYS;
          if (key0 < Lb(lpd.type)[lseg / P.nkv]) {
            lvalid = true;
            return;
          }
          ++li;
        }
      }
      loader_enter(lp + 1);
    }
  }
  __device__ void loader_issue() {
    const int sl = issued % NSLOT;
    uint64_t* bar = mbar(sl);
    uint8_t* dst = ring(sl);
    if (lpd.kind == PK_GEMV_W4 || lpd.kind == PK_GEMV_BF16) {
      const long long upsl = (long long)lpd.nrb * lpd.kps;
      const long long s = li / upsl, r = li - s * upsl;
      const long long rb = r / lpd.kps;
      const long long kc = s * lpd.kps + (r - rb * lpd.kps);
      const uint8_t* src = lpd.blob + (rb * lpd.nkc + kc) * lpd.ub;
      if (lane == 0) {
        mbar_expect_tx(bar, lpd.ub);
        bulk_g2s(dst, src, lpd.ub, bar);
      }
    } else {
      const int* st = sst(lpd.type);
      const int seg = lseg;
      const int bq = seg / P.nkv, g = seg % P.nkv;
      const int key0 = int(li - st[seg]) * ATT_CTA_KEYS + warp * ATT_KEYS;
      const size_t row = ((size_t)(lpd.seqoff + bq) * P.nkv + g) * lpd.slots + key0;
      constexpr uint32_t bytes = ATT_KEYS * HD * 2;
      if (lane == 0) {
        mbar_expect_tx(bar, 2 * bytes);
        bulk_g2s(dst, lpd.kc + row * HD * 2, bytes, bar);
        bulk_g2s(dst + bytes, lpd.vc + row * HD * 2, bytes, bar);
      }
    }
    ++issued;
  }
  __device__ void loader_start() {
    loader_enter(P.phase_begin);
    loader_normalize();
    for (int i = 0; i < NSLOT && lvalid; ++i) {
      loader_issue();
      ++li;
      loader_normalize();
    }
  }

  // ---- ring consumption ----
  __device__ const uint8_t* wait_slot() {
    const int sl = consumed % NSLOT;
    const uint32_t par = (consumed / NSLOT) & 1u;
    if (!bad && !mbar_try_wait(mbar(sl), par)) {
      const long long t0 = clock64();
      while (!mbar_try_wait(mbar(sl), par)) {
        if (clock64() - t0 > WAIT_CYCLES) {
          if (lane == 0) set_error(EW_MBAR_TIMEOUT);
          bad = true;
          break;
        }
      }
    }
    return ring(sl);
  }
  __device__ void release_slot() {
    // order this lane's generic accesses of the slot before the async re-fill
    fence_proxy_async();
    __syncwarp();
    ++consumed;
    if (lvalid && !bad) {
      loader_issue();
      ++li;
      loader_normalize();
    }
  }
  __device__ void drain() {
    while (consumed < issued) {
      const int sl = consumed % NSLOT;
      const uint32_t par = (consumed / NSLOT) & 1u;
      const long long t0 = clock64();
      while (!mbar_try_wait(mbar(sl), par)) {
        if (clock64() - t0 > WAIT_CYCLES) {
          if (lane == 0) set_error(EW_DRAIN_TIMEOUT);
          return;
        }
      }
      ++consumed;
    }
  }

  // ---- grid barrier ----
  __device__ bool grid_wait(uint32_t target) {
    if (tid == 0) {
      int ok = 1;
      const long long t0 = clock64();
      while (ld_acquire(P.ws.ctl) < target) {
        if (ld_volatile_u32(P.ws.ctl + 2) != 0u) {
          ok = 0;
          break;
        }
        if (clock64() - t0 > WAIT_CYCLES) {
          set_error(EW_BARRIER_TIMEOUT);
          ok = 0;
          break;
        }
        __nanosleep(32);
      }
      flags()[0] = ok;
    }
    __syncthreads();
    return flags()[0] != 0;
  }
  __device__ void grid_arrive() {
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      red_release_add(P.ws.ctl, 1u);
    }
  }

  // ---- GEMV phase ----
  __device__ void fill_x(const PD& d, long long a, long long b, int& kbase, int& klen) {
    const int B = P.B, dm = P.d;
    kbase = 0;
    klen = 0;
    if (a < b) {
      const long long upsl = (long long)d.nrb * d.kps;
      const int KS = d.kps * d.kcw;
      const int s0 = int(a / upsl), s1 = int((b - 1) / upsl);
      kbase = s0 * KS;
      klen = (s1 - s0 + 1) * KS;
    }
    if (B * (klen * 2 + 64) > xs_cap(NB)) {  // the host sizes slabs so this never happens
      if (tid == 0) set_error(EW_BAD_SHAPE);
      klen = 0;
    }
    float* rd = red();
    if (d.xsrc == XS_RESID || d.xsrc == XS_FINAL) {
      // RMSNorm factor of the branch output from its per-16-row sums of squares.
      if (warp < B) {
        float s = 0.f;
        for (int i = lane; i < d.vnrb; i += 32) s += __ldcg(d.vss + (size_t)i * B + warp);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) rd[warp] = rsqrtf(s / float(dm) + P.eps);
      }
      __syncthreads();
    }
    if (d.xsrc == XS_FINAL && d.gain2 != nullptr) {
      // sum of squares of the new residual over the whole model width
      float part[MAX_B];
#pragma unroll
      for (int bb = 0; bb < MAX_B; ++bb) part[bb] = 0.f;
      for (int k = tid; k < dm; k += NT) {
        const float g = d.gain[k];
#pragma unroll
        for (int bb = 0; bb < MAX_B; ++bb) {
          if (bb < B) {
            const float x1 = __ldcg(d.xres + (size_t)bb * dm + k) + __ldcg(d.vres + (size_t)bb * dm + k) * rd[bb] * g;
            part[bb] = fmaf(x1, x1, part[bb]);
          }
        }
      }
      float* wr = wsp();
#pragma unroll
      for (int bb = 0; bb < MAX_B; ++bb) {
        if (bb < B) {
          float s = part[bb];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
          if (lane == 0) wr[warp * MAX_B + bb] = s;
        }
      }
      __syncthreads();
      if (tid < B) {
        float s = 0.f;
        for (int w = 0; w < NW; ++w) s += wr[w * MAX_B + tid];
        rd[16 + tid] = rsqrtf(s / float(dm) + P.eps);
      }
      __syncthreads();
    }
    // x fragments for [kbase, kbase + klen): fp16 for the int4 GEMVs, bf16 for the lm_head
    const bool f16 = (d.kind == PK_GEMV_W4);
    uint16_t* xh = reinterpret_cast<uint16_t*>(xs());
    uint32_t* xmax = reinterpret_cast<uint32_t*>(rd + 32);   // |x| max bits per batch row
    float* xscale = rd + 48;                                 // 2^e per batch row
    if (tid < MAX_B) {
      xmax[tid] = 0u;
      xscale[tid] = 1.f;
    }
    __syncthreads();
    const int xrow = klen / 2 + 16;
    const int total = B * klen;
    {
      int curb = -1;
      float m = 0.f;
      for (int idx = tid; idx < total; idx += NT) {
        const int bb = idx / klen, kl = idx - bb * klen;
        if (bb != curb) {
          if (curb >= 0) atomicMax(xmax + curb, __float_as_uint(m));
          curb = bb;
          m = 0.f;
        }
        const float v = load_x(d, bb, kbase + kl);
        m = fmaxf(m, fabsf(v));
        xh[xfrag_half(bb, kl, xrow)] = f16 ? f32_to_f16(v) : f32_to_bf16(v);
      }
      if (curb >= 0) atomicMax(xmax + curb, __float_as_uint(m));
    }
    __syncthreads();
    if (f16) {
      // fp16 range guard: rows whose max |x| reaches 2^15 are scaled by an exact
      // power of two (undone on the partial sums in flush()).
      bool any = false;
      for (int bb = 0; bb < B; ++bb) any |= __uint_as_float(xmax[bb]) >= 32768.f;
      if (any) {
        for (int idx = tid; idx < total; idx += NT) {
          const int bb = idx / klen, kl = idx - bb * klen;
          const float mx = __uint_as_float(xmax[bb]);
          if (!(mx >= 32768.f)) continue;
          int ex;
          frexpf(mx, &ex);
          xh[xfrag_half(bb, kl, xrow)] = f32_to_f16(ldexpf(load_x(d, bb, kbase + kl), 15 - ex));
        }
        __syncthreads();
        if (tid < B) {
          const float mx = __uint_as_float(xmax[tid]);
          if (mx >= 32768.f) {
            int ex;
            frexpf(mx, &ex);
            xscale[tid] = ldexpf(1.f, ex - 15);
          }
        }
      }
    }
    // residual copy and hidden-state dump (one CTA, the whole width)
    if (cta == 0 && (d.xdst != nullptr || d.dump != nullptr)) {
      for (int idx = tid; idx < B * dm; idx += NT) {
        const int bb = idx / dm, k = idx - bb * dm;
        float x;
        if (d.xsrc == XS_EMBED) {
          x = bf16_to_f32(P.embed[(size_t)clamp_token(bb) * dm + k]);
        } else {
          x = __ldcg(d.xres + idx) + __ldcg(d.vres + idx) * rd[bb] * d.gain[k];
        }
        if (d.xdst) d.xdst[idx] = x;
        if (d.dump) d.dump[idx] = x;
      }
    }
    if (cta == 0 && tid == 0 && d.xsrc == XS_EMBED) {
      for (int bb = 0; bb < B; ++bb)
        if (P.tokens[bb] < 0 || P.tokens[bb] >= P.vocab) set_error(EW_BAD_SHAPE);
    }
    __syncthreads();
    // per-(batch, 128-group) sums of the x values as stored (zero for unused columns)
    float* xsm = xsum();
    const int ngr = klen / GROUP;
    for (int pr = warp; pr < ngr * 8 * NB; pr += NW) {
      const int grp = pr / (8 * NB), bb = pr - grp * (8 * NB);
      float s = 0.f;
      if (bb < B) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint16_t hv = xh[xfrag_half(bb, grp * GROUP + lane * 4 + e, xrow)];
          s += f16 ? half_bits_to_f32(hv) : bf16_to_f32(hv);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) xsm[pr] = s;
    }
    __syncthreads();
  }

  __device__ int clamp_token(int bb) const {
    const int tok = P.tokens[bb];
    return tok < 0 ? 0 : (tok >= P.vocab ? P.vocab - 1 : tok);
  }

  // One activation of the GEMV input (fp32), from the phase's source.
  __device__ float load_x(const PD& d, int bb, int k) const {
    const int dm = P.d;
    const float* rd = red();
    switch (d.xsrc) {
      case XS_BF16:
        return bf16_to_f32(__ldcg(d.xbf + (size_t)bb * d.xbf_stride + k));
      case XS_F16:
        return half_bits_to_f32(__ldcg(d.xbf + (size_t)bb * d.xbf_stride + k));
      case XS_EMBED:
        return bf16_to_f32(P.embed[(size_t)clamp_token(bb) * dm + k]);
      default: {
        float x = __ldcg(d.xres + (size_t)bb * dm + k) + __ldcg(d.vres + (size_t)bb * dm + k) * rd[bb] * d.gain[k];
        if (d.xsrc == XS_FINAL && d.gain2 != nullptr) x = x * rd[16 + bb] * d.gain2[k];
        return x;
      }
    }
  }

  __device__ int expected_pieces(const PD& d, int rb) const {
    int e = 0;
    for (int s = 0; s < d.ns; ++s) {
      const long long u0 = ((long long)s * d.nrb + rb) * d.kps;
      e += owner(d.U, d.nca, u0 + d.kps - 1) - owner(d.U, d.nca, u0) + 1;
    }
    return e;
  }

  __device__ void finalize(const PD& d, int rb, const float (&v)[NB][4]) {
    const int g = lane >> 2, t = lane & 3, B = P.B;
    if (d.epi == EPI_SILU) {
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const float u0 = __shfl_down_sync(0xffffffffu, v[nb][0], 4);
        const float u1 = __shfl_down_sync(0xffffffffu, v[nb][1], 4);
        const float u2 = __shfl_down_sync(0xffffffffu, v[nb][2], 4);
        const float u3 = __shfl_down_sync(0xffffffffu, v[nb][3], 4);
        if ((g & 1) == 0) {
          const int j0 = rb * 8 + g / 2, j1 = rb * 8 + (g + 8) / 2;
          const int b0 = nb * 8 + 2 * t, b1 = b0 + 1;
          const float s0 = v[nb][0] / (1.f + expf(-v[nb][0]));
          const float s1 = v[nb][1] / (1.f + expf(-v[nb][1]));
          const float s2 = v[nb][2] / (1.f + expf(-v[nb][2]));
          const float s3 = v[nb][3] / (1.f + expf(-v[nb][3]));
          if (b0 < B) {
            d.hout[(size_t)b0 * d.hstride + j0] = d.out_f16 ? f32_to_f16(s0 * u0) : f32_to_bf16(s0 * u0);
            d.hout[(size_t)b0 * d.hstride + j1] = d.out_f16 ? f32_to_f16(s2 * u2) : f32_to_bf16(s2 * u2);
          }
          if (b1 < B) {
            d.hout[(size_t)b1 * d.hstride + j0] = d.out_f16 ? f32_to_f16(s1 * u1) : f32_to_bf16(s1 * u1);
            d.hout[(size_t)b1 * d.hstride + j1] = d.out_f16 ? f32_to_f16(s3 * u3) : f32_to_bf16(s3 * u3);
          }
        }
      }
      return;
    }
    const int r0 = rb * RB + g, r1 = r0 + 8;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const int b0 = nb * 8 + 2 * t, b1 = b0 + 1;
      if (r0 < d.rows_valid) {
        if (b0 < B) d.yout[(size_t)b0 * d.ystride + r0] = v[nb][0];
        if (b1 < B) d.yout[(size_t)b1 * d.ystride + r0] = v[nb][1];
      }
      if (r1 < d.rows_valid) {
        if (b0 < B) d.yout[(size_t)b0 * d.ystride + r1] = v[nb][2];
        if (b1 < B) d.yout[(size_t)b1 * d.ystride + r1] = v[nb][3];
      }
      if (d.epi == EPI_Y_SUMSQ) {
        float s0 = v[nb][0] * v[nb][0] + v[nb][2] * v[nb][2];
        float s1 = v[nb][1] * v[nb][1] + v[nb][3] * v[nb][3];
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          s0 += __shfl_xor_sync(0xffffffffu, s0, o);
          s1 += __shfl_xor_sync(0xffffffffu, s1, o);
        }
        if (g == 0) {
          if (b0 < B) d.ssout[(size_t)rb * B + b0] = s0;
          if (b1 < B) d.ssout[(size_t)rb * B + b1] = s1;
        }
      }
    }
  }

  // A piece of segment `seg` (slab s, row block rb) held in this warp's registers.
  __device__ void piece_out(const PD& d, long long seg, const float (&v)[NB][4]) {
    const int s = int(seg / d.nrb), rb = int(seg - (long long)s * d.nrb);
    const long long u0 = seg * d.kps;
    const int c0 = owner(d.U, d.nca, u0), c1 = owner(d.U, d.nca, u0 + d.kps - 1);
    if (d.ns == 1 && c0 == c1) {
      finalize(d, rb, v);
      return;
    }
    constexpr int PF = 32 * 4 * NB;  // floats per piece
    float* gp = P.ws.gpart + (seg * 2 + (cta - c0)) * PF + lane * 4 * NB;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
      reinterpret_cast<float4*>(gp)[nb] = make_float4(v[nb][0], v[nb][1], v[nb][2], v[nb][3]);
    __threadfence();
    __syncwarp();
    uint32_t old = 0;
    if (lane == 0) old = atomicAdd(P.ws.seg_ctr + rb, 1u);
    old = __shfl_sync(0xffffffffu, old, 0);
    if (int(old) == expected_pieces(d, rb) - 1) {
      __threadfence();
      float sum[NB][4];
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) sum[nb][0] = sum[nb][1] = sum[nb][2] = sum[nb][3] = 0.f;
      for (int ss = 0; ss < d.ns; ++ss) {
        const long long sg = (long long)ss * d.nrb + rb;
        const long long w0 = sg * d.kps;
        const int np = owner(d.U, d.nca, w0 + d.kps - 1) - owner(d.U, d.nca, w0) + 1;
        for (int pc = 0; pc < np; ++pc) {
          const float* q = P.ws.gpart + (sg * 2 + pc) * PF + lane * 4 * NB;
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            const float4 f = __ldcg(reinterpret_cast<const float4*>(q) + nb);
            sum[nb][0] += f.x;
            sum[nb][1] += f.y;
            sum[nb][2] += f.z;
            sum[nb][3] += f.w;
          }
        }
      }
      finalize(d, rb, sum);
      if (lane == 0) P.ws.seg_ctr[rb] = 0u;
    }
  }

  __device__ void run_gemv(const PD& d) {
    long long a, b;
    gemv_cta_range(d, a, b);
    int kbase, klen;
    fill_x(d, a, b, kbase, klen);
    if (a >= b) return;
    const uint4* xs4 = reinterpret_cast<const uint4*>(xs());
    const int xrow4 = (klen / 2 + 16) / 4;
    const float* xsm = xsum();
    long long wa, wb;
    warp_range(a, b, warp, wa, wb);
    const long long upsl = (long long)d.nrb * d.kps;
    float acc[NB][4];
    long long cur = -1;
    float* my = wsp() + warp * (2 * 32 * 4 * NB);
    for (long long u = wa; u < wb; ++u) {
      const long long seg = u / d.kps;
      if (seg != cur) {
        if (cur >= 0) flush(d, cur, acc, wa, wb, my);
        cur = seg;
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0.f;
      }
      const long long s = u / upsl, r = u - s * upsl;
      const long long rb = r / d.kps;
      const int kc = int(s * d.kps + (r - rb * d.kps));
      const int koff = kc * d.kcw - kbase;
      const uint8_t* slot = wait_slot();
      if (d.kind == PK_GEMV_W4)
        w4_unit<NB>(slot, xs4, xrow4, koff >> 4, xsm, koff >> 7, acc, P.B, lane);
      else
        bf_unit<NB>(slot, xs4, xrow4, koff >> 4, acc, P.B, lane);
      release_slot();
    }
    if (cur >= 0) flush(d, cur, acc, wa, wb, my);
    __syncthreads();
    cta_combine(d, a, b);
  }

  __device__ void flush(const PD& d, long long seg, float (&acc)[NB][4], long long wa, long long wb,
                        float* my) {
    if (d.kind == PK_GEMV_W4) {
      const float* xscale = red() + 48;
      const int t = lane & 3;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const float s0 = xscale[nb * 8 + 2 * t], s1 = xscale[nb * 8 + 2 * t + 1];
        acc[nb][0] *= s0;
        acc[nb][1] *= s1;
        acc[nb][2] *= s0;
        acc[nb][3] *= s1;
      }
    }
    const long long u0 = seg * d.kps;
    if (u0 >= wa && u0 + d.kps <= wb) {
      piece_out(d, seg, acc);
    } else {
      const int sl = (seg == wa / d.kps) ? 0 : 1;
      float* q = my + sl * (32 * 4 * NB) + lane * 4 * NB;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
        reinterpret_cast<float4*>(q)[nb] = make_float4(acc[nb][0], acc[nb][1], acc[nb][2], acc[nb][3]);
    }
  }

  __device__ void cta_combine(const PD& d, long long a, long long b) {
    int count = 0;
    long long last = -1;
    for (int w = 0; w < NW; ++w) {
      long long wa, wb;
      warp_range(a, b, w, wa, wb);
      if (wa >= wb) continue;
      const long long fs = wa / d.kps, ls = (wb - 1) / d.kps;
      for (int which = 0; which < 2; ++which) {
        const long long S = which ? ls : fs;
        if (which && ls == fs) break;
        const bool complete = (S * d.kps >= wa) && (S * d.kps + d.kps <= wb);
        if (complete || S == last) continue;
        if (count % NW == warp) combine_segment(d, S, a, b);
        ++count;
        last = S;
      }
    }
  }

  __device__ void combine_segment(const PD& d, long long S, long long a, long long b) {
    float sum[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) sum[nb][0] = sum[nb][1] = sum[nb][2] = sum[nb][3] = 0.f;
    for (int w = 0; w < NW; ++w) {
      long long wa, wb;
      warp_range(a, b, w, wa, wb);
      if (wa >= wb || S * d.kps >= wb || S * d.kps + d.kps <= wa) continue;
      const int sl = (S == wa / d.kps) ? 0 : 1;
      const float* q = wsp() + w * (2 * 32 * 4 * NB) + sl * (32 * 4 * NB) + lane * 4 * NB;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const float4 f = reinterpret_cast<const float4*>(q)[nb];
        sum[nb][0] += f.x;
        sum[nb][1] += f.y;
        sum[nb][2] += f.z;
        sum[nb][3] += f.w;
      }
    }
    piece_out(d, S, sum);
  }

  // ---- attention phase ----
  __device__ float sum_ss(const float* ss, int rb0, int rb1, int bq) const {
    float s = 0.f;
    for (int i = rb0 + lane; i < rb1; i += 32) s += __ldcg(ss + (size_t)i * P.B + bq);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
  }

  __device__ void attn_prologue(const PD& d, int seg, bool own_new) {
    const int bq = seg / P.nkv, g = seg % P.nkv;
    const int GQ = P.nq / P.nkv;
    float* q = qs();
    float* rd = red();
    const float qscale = 1.4426950408889634f * rsqrtf(float(HD));
    if (d.newkv) {
      const int qkv_dim = (P.nq + 2 * P.nkv) * HD;
      const float* y = P.ws.y_qkv + (size_t)bq * qkv_dim;
      const int nqrb = P.nq * HD / RB, nkrb = P.nkv * HD / RB;
      if (warp == 0) {
        const float s = sum_ss(P.ws.ss_qkv, 0, nqrb, bq);
        if (lane == 0) rd[32] = rsqrtf(s / float(P.nq * HD) + P.eps);
      } else if (warp == 1) {
        const float s = sum_ss(P.ws.ss_qkv, nqrb, nqrb + nkrb, bq);
        if (lane == 0) rd[33] = rsqrtf(s / float(P.nkv * HD) + P.eps);
      }
      __syncthreads();
      const float rq = rd[32], rk = rd[33];
      const int pos = posb()[bq];
      const double* fr = P.inv_freq[d.type];
      const float ms = P.mscale[d.type];
      const float* qn = P.layers[d.layer].q_norm;
      const float* kg = P.layers[d.layer].k_norm;
      constexpr int H2 = HD / 2;
      for (int idx = tid; idx < GQ * H2; idx += NT) {
        const int h = idx / H2, i = idx - h * H2;
        const int row = (g * GQ + h) * HD;
        const float x1 = __ldcg(y + row + i) * rq * qn[row + i];
        const float x2 = __ldcg(y + row + i + H2) * rq * qn[row + i + H2];
        double sn, cs;
        sincos(double(pos) * fr[i], &sn, &cs);
        const float c = float(cs) * ms, s = float(sn) * ms;
        q[h * HD + i] = (x1 * c - x2 * s) * qscale;
        q[h * HD + i + H2] = (x2 * c + x1 * s) * qscale;
      }
      if (own_new) {
        const int krow = P.nq * HD + g * HD, vrow = (P.nq + P.nkv) * HD + g * HD;
        for (int i = tid; i < H2; i += NT) {
          const float x1 = __ldcg(y + krow + i) * rk * kg[g * HD + i];
          const float x2 = __ldcg(y + krow + i + H2) * rk * kg[g * HD + i + H2];
          double sn, cs;
          sincos(double(pos) * fr[i], &sn, &cs);
          const float c = float(cs) * ms, s = float(sn) * ms;
          kn()[i] = f32_to_bf16(x1 * c - x2 * s);
          kn()[i + H2] = f32_to_bf16(x2 * c + x1 * s);
        }
        for (int i = tid; i < HD; i += NT) vn()[i] = f32_to_bf16(__ldcg(y + vrow + i));
        __syncthreads();
        const int sn_ = snew(d.type)[bq];
        const size_t row = ((size_t)(d.seqoff + bq) * P.nkv + g) * d.slots + sn_;
        uint16_t* kd = reinterpret_cast<uint16_t*>(const_cast<uint8_t*>(d.kc)) + row * HD;
        uint16_t* vd = reinterpret_cast<uint16_t*>(const_cast<uint8_t*>(d.vc)) + row * HD;
        for (int i = tid; i < HD; i += NT) {
          const int sw = (((i >> 3) ^ (sn_ & 7)) << 3) | (i & 7);
          kd[sw] = kn()[i];
          vd[sw] = vn()[i];
        }
      }
    } else {
      const uint16_t* qin = P.a_q + ((size_t)bq * P.nq + g * GQ) * HD;
      for (int idx = tid; idx < GQ * HD; idx += NT) q[idx] = bf16_to_f32(qin[idx]) * qscale;
    }
    __syncthreads();
    // q as hi + lo bf16 mma A fragments: {a0 hi, a2 hi, a0 lo, a2 lo} per (k-step, lane)
    if (tid < (HD / 16) * 32) {
      const int s = tid >> 5, ln = tid & 31, gg = ln >> 2, t = ln & 3;
      uint4 f = make_uint4(0u, 0u, 0u, 0u);
      if (gg < GQ) {
        const float* qr = q + gg * HD + 16 * s + 2 * t;
        split_bf16x2(qr[0], qr[1], f.x, f.z);
        split_bf16x2(qr[8], qr[9], f.y, f.w);
      }
      qf()[tid] = f;
    }
    __syncthreads();
  }

  __device__ void run_attn(const PD& d) {
    long long a, b;
    int nca;
    attn_cta_range(d, a, b, nca);
    if (a >= b) return;
    const int* st = sst(d.type);
    const int GQ = P.nq / P.nkv;
    constexpr int PW = MAX_GQ * (HD + 2);  // floats per (warp or CTA) partial
    const int g = lane >> 2, t = lane & 3;
    int seg = 0;
    long long u = a;
    while (u < b) {
      while (st[seg + 1] <= u) ++seg;
      const long long run_end = (b < st[seg + 1]) ? b : st[seg + 1];
      const int bq = seg / P.nkv;
      const int Lk = Lb(d.type)[bq];
      const int sn_ = d.newkv ? snew(d.type)[bq] : -1;
      const long long jnew = st[seg] + (sn_ >= 0 ? sn_ / ATT_CTA_KEYS : 0);
      const bool own_new = d.newkv && sn_ >= 0 && jnew >= u && jnew < run_end;
      attn_prologue(d, seg, own_new);
      const uint4* qfr = qf();
      float m = -INFINITY, lsum = 0.f;
      float o[HD / 8][4];
#pragma unroll
      for (int n = 0; n < HD / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
      for (long long j = u; j < run_end; ++j) {
        const int key0 = int(j - st[seg]) * ATT_CTA_KEYS + warp * ATT_KEYS;
        if (key0 >= Lk) continue;
        uint8_t* slot = const_cast<uint8_t*>(wait_slot());
        uint8_t* Ks = slot;
        uint8_t* Vs = slot + ATT_KEYS * HD * 2;
        if (own_new && sn_ >= key0 && sn_ < key0 + ATT_KEYS) {
          const int r = sn_ - key0;  // == sn_ & 7
          uint16_t* kr = reinterpret_cast<uint16_t*>(Ks + r * HD * 2);
          uint16_t* vr = reinterpret_cast<uint16_t*>(Vs + r * HD * 2);
          for (int i = lane; i < HD; i += 32) {
            const int sw = (((i >> 3) ^ r) << 3) | (i & 7);
            kr[sw] = kn()[i];
            vr[sw] = vn()[i];
          }
          __syncwarp();
        }
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
        const int r = lane & 7, mi = lane >> 3;
#pragma unroll
        for (int s = 0; s < HD / 16; s += 2) {
          uint32_t k0, k1, k2, k3;
          ldsm_x4(k0, k1, k2, k3, Ks + r * HD * 2 + (((2 * s + mi) ^ r) << 4));
          const uint4 f0 = qfr[s * 32 + lane], f1 = qfr[(s + 1) * 32 + lane];
          mma_16816(sc, f0.x, 0u, f0.y, 0u, k0, k1);
          mma_16816(sc, f0.z, 0u, f0.w, 0u, k0, k1);
          mma_16816(sc, f1.x, 0u, f1.y, 0u, k2, k3);
          mma_16816(sc, f1.z, 0u, f1.w, 0u, k2, k3);
        }
        const int ka = key0 + 2 * t;
        const float s0 = (ka < Lk) ? sc[0] : -INFINITY;
        const float s1 = (ka + 1 < Lk) ? sc[1] : -INFINITY;
        float mx = fmaxf(s0, s1);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float mn = fmaxf(m, mx);
        const float alpha = exp2f(m - mn);
        const float p0 = exp2f(s0 - mn), p1 = exp2f(s1 - mn);
        lsum = lsum * alpha + p0 + p1;
        m = mn;
#pragma unroll
        for (int n = 0; n < HD / 8; ++n) {
          o[n][0] *= alpha;
          o[n][1] *= alpha;
        }
        uint32_t pa, pl;
        split_bf16x2(p0, p1, pa, pl);
#pragma unroll
        for (int q4 = 0; q4 < HD / 32; ++q4) {
          uint32_t v0, v1, v2, v3;
          ldsm_x4_t(v0, v1, v2, v3, Vs + r * HD * 2 + (((4 * q4 + mi) ^ r) << 4));
          mma_1688(o[4 * q4 + 0], pa, 0u, v0);
          mma_1688(o[4 * q4 + 0], pl, 0u, v0);
          mma_1688(o[4 * q4 + 1], pa, 0u, v1);
          mma_1688(o[4 * q4 + 1], pl, 0u, v1);
          mma_1688(o[4 * q4 + 2], pa, 0u, v2);
          mma_1688(o[4 * q4 + 2], pl, 0u, v2);
          mma_1688(o[4 * q4 + 3], pa, 0u, v3);
          mma_1688(o[4 * q4 + 3], pl, 0u, v3);
        }
        release_slot();
      }
      lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
      lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
      float* wp = apw() + warp * PW;
      if (g < GQ) {
#pragma unroll
        for (int n = 0; n < HD / 8; ++n) {
          wp[g * (HD + 2) + 8 * n + 2 * t] = o[n][0];
          wp[g * (HD + 2) + 8 * n + 2 * t + 1] = o[n][1];
        }
        if (t == 0) {
          wp[g * (HD + 2) + HD] = m;
          wp[g * (HD + 2) + HD + 1] = lsum;
        }
      }
      __syncthreads();
      attn_combine(d, seg, a, b, nca);
      __syncthreads();
      u = run_end;
    }
  }

  __device__ void attn_combine(const PD& d, int seg, long long a, long long b, int nca) {
    constexpr int PW = MAX_GQ * (HD + 2);
    const int* st = sst(d.type);
    const int GQ = P.nq / P.nkv;
    const int bq = seg / P.nkv, g = seg % P.nkv;
    const bool split = (st[seg] < a) || (st[seg + 1] > b);
    const float* wp = apw();
    uint16_t* out = d.aout + ((size_t)bq * P.nq + g * GQ) * HD;
    const int pslot = (st[seg] < a) ? 0 : 1;
    float* piece = P.ws.apart + ((size_t)cta * 2 + pslot) * PW;
    for (int idx = tid; idx < GQ * HD; idx += NT) {
      const int h = idx / HD, dd = idx - h * HD;
      float M = -INFINITY;
      for (int w = 0; w < NW; ++w) M = fmaxf(M, wp[w * PW + h * (HD + 2) + HD]);
      float ls = 0.f, os = 0.f;
      for (int w = 0; w < NW; ++w) {
        const float e = exp2f(wp[w * PW + h * (HD + 2) + HD] - M);
        ls += e * wp[w * PW + h * (HD + 2) + HD + 1];
        os += e * wp[w * PW + h * (HD + 2) + dd];
      }
      if (!split) {
        out[h * HD + dd] = d.out_f16 ? f32_to_f16(os / ls) : f32_to_bf16(os / ls);
      } else {
        piece[h * (HD + 2) + dd] = os;
        if (dd == 0) {
          piece[h * (HD + 2) + HD] = M;
          piece[h * (HD + 2) + HD + 1] = ls;
        }
      }
    }
    if (!split) return;
    __threadfence();
    __syncthreads();
    const int c0 = owner(st[P.B * P.nkv], nca, st[seg]);
    const int c1 = owner(st[P.B * P.nkv], nca, st[seg + 1] - 1);
    if (tid == 0) {
      const uint32_t old = atomicAdd(P.ws.seg_ctr + seg, 1u);
      flags()[1] = (int(old) == c1 - c0) ? 1 : 0;
    }
    __syncthreads();
    if (!flags()[1]) return;
    __threadfence();
    const long long total = st[P.B * P.nkv];
    for (int idx = tid; idx < GQ * HD; idx += NT) {
      const int h = idx / HD, dd = idx - h * HD;
      float M = -INFINITY;
      for (int c = c0; c <= c1; ++c) {
        const int sl = (st[seg] < rstart(total, nca, c)) ? 0 : 1;
        M = fmaxf(M, __ldcg(P.ws.apart + ((size_t)c * 2 + sl) * PW + h * (HD + 2) + HD));
      }
      float ls = 0.f, os = 0.f;
      for (int c = c0; c <= c1; ++c) {
        const int sl = (st[seg] < rstart(total, nca, c)) ? 0 : 1;
        const float* pc = P.ws.apart + ((size_t)c * 2 + sl) * PW + h * (HD + 2);
        const float e = exp2f(__ldcg(pc + HD) - M);
        ls += e * __ldcg(pc + HD + 1);
        os += e * __ldcg(pc + dd);
      }
      out[h * HD + dd] = d.out_f16 ? f32_to_f16(os / ls) : f32_to_bf16(os / ls);
    }
    if (tid == 0) P.ws.seg_ctr[seg] = 0u;
  }

  // ---- argmax phase ----
  __device__ void run_argmax() {
    if (P.next_token == nullptr) return;
    const int V = P.vocab, B = P.B;
    const int r0 = int(rstart(V, P.nc, cta)), r1 = int(rstart(V, P.nc, cta + 1));
    float* rv = red();
    int* ri = reinterpret_cast<int*>(red() + 32);
    for (int bq = 0; bq < B; ++bq) {
      float best = -INFINITY;
      int bi = 0x7fffffff;
      for (int r = r0 + tid; r < r1; r += NT) {
        const float v = __ldcg(P.logits + (size_t)bq * V + r);
        if (v > best || (v == best && r < bi)) {
          best = v;
          bi = r;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > best || (ov == best && oi < bi)) {
          best = ov;
          bi = oi;
        }
      }
      if (lane == 0) {
        rv[warp] = best;
        ri[warp] = bi;
      }
      __syncthreads();
      if (tid == 0) {
        float bb = -INFINITY;
        int bbi = 0x7fffffff;
        for (int w = 0; w < NW; ++w)
          if (rv[w] > bb || (rv[w] == bb && ri[w] < bbi)) {
            bb = rv[w];
            bbi = ri[w];
          }
        P.ws.amax_val[(size_t)cta * B + bq] = bb;
        P.ws.amax_idx[(size_t)cta * B + bq] = bbi;
      }
      __syncthreads();
    }
    if (tid == 0) {
      __threadfence();
      const uint32_t old = atomicAdd(P.ws.ctl + 3, 1u);
      if (int(old) == P.nc - 1) {
        __threadfence();
        for (int bq = 0; bq < B; ++bq) {
          float bb = -INFINITY;
          int bbi = 0x7fffffff;
          for (int c = 0; c < P.nc; ++c) {
            const float v = __ldcg(P.ws.amax_val + (size_t)c * B + bq);
            const int i = __ldcg(P.ws.amax_idx + (size_t)c * B + bq);
            if (v > bb || (v == bb && i < bbi)) {
              bb = v;
              bbi = i;
            }
          }
          P.next_token[bq] = (bbi == 0x7fffffff) ? 0 : bbi;
        }
        P.ws.ctl[3] = 0u;
      }
    }
  }

  // ---- launch-level setup ----
  __device__ void setup() {
    if (lane == 0) {
      for (int s = 0; s < NSLOT; ++s) mbar_init(mbar(s), 1u);
      fence_mbar_init();
    }
    if (tid == 0) flags()[0] = 1;
    const int B = P.B;
    if (P.mode != MODE_GEMV && tid < B) posb()[tid] = (P.pos_const >= 0) ? P.pos_const : P.pos[tid];
    __syncthreads();
    if (P.mode != MODE_GEMV && tid < 2 * B) {
      const int type = tid / B, bq = tid - type * B;
      const int pos = posb()[bq];
      int Lk = 0, sn = -1;
      bool bad_pos = pos < 0;
      if (P.mode == MODE_DECODE) {
        if (type == 1) {
          bad_pos |= pos >= P.max_ctx;
          Lk = pos + 1;
          sn = pos;
        } else {
          Lk = pos + 1 < P.window ? pos + 1 : P.window;
          sn = pos % P.window;
        }
      } else if (type == 0) {
        if (P.a_window == 0) {
          bad_pos |= pos >= P.a_slots;
          Lk = pos + 1;
        } else {
          Lk = pos + 1 < P.a_window ? pos + 1 : P.a_window;
        }
      }
      if (bad_pos) {
        if (cta == 0) set_error(EW_BAD_POS);
        Lk = 0;
        sn = -1;
      }
      Lb(type)[bq] = Lk;
      snew(type)[bq] = sn;
    }
    __syncthreads();
    if (P.mode != MODE_GEMV && tid < 2) {
      int* st = sst(tid);
      st[0] = 0;
      for (int s = 0; s < B * P.nkv; ++s) {
        const int Lk = Lb(tid)[s / P.nkv];
        st[s + 1] = st[s] + (Lk + ATT_CTA_KEYS - 1) / ATT_CTA_KEYS;
      }
    }
    __syncthreads();
  }

  __device__ void run() {
    setup();
    loader_start();
    for (int p = P.phase_begin; p < P.phase_end; ++p) {
      if (p != P.phase_begin) {
        if (!grid_wait(uint32_t(p - P.phase_begin) * uint32_t(P.nc))) break;
      }
      const PD d = get_phase(p);
      if (d.kind == PK_GEMV_W4 || d.kind == PK_GEMV_BF16)
        run_gemv(d);
      else if (d.kind == PK_ATTN)
        run_attn(d);
      else
        run_argmax();
      grid_arrive();
    }
    drain();
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      const uint32_t old = atomicAdd(P.ws.ctl + 1, 1u);
      if (int(old) == P.nc - 1) {
        P.ws.ctl[0] = 0u;
        P.ws.ctl[1] = 0u;
        __threadfence();
      }
    }
  }
};

template <int NB, int HD>
__global__ void __launch_bounds__(NT, 1) w4a_engine_kernel(const __grid_constant__ EngineParams P) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Engine<NB, HD> e(P, smem_raw);
  e.run();
}

template <int NB>
constexpr int engine_smem_bytes() {
  return Lay<NB>::TOTAL;
}

}  // namespace w4a
