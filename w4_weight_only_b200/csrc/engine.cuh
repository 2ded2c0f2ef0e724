// The persistent decode engine.
//
// One CTA per SM, 16 warps.  A launch runs a list of phases (decode: per layer
// QKV GEMV, GQA attention, O GEMV, gate/up GEMV, down GEMV; then lm_head and
// argmax) separated by grid-wide barriers.  Every warp streams its own
// contiguous range of 4 KB "units" (16 weight rows x 512 int4 columns, 16 rows
// x 128 bf16 columns, or 8 keys of K and V) from HBM into a two-slot ring of
// shared memory with bulk asynchronous copies completing on mbarriers, and
// refills a slot with its next unit as soon as it has used it.  The stream
// runs across phase boundaries: weights and old KV entries do not depend on
// the activations, so the copies for phase p+1 are in flight while the CTA
// waits at the barrier that ends phase p.
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
// Work split of a GEMV phase: K is cut into `ns` slabs; a "segment" is one
// 16-row block of one slab.  Every CTA owns whole segments (so no segment is
// shared between CTAs); its warps split the CTA's units and the pieces of a
// segment held by different warps are summed in warp order in shared memory.
// With one slab the CTA finishes the rows (plain store, sums of squares, or
// SiLU * up); with several it stores one partial row per slab and the phase
// that consumes the vector adds the slabs in order (and computes any RMSNorm
// over the whole vector itself).  Every sum has a fixed order, so results are
// bit-reproducible.
//
// Attention splits each (sequence, KV head) over CTAs by keys; the last CTA to
// arrive on a segment's counter merges the pieces in CTA order (no waiting).
#pragma once
#include <float.h>
#include <math.h>

#include "ptx.cuh"
#include "w4a_internal.h"

namespace w4a {

constexpr long long WAIT_CYCLES = 4000000000LL;  // bound on any single wait (~2 s)
constexpr int MAX_SEG = MAX_B * 16;              // attention segments (batch x kv heads)
constexpr int NS_MAX = 8;                        // k-slabs a GEMV phase may use

__host__ __device__ inline long long rstart(long long U, int n, int i) { return (U * i) / n; }
// CTA (of n) whose range [rstart(c), rstart(c+1)) contains unit u.
__host__ __device__ inline int owner(long long U, int n, long long u) {
  return int(((u + 1) * n + U - 1) / U) - 1;
}

// x of klen columns for B rows fits the staging buffers (fragments and the
// per-group sums).
__host__ __device__ inline bool x_fits(long long klen, int B, int nb) {
  return B * (klen * 2 + 64) <= xs_cap(nb) && (klen / GROUP) * 8 * nb * 4 <= XSUM_BYTES;
}

// Largest k-chunks per slab whose x fragments fit the shared-memory budget
// (one slab when it fits whole, else two slabs must fit); 0 when none does.
__host__ __device__ inline int choose_kps(int nkc, int kcw, int B, int nb) {
  if (x_fits((long long)nkc * kcw, B, nb)) return nkc;
  for (int dv = nkc - 1; dv >= 1; --dv)
    if (nkc % dv == 0 && x_fits(2LL * dv * kcw, B, nb)) return dv;
  return 0;
}

// The geometry the host computes for a GEMV phase (see Geo).
// Chooses how many k-slabs a GEMV phase uses.  The phase lasts as long as its
// busiest CTA, i.e. ceil(segments / CTAs) segments of kps units each; every
// slab beyond the first makes the consuming phase read one more copy of the
// output vector from L2 (`readers` CTAs read all of it).  Both are counted in
// bytes moved per SM: an L2 byte costs 1 / L2_VS_SM_HBM of an HBM byte on one
// SM (an estimate: ~12 TB/s of L2 against 6.5 TB/s of HBM shared by the SMs).
constexpr double L2_VS_SM_HBM = 270.0;
inline Geo gemv_geo(long long n, long long k, int kcw, int B, int nb, int nc, int readers) {
  Geo g;
  g.nrb = int((n + RB - 1) / RB);
  g.nkc = int(k / kcw);
  g.ns = g.kps = g.nseg = g.nca = 0;
  const int kmax = choose_kps(g.nkc, kcw, B, nb);
  if (kmax <= 0 || nc <= 0) return g;
  const int ns0 = g.nkc / kmax;
  const int ub = kcw == W4_KC ? W4_UNIT : BF_UNIT;
  const double slab_cost = double(readers) * B * double(n) * 4.0 / L2_VS_SM_HBM;
  double best = 0.0;
  for (int ns = ns0; ns <= g.nkc && (ns == ns0 || ns <= NS_MAX); ++ns) {
    if (g.nkc % ns) continue;
    const int kps = g.nkc / ns;
    if (!(ns == 1 ? x_fits((long long)g.nkc * kcw, B, nb) : x_fits(2LL * kps * kcw, B, nb))) continue;
    const long long nseg = (long long)ns * g.nrb;
    const long long nca = nseg < nc ? nseg : nc;
    const long long per = (nseg + nca - 1) / nca;
    if (ns > 1 && per > g.nrb + 1) continue;  // a CTA's segments must span at most two slabs
    const double cost = double(per) * kps * ub + (ns - 1) * slab_cost;
    if (g.ns == 0 || cost < best) {
      best = cost;
      g.ns = ns;
      g.kps = kps;
      g.nseg = int(nseg);
      g.nca = int(nca);
    }
  }
  return g;
}

struct PD {
  int kind, layer;
  // GEMV
  const uint8_t* blob;
  int n, k, kcw, ub;
  Geo g;
  int xsrc;
  const uint16_t* xbf;    // 16-bit input rows (XS_BF16 / XS_F16)
  int xbf_stride;
  const float* xres;      // residual (XS_RESID / XS_FINAL)
  const float* vpart;     // branch output slabs [vns][B][vstride] (XS_RESID / XS_FINAL / XS_SILU)
  int vns, vstride;
  const float* gain;
  const float* gain2;
  float* xdst;
  float* dump;
  int epi;
  float* yout;
  int ystride;
  uint16_t* hout;
  int hstride;
  int out_f16;
  float* ssout;
  int rows_valid;
  float* part;            // EPI_PART target [ns][B][pstride]
  int pstride;
  // attention
  int type, newkv, slots, seqoff;
  const uint8_t* kc;
  const uint8_t* vc;
  uint16_t* aout;
  const float* qpart;     // QKV output slabs (decode)
  int qns;
  // argmax
  const float* lpart;
  int lns;
};

static_assert(sizeof(PD) <= 512, "phase descriptor slot");

struct Cursor {
  int p;     // phase
  int kind;  // PK_* of the phase, -1 past the last phase
  int i, end;  // unit index in [i, end) (GEMV: phase order; attention: CTA unit)
  // GEMV:      p0 = weights, x0 = unit bytes, x1 = k-chunks per row block,
  //            x2 = k-chunks per slab, x3 = row blocks, x4 = slab, x5 = row
  //            block, x6 = k-chunk within the slab (all of unit i)
  // attention: p0 = K region, p1 = V region, x0 = slots, x1 = first sequence,
  //            x2 = layer type, x3 = segment of unit i
  const uint8_t* p0;
  const uint8_t* p1;
  int x0, x1, x2, x3, x4, x5, x6;
};

// Ring state of a warp (a local value that only inlined code touches, so it
// stays in registers through the unit loops).
struct Stream {
  uint32_t consumed, issued;
  bool bad;   // this warp saw a timeout: stop waiting and issuing
  Cursor ld;  // next unit to copy into the ring (kind < 0: none left)
};

// Per-warp ring addresses and ids, held in registers by the unit loops.
struct RingCtx {
  uint8_t* base;   // slot 0 of this warp's ring
  uint64_t* bar;   // mbarrier of slot 0
  uint32_t* err;   // device error word
  int lane;
};

template <int NB>
struct Acc {
  float v[NB][4];
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
  static constexpr int PDS = FLAGS + 64;
  static constexpr int TOTAL = PDS + 512;
  static constexpr int APW_BYTES = xs_cap(NB) + XSUM_BYTES + wsp_bytes(NB);  // attention warp partials
  static constexpr int QF = XS + NW * MAX_GQ * (128 + 2) * 4;                 // q fragments (after the partials)
};
static_assert(Lay<1>::TOTAL <= 232448 && Lay<2>::TOTAL <= 232448, "shared memory budget");
static_assert(Lay<1>::QF + 4096 <= Lay<1>::XS + Lay<1>::APW_BYTES, "q fragments overlap");
static_assert(Lay<2>::QF + 4096 <= Lay<2>::XS + Lay<2>::APW_BYTES, "q fragments overlap");

// cos / sin of the rotation angle pos * f, times the attention factor: the
// angle is formed and reduced to [-pi, pi] in fp64, then evaluated in fp32.
__device__ __forceinline__ void rope_cs(int pos, double f, float ms, float& c, float& s) {
  const double a = double(pos) * f;
  const double r = a - 6.283185307179586 * rint(a * 0.15915494309189535);
  float sn, cs;
  sincosf(float(r), &sn, &cs);
  c = cs * ms;
  s = sn * ms;
}

__device__ __forceinline__ uint32_t u4_word(const uint4& v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
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
      const float2 xs2 = *reinterpret_cast<const float2*>(xsum + (grp0 + grp) * (8 * NB) + nb * 8 + 2 * t);
      acc[nb][0] = fmaf(sl, c[nb][0] - zl * xs2.x, acc[nb][0]);
      acc[nb][1] = fmaf(sl, c[nb][1] - zl * xs2.y, acc[nb][1]);
      acc[nb][2] = fmaf(sh, c[nb][2] - zh * xs2.x, acc[nb][2]);
      acc[nb][3] = fmaf(sh, c[nb][3] - zh * xs2.y, acc[nb][3]);
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
  int cur_phase = 0;

  __device__ Engine(const EngineParams& p, uint8_t* s) : P(p), sm(s) {
    tid = threadIdx.x;
    warp = tid >> 5;
    lane = tid & 31;
    cta = blockIdx.x;
  }

  // ---- shared-memory views ----
  __device__ uint64_t* fullb(int w, int sl) const {
    return reinterpret_cast<uint64_t*>(sm + L::MBAR) + w * NSLOT + sl;
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

  __device__ void set_error(uint32_t bits) const { atomicOr(P.ws.ctl + 2, bits); }
  // barrier over the CTA's warps (named barrier 1)
  __device__ static __forceinline__ void cbar() { asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory"); }

  __device__ void mark(int slot) const {
    if (P.trace != nullptr && tid == 0 && cur_phase < P.trace_phases)
      P.trace[((size_t)cur_phase * P.nc + cta) * 4 + slot] = globaltimer();
  }

  // ---- phase descriptors ----
  __device__ __noinline__ void get_phase(int p, PD& d) const {
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
      d.g = P.geo[0];
      if (d.g.ns > 1) {
        // partial rows, finished by the reduce phase
        d.epi = EPI_PART;
        d.part = P.ws.g_part;
        d.pstride = P.g_n;
      } else if (P.g_epi == W4A_EPI_SILU_MUL) {
        d.epi = EPI_SILU;
        d.hout = reinterpret_cast<uint16_t*>(P.g_out);
        d.hstride = P.g_n / 2;
      } else {
        d.epi = (P.g_epi == W4A_EPI_SUMSQ) ? EPI_Y_SUMSQ : EPI_Y;
        d.yout = reinterpret_cast<float*>(P.g_out);
        d.ystride = P.g_n;
        d.ssout = P.g_aux;
      }
      if (p == 1) d.kind = PK_REDUCE;
      return;
    }
    if (P.mode == MODE_ATTN) {
      d.kind = PK_ATTN;
      d.slots = P.a_slots;
      d.kc = reinterpret_cast<const uint8_t*>(P.a_k);
      d.vc = reinterpret_cast<const uint8_t*>(P.a_v);
      d.aout = P.a_out;
      return;
    }
    const int nl = P.n_layers, dm = P.d;
    const int qd = P.nq * P.hd, qkv_dim = (P.nq + 2 * P.nkv) * P.hd;
    const Geo& g_qkv = P.geo[0];
    const Geo& g_o = P.geo[1];
    const Geo& g_gu = P.geo[2];
    const Geo& g_dn = P.geo[3];
    const Geo& g_lm = P.geo[4];
    if (p == 5 * nl) {
      d.kind = PK_GEMV_BF16;
      d.blob = P.lm_head;
      d.n = (P.vocab + RB - 1) / RB * RB;
      d.k = dm;
      d.kcw = BF_KC;
      d.ub = BF_UNIT;
      d.g = g_lm;
      d.xsrc = XS_FINAL;
      d.xres = P.ws.xB;
      d.vpart = P.ws.f_part;
      d.vns = g_dn.ns;
      d.vstride = dm;
      d.gain = P.layers[nl - 1].ffn_norm;
      d.gain2 = P.final_norm ? P.final_gain : nullptr;
      d.dump = P.dump ? P.dump + (size_t)nl * B * dm : nullptr;
      d.rows_valid = P.vocab;
      if (d.g.ns == 1) {
        d.epi = EPI_Y;
        d.yout = P.logits;
        d.ystride = P.vocab;
      } else {
        d.epi = EPI_PART;
        d.part = P.ws.lg_part;
        d.pstride = P.vocab;
      }
      return;
    }
    if (p == 5 * nl + 1) {
      d.kind = PK_ARGMAX;
      d.lpart = g_lm.ns > 1 ? P.ws.lg_part : nullptr;
      d.lns = g_lm.ns;
      return;
    }
    const int l = p / 5, sub = p % 5;
    const LayerPtrs& lw = P.layers[l];
    d.layer = l;
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
      d.qpart = P.ws.y_part;
      d.qns = g_qkv.ns;
      return;
    }
    d.kind = PK_GEMV_W4;
    d.kcw = W4_KC;
    d.ub = W4_UNIT;
    d.rows_valid = 1 << 30;
    d.epi = EPI_PART;
    if (sub == 0) {
      d.blob = lw.qkv;
      d.n = qkv_dim;
      d.k = dm;
      d.g = g_qkv;
      if (l == 0) {
        d.xsrc = XS_EMBED;
      } else {
        d.xsrc = XS_RESID;
        d.xres = P.ws.xB;
        d.vpart = P.ws.f_part;
        d.vns = g_dn.ns;
        d.vstride = dm;
        d.gain = P.layers[l - 1].ffn_norm;
      }
      d.xdst = P.ws.xA;
      d.dump = P.dump ? P.dump + (size_t)l * B * dm : nullptr;
      d.part = P.ws.y_part;
      d.pstride = qkv_dim;
    } else if (sub == 2) {
      d.blob = lw.o;
      d.n = dm;
      d.k = qd;
      d.g = g_o;
      d.xsrc = XS_F16;
      d.xbf = P.ws.o;
      d.xbf_stride = qd;
      d.part = P.ws.a_part;
      d.pstride = dm;
    } else if (sub == 3) {
      d.blob = lw.gu;
      d.n = 2 * P.ffn;
      d.k = dm;
      d.g = g_gu;
      d.xsrc = XS_RESID;
      d.xres = P.ws.xA;
      d.vpart = P.ws.a_part;
      d.vns = g_o.ns;
      d.vstride = dm;
      d.gain = lw.attn_norm;
      d.xdst = P.ws.xB;
      if (d.g.ns == 1) {
        d.epi = EPI_SILU;
        d.hout = P.ws.h;
        d.hstride = P.ffn;
        d.out_f16 = 1;
      } else {
        d.part = P.ws.gu_part;
        d.pstride = 2 * P.ffn;
      }
    } else {
      d.blob = lw.down;
      d.n = dm;
      d.k = P.ffn;
      d.g = g_dn;
      if (g_gu.ns == 1) {
        d.xsrc = XS_F16;
        d.xbf = P.ws.h;
        d.xbf_stride = P.ffn;
      } else {
        d.xsrc = XS_SILU;
        d.vpart = P.ws.gu_part;
        d.vns = g_gu.ns;
        d.vstride = 2 * P.ffn;
      }
      d.part = P.ws.f_part;
      d.pstride = dm;
    }
  }

  // ---- ranges ----
  // A GEMV CTA owns whole segments: units [a, b) of the phase order.
  __device__ void gemv_cta_range(const PD& d, long long& a, long long& b) const {
    if (cta < d.g.nca) {
      a = rstart(d.g.nseg, d.g.nca, cta) * d.g.kps;
      b = rstart(d.g.nseg, d.g.nca, cta + 1) * d.g.kps;
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
  // Every warp walks its own unit stream across phases with a cursor and keeps
  // its NSLOT-slot ring full: it refills a slot with its next unit as soon as
  // it has consumed it, so copies for the next phase are already in flight
  // while the CTA waits at a barrier.
  __device__ __noinline__ Cursor cur_enter(int p, int w) const {
    Cursor c;
    memset(&c, 0, sizeof(c));
    c.p = p;
    if (p >= P.phase_end) {
      c.kind = -1;
      return c;
    }
    PD d;
    get_phase(p, d);
    c.kind = d.kind;
    if (d.kind == PK_GEMV_W4 || d.kind == PK_GEMV_BF16) {
      long long a, b, wa, wb;
      gemv_cta_range(d, a, b);
      warp_range(a, b, w, wa, wb);
      c.p0 = d.blob;
      c.x0 = d.ub;
      c.x1 = d.g.nkc;
      c.x2 = d.g.kps;
      c.x3 = d.g.nrb;
      c.i = int(wa);
      c.end = int(wb);
      const int upsl = d.g.nrb * d.g.kps;
      c.x4 = c.i / upsl;
      const int r = c.i - c.x4 * upsl;
      c.x5 = r / d.g.kps;
      c.x6 = r - c.x5 * d.g.kps;
    } else if (d.kind == PK_ATTN) {
      long long a, b;
      int nca;
      attn_cta_range(d, a, b, nca);
      c.i = int(a);
      c.end = int(b);
      c.p0 = d.kc;
      c.p1 = d.vc;
      c.x0 = d.slots;
      c.x1 = d.seqoff;
      c.x2 = d.type;
      c.x3 = 0;
    }
    return c;
  }
  // The next unit of warp w's stream at or after c (possibly in a later
  // phase); kind < 0 when the launch has no more.
  __device__ __noinline__ Cursor cur_normalize(Cursor c, int w) const {
    for (;;) {
      if (c.kind < 0) return c;
      if (c.kind == PK_GEMV_W4 || c.kind == PK_GEMV_BF16) {
        if (c.i < c.end) return c;
      } else if (c.kind == PK_ATTN) {
        const int* st = sst(c.x2);
        while (c.i < c.end) {
          while (st[c.x3 + 1] <= c.i) ++c.x3;
          const int key0 = (c.i - st[c.x3]) * ATT_CTA_KEYS + w * ATT_KEYS;
          if (key0 < Lb(c.x2)[c.x3 / P.nkv]) return c;
          ++c.i;
        }
      }
      c = cur_enter(c.p + 1, w);
    }
  }
  __device__ __forceinline__ void cur_advance(Cursor& c) const {
    ++c.i;
    if (c.kind == PK_GEMV_W4 || c.kind == PK_GEMV_BF16) {
      if (++c.x6 == c.x2) {
        c.x6 = 0;
        if (++c.x5 == c.x3) {
          c.x5 = 0;
          ++c.x4;
        }
      }
      if (c.i < c.end) return;  // fast path: same phase
    }
    c = cur_normalize(c, warp);
  }
  __device__ __forceinline__ void cur_src(const Cursor& c, const uint8_t*& s1, const uint8_t*& s2,
                                          uint32_t& bytes) const {
    if (c.kind == PK_GEMV_W4 || c.kind == PK_GEMV_BF16) {
      s1 = c.p0 + ((size_t)c.x5 * c.x1 + c.x4 * c.x2 + c.x6) * c.x0;
      s2 = nullptr;
      bytes = c.x0;
    } else {
      const int* st = sst(c.x2);
      const int bq = c.x3 / P.nkv, g = c.x3 - bq * P.nkv;
      const int key0 = (c.i - st[c.x3]) * ATT_CTA_KEYS + warp * ATT_KEYS;
      const size_t row = ((size_t)(c.x1 + bq) * P.nkv + g) * c.x0 + key0;
      bytes = ATT_KEYS * HD * 2;
      s1 = c.p0 + row * HD * 2;
      s2 = c.p1 + row * HD * 2;
    }
  }
  __device__ __forceinline__ RingCtx ringctx() const {
    RingCtx R;
    R.base = sm + L::RING + warp * NSLOT * SLOT_BYTES;
    R.bar = fullb(warp, 0);
    R.err = P.ws.ctl + 2;
    R.lane = lane;
    return R;
  }
  __device__ __forceinline__ void loader_issue(const RingCtx& R, Stream& S) const {
    const int sl = S.issued % NSLOT;
    const uint8_t *s1, *s2;
    uint32_t bytes;
    cur_src(S.ld, s1, s2, bytes);
    if (R.lane == 0) {
      uint64_t* bar = R.bar + sl;
      uint8_t* dst = R.base + sl * SLOT_BYTES;
      mbar_expect_tx(bar, s2 ? 2 * bytes : bytes);
      bulk_g2s(dst, s1, bytes, bar);
      if (s2) bulk_g2s(dst + bytes, s2, bytes, bar);
    }
    ++S.issued;
    cur_advance(S.ld);
  }
  __device__ Stream loader_start() const {
    Stream S;
    S.consumed = S.issued = 0;
    S.bad = false;
    S.ld = cur_normalize(cur_enter(P.phase_begin, warp), warp);
    const RingCtx R = ringctx();
    for (int i = 0; i < NSLOT && S.ld.kind >= 0; ++i) loader_issue(R, S);
    return S;
  }

  // ---- ring consumption ----
  __device__ __forceinline__ static const uint8_t* wait_slot(const RingCtx& R, Stream& S) {
    const int sl = S.consumed % NSLOT;
    const uint32_t par = (S.consumed / NSLOT) & 1u;
    if (!S.bad && !mbar_try_wait(R.bar + sl, par)) {
      const long long t0 = clock64();
      while (!mbar_try_wait(R.bar + sl, par)) {
        if (clock64() - t0 > WAIT_CYCLES) {
          if (R.lane == 0) atomicOr(R.err, EW_MBAR_TIMEOUT);
          S.bad = true;
          break;
        }
      }
    }
    return R.base + sl * SLOT_BYTES;
  }
  // Hand the slot back and refill it with the warp's next unit.
  __device__ __forceinline__ void release_slot(const RingCtx& R, Stream& S, bool wrote_slot = false) const {
    // order generic accesses of the slot before the async re-fill (every lane
    // when lanes wrote into the slot, else lane 0 after the warp's reads)
    if (wrote_slot) fence_proxy_async();
    __syncwarp();
    if (!wrote_slot && R.lane == 0) fence_proxy_async();
    ++S.consumed;
    if (S.ld.kind >= 0 && !S.bad) loader_issue(R, S);
  }
  __device__ void drain(Stream& S) const {
    const RingCtx R = ringctx();
    while (S.consumed < S.issued) {
      const int sl = S.consumed % NSLOT;
      const uint32_t par = (S.consumed / NSLOT) & 1u;
      const long long t0 = clock64();
      while (!mbar_try_wait(R.bar + sl, par)) {
        if (clock64() - t0 > WAIT_CYCLES) {
          if (R.lane == 0) atomicOr(R.err, EW_DRAIN_TIMEOUT);
          return;
        }
      }
      ++S.consumed;
    }
  }

  // ---- grid barrier ----
  __device__ __noinline__ bool grid_wait(uint32_t target) {
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
    cbar();
    return flags()[0] != 0;
  }
  __device__ void grid_arrive() {
    cbar();
    if (tid == 0) {
      __threadfence();
      red_release_add(P.ws.ctl, 1u);
    }
  }

  // Deterministic per-batch-row totals of the per-warp slots wsum[warp][b].
  __device__ void block_rows_total(const float* wsum, float* out, int B) const {
    cbar();
    if (tid < B) {
      float s = 0.f;
      for (int w = 0; w < NW; ++w) s += wsum[w * MAX_B + tid];
      out[tid] = s;
    }
    cbar();
  }

  // ---- GEMV input staging ----
  __device__ int clamp_token(int bb) const {
    const int tok = P.tokens[bb];
    return tok < 0 ? 0 : (tok >= P.vocab ? P.vocab - 1 : tok);
  }
  // Eight consecutive values x[bb][k0 .. k0 + 8) (k0 % 8 == 0) of a 16-bit source
  // or of the SiLU(gate) * up source, in fp32.
  __device__ void load_simple8(const PD& d, int bb, int k0, float (&v)[8]) const {
    if (d.xsrc == XS_SILU) {
      float g[8], u[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) g[i] = u[i] = 0.f;
      for (int s0 = 0; s0 < d.vns; s0 += 2) {
        float4 f[2][4];
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            f[i][q] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (s0 + i < d.vns)
              f[i][q] = __ldcg(reinterpret_cast<const float4*>(
                                   d.vpart + ((size_t)(s0 + i) * P.B + bb) * d.vstride + 2 * k0) + q);
          }
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (s0 + i < d.vns) {  // tiled rows 2j (gate j), 2j+1 (up j)
              g[2 * q] += f[i][q].x;
              u[2 * q] += f[i][q].y;
              g[2 * q + 1] += f[i][q].z;
              u[2 * q + 1] += f[i][q].w;
            }
          }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = g[i] / (1.f + expf(-g[i])) * u[i];
      return;
    }
    cvt16(d.xsrc == XS_F16, load_raw16(d, bb, k0), v);
  }
  // Eight 16-bit values of a bf16 / fp16 / embedding source, undecoded.
  __device__ __forceinline__ uint4 load_raw16(const PD& d, int bb, int k0) const {
    if (d.xsrc == XS_EMBED)
      return __ldg(reinterpret_cast<const uint4*>(P.embed + (size_t)clamp_token(bb) * P.d + k0));
    return __ldcg(reinterpret_cast<const uint4*>(d.xbf + (size_t)bb * d.xbf_stride + k0));
  }
  __device__ __forceinline__ static void cvt16(bool f16, const uint4& u, float (&v)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint16_t lo = uint16_t(w[i] & 0xffffu), hi = uint16_t(w[i] >> 16);
      v[2 * i] = f16 ? half_bits_to_f32(lo) : bf16_to_f32(lo);
      v[2 * i + 1] = f16 ? half_bits_to_f32(hi) : bf16_to_f32(hi);
    }
  }
  // Sum of the branch slabs for x[bb][k0 .. k0 + 8), in slab order (loads of
  // up to four slabs in flight at once).
  __device__ void load_branch8(const PD& d, int bb, int k0, float (&v)[8]) const {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.f;
    const float* base = d.vpart + (size_t)bb * d.vstride + k0;
    const size_t sstride = (size_t)P.B * d.vstride;
    for (int s0 = 0; s0 < d.vns; s0 += 4) {
      float4 a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = b[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (s0 + i < d.vns) {
          const float4* pr = reinterpret_cast<const float4*>(base + (s0 + i) * sstride);
          a[i] = __ldcg(pr);
          b[i] = __ldcg(pr + 1);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (s0 + i < d.vns) {
          v[0] += a[i].x;
          v[1] += a[i].y;
          v[2] += a[i].z;
          v[3] += a[i].w;
          v[4] += b[i].x;
          v[5] += b[i].y;
          v[6] += b[i].z;
          v[7] += b[i].w;
        }
      }
    }
  }
  __device__ static void load8f(const float* p, float (&v)[8], bool ro) {
    const float4* q = reinterpret_cast<const float4*>(p);
    const float4 a = ro ? __ldg(q) : __ldcg(q);
    const float4 b = ro ? __ldg(q + 1) : __ldcg(q + 1);
    v[0] = a.x;
    v[1] = a.y;
    v[2] = a.z;
    v[3] = a.w;
    v[4] = b.x;
    v[5] = b.y;
    v[6] = b.z;
    v[7] = b.w;
  }

  // Store a chunk of eight activations in fragment order.  The 16 lanes of a
  // half-warp hold one 128-group, whose sum (of the stored, rounded values)
  // and max |x| they reduce here.  Warp-uniform: every lane calls it.
  __device__ void emit_chunk(bool valid, int bb, int kl0, int xrow, const float (&v)[8], bool f16, float scale,
                             bool track_max) const {
    uint32_t* xw = xs();
    float s8 = 0.f, m8 = 0.f;
    if (valid) {
      const int ks = kl0 >> 4, hi = (kl0 >> 3) & 1;
      const int base = bb * xrow + ((ks >> 1) * 4) * 4 + (ks & 1) * 2 + hi;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float a = v[2 * t] * scale, b = v[2 * t + 1] * scale;
        uint32_t w;
        if (f16) {
          const uint16_t ha = f32_to_f16(a), hb = f32_to_f16(b);
          w = uint32_t(ha) | (uint32_t(hb) << 16);
          s8 += half_bits_to_f32(ha) + half_bits_to_f32(hb);
        } else {
          const uint16_t ha = f32_to_bf16(a), hb = f32_to_bf16(b);
          w = uint32_t(ha) | (uint32_t(hb) << 16);
          s8 += bf16_to_f32(ha) + bf16_to_f32(hb);
        }
        xw[base + t * 4] = w;
        m8 = fmaxf(m8, fmaxf(fabsf(v[2 * t]), fabsf(v[2 * t + 1])));
      }
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) {
      s8 += __shfl_xor_sync(0xffffffffu, s8, o);
      m8 = fmaxf(m8, __shfl_xor_sync(0xffffffffu, m8, o));
    }
    if (valid && (lane & 15) == 0) {
      xsum()[(kl0 >> 7) * (8 * NB) + bb] = s8;
      if (track_max) atomicMax(reinterpret_cast<uint32_t*>(red() + 32) + bb, __float_as_uint(m8));
    }
  }

  __device__ __noinline__ void fill_x(const PD& d, long long a, long long b, int& kbase, int& klen) {
    const int B = P.B, dm = P.d;
    kbase = 0;
    klen = 0;
    if (a < b) {
      const long long upsl = (long long)d.g.nrb * d.g.kps;
      const int KS = d.g.kps * d.kcw;
      const int s0 = int(a / upsl), s1 = int((b - 1) / upsl);
      kbase = s0 * KS;
      klen = (s1 - s0 + 1) * KS;
    }
    if (!x_fits(klen, B, NB)) {  // the host sizes slabs so this never happens
      if (tid == 0) set_error(EW_BAD_SHAPE);
      klen = 0;
    }
    const bool f16 = (d.kind == PK_GEMV_W4);
    float* rd = red();
    float* xscale = rd + 48;  // 2^e per batch row
    float* xsm = xsum();
    for (int i = tid; i < XSUM_BYTES / 4; i += NT) xsm[i] = 0.f;
    if (tid < MAX_B) {
      reinterpret_cast<uint32_t*>(rd + 32)[tid] = 0u;
      xscale[tid] = 1.f;
    }
    float* wsum = wsp();   // [NW][MAX_B] per-warp partial sums of squares
    for (int w = tid; w < NW * MAX_B; w += NT) wsum[w] = 0.f;
    cbar();
    const int xrow = klen / 2 + 16;
    const bool has_out = (d.xdst != nullptr || d.dump != nullptr);
    const int nout = B * dm / 8;
    const int out_per = (nout + P.nc - 1) / P.nc;
    const int o0 = cta * out_per, o1 = min(nout, o0 + out_per);

    if (d.xsrc == XS_RESID || d.xsrc == XS_FINAL) {
      // Residual update over the whole width: v = sum of the branch slabs,
      // x = xres + v * rsqrt(mean(v^2) + eps) * gain  [then the final norm].
      const int n8 = dm / 8, total8 = B * n8;
      const bool fin = (d.xsrc == XS_FINAL) && d.gain2 != nullptr;
      // pass 1: sums of squares of v per batch row (a warp iteration covers 32
      // consecutive chunks of one batch row since d % 256 == 0)
      for (int j = 0; warp * 32 + j * NT < total8; ++j) {
        const int cw = warp * 32 + j * NT, c = cw + lane;
        const int bb = cw / n8;
        const int k0 = (c - bb * n8) * 8;
        float v[8];
        load_branch8(d, bb, k0, v);
        float sq = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) sq = fmaf(v[i], v[i], sq);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (lane == 0) wsum[warp * MAX_B + bb] += sq;
      }
      block_rows_total(wsum, rd, B);
      if (tid < B) rd[tid] = rsqrtf(rd[tid] / float(dm) + P.eps);
      cbar();
      // x = xres + v * r * gain (v re-read: the slabs are L2-resident)
      auto x1_of = [&](int bb, int k0, float (&x)[8]) {
        float v[8], xr[8], g[8];
        load_branch8(d, bb, k0, v);
        load8f(d.xres + (size_t)bb * dm + k0, xr, false);
        load8f(d.gain + k0, g, true);
        const float r = rd[bb];
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = fmaf(v[i] * r, g[i], xr[i]);
      };
      if (fin) {
        // pass 2: the final norm's sums of squares
        for (int w = tid; w < NW * MAX_B; w += NT) wsum[w] = 0.f;
        cbar();
        for (int j = 0; warp * 32 + j * NT < total8; ++j) {
          const int cw = warp * 32 + j * NT, c = cw + lane;
          const int bb = cw / n8;
          float x[8];
          x1_of(bb, (c - bb * n8) * 8, x);
          float sq = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) sq = fmaf(x[i], x[i], sq);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
          if (lane == 0) wsum[warp * MAX_B + bb] += sq;
        }
        block_rows_total(wsum, rd + 16, B);
        if (tid < B) rd[16 + tid] = rsqrtf(rd[16 + tid] / float(dm) + P.eps);
        cbar();
      }
      // pass 3: convert the k-range, write the residual copy / dump slice
      for (int j = 0; warp * 32 + j * NT < total8; ++j) {
        const int cw = warp * 32 + j * NT, c = cw + lane;
        const int bb = cw / n8;
        const int k0 = (c - bb * n8) * 8;
        float x[8];
        x1_of(bb, k0, x);
        if (has_out && c >= o0 && c < o1) {
          const size_t o = (size_t)bb * dm + k0;
          const float4 lo = make_float4(x[0], x[1], x[2], x[3]), hi = make_float4(x[4], x[5], x[6], x[7]);
          if (d.xdst) {
            reinterpret_cast<float4*>(d.xdst + o)[0] = lo;
            reinterpret_cast<float4*>(d.xdst + o)[1] = hi;
          }
          if (d.dump) {
            reinterpret_cast<float4*>(d.dump + o)[0] = lo;
            reinterpret_cast<float4*>(d.dump + o)[1] = hi;
          }
        }
        if (fin) {
          float g2[8];
          load8f(d.gain2 + k0, g2, true);
          const float rf = rd[16 + bb];
#pragma unroll
          for (int i = 0; i < 8; ++i) x[i] = x[i] * rf * g2[i];
        }
        // half-warps are uniformly inside or outside (128-aligned k-range)
        const bool inside = k0 >= kbase && k0 < kbase + klen;
        emit_chunk(inside, bb, k0 - kbase, xrow, x, f16, 1.f, f16);
      }
    } else {
      // 16-bit / SiLU sources: the k-range only, several chunks per thread in flight
      const int n8 = klen / 8, total8 = B * n8;
      if (d.xsrc != XS_SILU) {
        constexpr int JU = 4;
        for (int j0 = 0; warp * 32 + j0 * NT < total8; j0 += JU) {
          uint4 raw[JU];
#pragma unroll
          for (int jj = 0; jj < JU; ++jj) {
            const int c = warp * 32 + (j0 + jj) * NT + lane;
            raw[jj] = make_uint4(0u, 0u, 0u, 0u);
            if (c < total8) {
              const int bb = c / n8;
              raw[jj] = load_raw16(d, bb, kbase + (c - bb * n8) * 8);
            }
          }
#pragma unroll
          for (int jj = 0; jj < JU; ++jj) {
            const int cw = warp * 32 + (j0 + jj) * NT;
            if (cw < total8) {  // warp-uniform
              const int c = cw + lane;
              const int bb = c / n8;
              float v[8];
              cvt16(d.xsrc == XS_F16, raw[jj], v);
              emit_chunk(c < total8, bb, (c - bb * n8) * 8, xrow, v, f16, 1.f, f16);
            }
          }
        }
      } else {
        constexpr int JU = 2;
        for (int j0 = 0; warp * 32 + j0 * NT < total8; j0 += JU) {
          float v[JU][8];
#pragma unroll
          for (int jj = 0; jj < JU; ++jj) {
            const int c = warp * 32 + (j0 + jj) * NT + lane;
            if (c < total8) {
              const int bb = c / n8;
              load_simple8(d, bb, kbase + (c - bb * n8) * 8, v[jj]);
            }
          }
#pragma unroll
          for (int jj = 0; jj < JU; ++jj) {
            const int cw = warp * 32 + (j0 + jj) * NT;
            if (cw < total8) {  // warp-uniform
              const int c = cw + lane;
              const int bb = c / n8;
              emit_chunk(c < total8, bb, (c - bb * n8) * 8, xrow, v[jj], f16, 1.f, f16);
            }
          }
        }
      }
      // residual copy / dump of the embedding (first layer)
      if (has_out) {
        for (int c = o0 + tid; c < o1; c += NT) {
          const int bb = (c * 8) / dm, k0 = c * 8 - bb * dm;
          float v[8];
          load_simple8(d, bb, k0, v);
          const float4 lo = make_float4(v[0], v[1], v[2], v[3]), hi = make_float4(v[4], v[5], v[6], v[7]);
          if (d.xdst) {
            reinterpret_cast<float4*>(d.xdst + (size_t)bb * dm + k0)[0] = lo;
            reinterpret_cast<float4*>(d.xdst + (size_t)bb * dm + k0)[1] = hi;
          }
          if (d.dump) {
            reinterpret_cast<float4*>(d.dump + (size_t)bb * dm + k0)[0] = lo;
            reinterpret_cast<float4*>(d.dump + (size_t)bb * dm + k0)[1] = hi;
          }
        }
      }
      if (cta == 0 && tid == 0 && d.xsrc == XS_EMBED) {
        for (int bb = 0; bb < B; ++bb)
          if (P.tokens[bb] < 0 || P.tokens[bb] >= P.vocab) set_error(EW_BAD_SHAPE);
      }
    }
    cbar();
    if (f16) {
      // fp16 range guard: rows whose max |x| reaches 2^15 are re-staged scaled
      // by an exact power of two, undone on the partial sums in flush().
      const uint32_t* xmax = reinterpret_cast<const uint32_t*>(rd + 32);
      bool any = false;
      for (int bb = 0; bb < B; ++bb) any |= __uint_as_float(xmax[bb]) >= 32768.f;
      if (any) restage_scaled(d, kbase, klen, xrow);
    }
  }

  // Rare path of the fp16 range guard.
  __device__ __noinline__ void restage_scaled(const PD& d, int kbase, int klen, int xrow) {
    const int B = P.B, dm = P.d;
    float* rd = red();
    const uint32_t* xmax = reinterpret_cast<const uint32_t*>(rd + 32);
    float* xscale = rd + 48;
    const int n8 = klen / 8, total8 = B * n8;
    for (int j = 0; warp * 32 + j * NT < total8; ++j) {
      const int cw = warp * 32 + j * NT, c = cw + lane;
      const int bb = cw / n8;  // n8 % 32 == 0: one batch row per warp iteration
      const float mx = __uint_as_float(xmax[bb]);
      if (!(mx >= 32768.f)) continue;  // warp-uniform
      int ex;
      frexpf(mx, &ex);
      const int k0 = kbase + (c - bb * n8) * 8;
      float v[8];
      if (d.xsrc == XS_RESID || d.xsrc == XS_FINAL) {
        float br[8], xr[8], g[8];
        load_branch8(d, bb, k0, br);
        load8f(d.xres + (size_t)bb * dm + k0, xr, false);
        load8f(d.gain + k0, g, true);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = fmaf(br[i] * rd[bb], g[i], xr[i]);
        if (d.xsrc == XS_FINAL && d.gain2 != nullptr) {
          load8f(d.gain2 + k0, g, true);
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] *= rd[16 + bb] * g[i];
        }
      } else {
        load_simple8(d, bb, k0, v);
      }
      emit_chunk(true, bb, k0 - kbase, xrow, v, true, ldexpf(1.f, 15 - ex), false);
    }
    cbar();
    if (tid < B) {
      const float mx = __uint_as_float(xmax[tid]);
      if (mx >= 32768.f) {
        int ex;
        frexpf(mx, &ex);
        xscale[tid] = ldexpf(1.f, ex - 15);
      }
    }
    cbar();
  }

  // ---- GEMV outputs ----
  // Rows of 16-row block rb of slab s, fragment layout v[nb][0..3] = (row g,
  // col 2t), (g, 2t+1), (g+8, 2t), (g+8, 2t+1), columns = batch nb*8 + ...
  __device__ __noinline__ void finalize(const PD& d, int s, int rb, Acc<NB> A) const {
    const float (&v)[NB][4] = A.v;
    const int g = lane >> 2, t = lane & 3, B = P.B;
    const int r0 = rb * RB + g, r1 = r0 + 8;
    if (d.epi == EPI_PART) {
      float* base = d.part + (size_t)s * B * d.pstride;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const int b0 = nb * 8 + 2 * t, b1 = b0 + 1;
        if (r0 < d.rows_valid) {
          if (b0 < B) base[(size_t)b0 * d.pstride + r0] = v[nb][0];
          if (b1 < B) base[(size_t)b1 * d.pstride + r0] = v[nb][1];
        }
        if (r1 < d.rows_valid) {
          if (b0 < B) base[(size_t)b0 * d.pstride + r1] = v[nb][2];
          if (b1 < B) base[(size_t)b1 * d.pstride + r1] = v[nb][3];
        }
      }
      return;
    }
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
          const float h0 = v[nb][0] / (1.f + expf(-v[nb][0])) * u0;
          const float h1 = v[nb][1] / (1.f + expf(-v[nb][1])) * u1;
          const float h2 = v[nb][2] / (1.f + expf(-v[nb][2])) * u2;
          const float h3 = v[nb][3] / (1.f + expf(-v[nb][3])) * u3;
          if (b0 < B) {
            d.hout[(size_t)b0 * d.hstride + j0] = d.out_f16 ? f32_to_f16(h0) : f32_to_bf16(h0);
            d.hout[(size_t)b0 * d.hstride + j1] = d.out_f16 ? f32_to_f16(h2) : f32_to_bf16(h2);
          }
          if (b1 < B) {
            d.hout[(size_t)b1 * d.hstride + j0] = d.out_f16 ? f32_to_f16(h1) : f32_to_bf16(h1);
            d.hout[(size_t)b1 * d.hstride + j1] = d.out_f16 ? f32_to_f16(h3) : f32_to_bf16(h3);
          }
        }
      }
      return;
    }
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
  __device__ void emit_segment(const PD& d, int seg, const Acc<NB>& A) const {
    const int s = seg / d.g.nrb, rb = seg - s * d.g.nrb;
    finalize(d, s, rb, A);
  }

  __device__ static Acc<NB> to_acc(const float (&a)[NB][4]) {
    Acc<NB> r;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int j = 0; j < 4; ++j) r.v[nb][j] = a[nb][j];
    return r;
  }

  // A segment piece leaves the warp: undo the range scaling, then emit it
  // (segment wholly inside this warp) or park it in the warp's slot.
  __device__ __noinline__ void flush(const PD& d, int seg, Acc<NB> A, int wa, int wb, float* my) const {
    if (d.kind == PK_GEMV_W4) {
      const float* xscale = red() + 48;
      const int t = lane & 3;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const float s0 = xscale[nb * 8 + 2 * t], s1 = xscale[nb * 8 + 2 * t + 1];
        A.v[nb][0] *= s0;
        A.v[nb][1] *= s1;
        A.v[nb][2] *= s0;
        A.v[nb][3] *= s1;
      }
    }
    const int u0 = seg * d.g.kps;
    if (u0 >= wa && u0 + d.g.kps <= wb) {
      emit_segment(d, seg, A);
    } else {
      const int sl = (seg == wa / d.g.kps) ? 0 : 1;
      float* q = my + sl * (32 * 4 * NB) + lane * 4 * NB;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
        reinterpret_cast<float4*>(q)[nb] = make_float4(A.v[nb][0], A.v[nb][1], A.v[nb][2], A.v[nb][3]);
    }
  }

  // Segments of this CTA split between warps: sum the pieces in warp order.
  __device__ __noinline__ void cta_combine(const PD& d, int a, int b) const {
    const int kps = d.g.kps;
    int count = 0, last = -1;
    for (int w = 0; w < NW; ++w) {
      long long wa64, wb64;
      warp_range(a, b, w, wa64, wb64);
      const int wa = int(wa64), wb = int(wb64);
      if (wa >= wb) continue;
      const int fs = wa / kps, ls = (wb - 1) / kps;
      for (int which = 0; which < 2; ++which) {
        const int S = which ? ls : fs;
        if (which && ls == fs) break;
        const bool complete = (S * kps >= wa) && (S * kps + kps <= wb);
        if (complete || S == last) continue;
        if (count % NW == warp) {
          Acc<NB> sum;
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) sum.v[nb][0] = sum.v[nb][1] = sum.v[nb][2] = sum.v[nb][3] = 0.f;
          for (int w2 = 0; w2 < NW; ++w2) {
            long long a2, b2;
            warp_range(a, b, w2, a2, b2);
            if (a2 >= b2 || S * kps >= b2 || S * kps + kps <= a2) continue;
            const int sl = (S == int(a2) / kps) ? 0 : 1;
            const float* q = wsp() + w2 * (2 * 32 * 4 * NB) + sl * (32 * 4 * NB) + lane * 4 * NB;
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
              const float4 f = reinterpret_cast<const float4*>(q)[nb];
              sum.v[nb][0] += f.x;
              sum.v[nb][1] += f.y;
              sum.v[nb][2] += f.z;
              sum.v[nb][3] += f.w;
            }
          }
          emit_segment(d, S, sum);
        }
        ++count;
        last = S;
      }
    }
  }

  __device__ __forceinline__ void run_gemv(const PD& d, Stream& S) {
    long long a, b;
    gemv_cta_range(d, a, b);
    int kbase, klen;
    fill_x(d, a, b, kbase, klen);
    mark(1);
    if (a >= b) return;
    long long wa64, wb64;
    warp_range(a, b, warp, wa64, wb64);
    S = gemv_loop(S, d, kbase, klen, int(wa64), int(wb64));
    cbar();
    mark(2);
    cta_combine(d, int(a), int(b));
  }

  // This warp's units [wa, wb) of a GEMV phase.  Its own (non-inlined) function
  // so that the loop's registers are allocated for the loop alone.
  __device__ __noinline__ Stream gemv_loop(Stream S, const PD& d, int kbase, int klen, int wa, int wb) const {
    const RingCtx R = ringctx();
    const uint4* xs4 = reinterpret_cast<const uint4*>(xs());
    const int xrow4 = (klen / 2 + 16) / 4;
    const float* xsm = xsum();
    const int kps = d.g.kps, nrb = d.g.nrb, kcw = d.kcw, B = P.B;
    const int upsl = nrb * kps;
    int u = wa;
    int s_ = u / upsl;
    int rb = (u - s_ * upsl) / kps;
    int kci = u - s_ * upsl - rb * kps;
    float acc[NB][4];
    int cur = -1;
    float* my = wsp() + warp * (2 * 32 * 4 * NB);
    const bool w4 = (d.kind == PK_GEMV_W4);
    const int ln = R.lane;
    for (; u < wb; ++u) {
      const int seg = s_ * nrb + rb;
      if (seg != cur) {
        if (cur >= 0) flush(d, cur, to_acc(acc), wa, wb, my);
        cur = seg;
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0.f;
      }
      const int koff = (s_ * kps + kci) * kcw - kbase;
      const uint8_t* slot = wait_slot(R, S);
      if (w4)
        w4_unit<NB>(slot, xs4, xrow4, koff >> 4, xsm, koff >> 7, acc, B, ln);
      else
        bf_unit<NB>(slot, xs4, xrow4, koff >> 4, acc, B, ln);
      release_slot(R, S);
      if (++kci == kps) {
        kci = 0;
        if (++rb == nrb) {
          rb = 0;
          ++s_;
        }
      }
    }
    if (cur >= 0) flush(d, cur, to_acc(acc), wa, wb, my);
    return S;
  }

  // Standalone GEMV with K split into slabs: y = sum of the slab rows in
  // order, then the requested epilogue.
  __device__ __noinline__ void run_reduce() const {
    const int B = P.B, n = P.g_n;
    const int ns = P.geo[0].ns;
    const float* part = P.ws.g_part;
    if (P.g_epi == W4A_EPI_SILU_MUL) {
      const int nh = n / 2, total = B * nh;
      for (int i = cta * NT + tid; i < total; i += P.nc * NT) {
        const int bb = i / nh, j = i - bb * nh;
        float gsum = 0.f, usum = 0.f;
        for (int s = 0; s < ns; ++s) {
          gsum += __ldcg(part + ((size_t)s * B + bb) * n + 2 * j);
          usum += __ldcg(part + ((size_t)s * B + bb) * n + 2 * j + 1);
        }
        reinterpret_cast<uint16_t*>(P.g_out)[(size_t)bb * nh + j] = f32_to_bf16(gsum / (1.f + expf(-gsum)) * usum);
      }
      return;
    }
    // one thread per (batch row, 16-row block): plain rows and their sum of squares
    const int nrb = n / RB, total = B * nrb;
    for (int i = cta * NT + tid; i < total; i += P.nc * NT) {
      const int bb = i / nrb, rb = i - bb * nrb;
      float ss = 0.f;
      for (int r = rb * RB; r < rb * RB + RB; ++r) {
        float y = 0.f;
        for (int s = 0; s < ns; ++s) y += __ldcg(part + ((size_t)s * B + bb) * n + r);
        reinterpret_cast<float*>(P.g_out)[(size_t)bb * n + r] = y;
        ss = fmaf(y, y, ss);
      }
      if (P.g_epi == W4A_EPI_SUMSQ) P.g_aux[(size_t)rb * B + bb] = ss;
    }
  }

  // ---- attention phase ----
  __device__ __noinline__ void attn_prologue(const PD& d, int seg, bool own_new) {
    const int bq = seg / P.nkv, g = seg % P.nkv;
    const int GQ = P.nq / P.nkv;
    float* q = qs();
    float* rd = red();
    const float qscale = 1.4426950408889634f * rsqrtf(float(HD));
    if (d.newkv) {
      // q, k, v of this sequence are the sums of the QKV slabs (four-row
      // chunks, several in flight per thread); the norms run over the whole Q
      // and K projections.  This group's k and v rows go to scratch.
      const int qd = P.nq * HD, kd = P.nkv * HD, qkv_dim = qd + 2 * kd;
      const float* ybase = d.qpart + (size_t)bq * qkv_dim;
      const size_t sstride = (size_t)P.B * qkv_dim;
      float* kraw = wsp() + 64;
      float* vraw = kraw + HD;
      const int nq4 = qd / 4, nk4 = kd / 4;
      const int total4 = nq4 + (own_new ? nk4 + HD / 4 : 0);
      float sq = 0.f, sk = 0.f;
      constexpr int JU = 4;
      for (int c0 = tid; c0 < total4; c0 += JU * NT) {
        int rows[JU];
        float4 v[JU];
#pragma unroll
        for (int j = 0; j < JU; ++j) {
          const int c = c0 + j * NT;
          rows[j] = c < nq4 + nk4 ? 4 * c : qd + kd + g * HD + 4 * (c - nq4 - nk4);
          v[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int sl = 0; sl < d.qns; ++sl) {
          float4 t[JU];
#pragma unroll
          for (int j = 0; j < JU; ++j)
            t[j] = (c0 + j * NT < total4) ? __ldcg(reinterpret_cast<const float4*>(ybase + sl * sstride + rows[j]))
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int j = 0; j < JU; ++j) {
            v[j].x += t[j].x;
            v[j].y += t[j].y;
            v[j].z += t[j].z;
            v[j].w += t[j].w;
          }
        }
#pragma unroll
        for (int j = 0; j < JU; ++j) {
          if (c0 + j * NT >= total4) continue;
          const int r = rows[j];
          const float ss = v[j].x * v[j].x + v[j].y * v[j].y + v[j].z * v[j].z + v[j].w * v[j].w;
          float* dst = nullptr;
          if (r < qd) {
            sq += ss;
            const int h = r / HD - g * GQ;
            if (h >= 0 && h < GQ) dst = q + (r - g * GQ * HD);
          } else if (r < qd + kd) {
            sk += ss;
            if ((r - qd) / HD == g) dst = kraw + (r - qd - g * HD);
          } else {
            dst = vraw + (r - qd - kd - g * HD);
          }
          if (dst) {
            dst[0] = v[j].x;
            dst[1] = v[j].y;
            dst[2] = v[j].z;
            dst[3] = v[j].w;
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        sq += __shfl_xor_sync(0xffffffffu, sq, o);
        sk += __shfl_xor_sync(0xffffffffu, sk, o);
      }
      float* wq = wsp();
      if (lane == 0) {
        wq[warp] = sq;
        wq[NW + warp] = sk;
      }
      cbar();
      if (tid == 0) {
        float a = 0.f, c = 0.f;
        for (int w = 0; w < NW; ++w) {
          a += wq[w];
          c += wq[NW + w];
        }
        rd[32] = rsqrtf(a / float(qd) + P.eps);
        rd[33] = rsqrtf(c / float(kd) + P.eps);
      }
      cbar();
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
        const float x1 = q[h * HD + i] * rq * qn[row + i];
        const float x2 = q[h * HD + i + H2] * rq * qn[row + i + H2];
        float c, s;
        rope_cs(pos, fr[i], ms, c, s);
        q[h * HD + i] = (x1 * c - x2 * s) * qscale;
        q[h * HD + i + H2] = (x2 * c + x1 * s) * qscale;
      }
      if (own_new) {
        for (int i = tid; i < H2; i += NT) {
          const float x1 = kraw[i] * rk * kg[g * HD + i];
          const float x2 = kraw[i + H2] * rk * kg[g * HD + i + H2];
          float c, s;
          rope_cs(pos, fr[i], ms, c, s);
          kn()[i] = f32_to_bf16(x1 * c - x2 * s);
          kn()[i + H2] = f32_to_bf16(x2 * c + x1 * s);
        }
        for (int i = tid; i < HD; i += NT) vn()[i] = f32_to_bf16(vraw[i]);
        cbar();
        const int sn_ = snew(d.type)[bq];
        const size_t row = ((size_t)(d.seqoff + bq) * P.nkv + g) * d.slots + sn_;
        uint16_t* kd_ = reinterpret_cast<uint16_t*>(const_cast<uint8_t*>(d.kc)) + row * HD;
        uint16_t* vd_ = reinterpret_cast<uint16_t*>(const_cast<uint8_t*>(d.vc)) + row * HD;
        for (int i = tid; i < HD; i += NT) {
          const int sw = (((i >> 3) ^ (sn_ & 7)) << 3) | (i & 7);
          kd_[sw] = kn()[i];
          vd_[sw] = vn()[i];
        }
      }
    } else {
      const uint16_t* qin = P.a_q + ((size_t)bq * P.nq + g * GQ) * HD;
      for (int idx = tid; idx < GQ * HD; idx += NT) q[idx] = bf16_to_f32(qin[idx]) * qscale;
    }
    cbar();
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
    cbar();
  }

  __device__ __forceinline__ void run_attn(const PD& d, Stream& S) {
    long long a, b;
    int nca;
    attn_cta_range(d, a, b, nca);
    if (a >= b) return;
    const int* st = sst(d.type);
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
      if (u == a) mark(1);
      S = attn_loop(S, d, seg, u, run_end, Lk, sn_, own_new);
      cbar();
      if (run_end == b) mark(2);
      attn_combine(d, seg, a, b, nca);
      cbar();
      u = run_end;
    }
  }

  // This warp's keys of CTA units [u, run_end) of segment seg; writes the
  // warp's (m, l, o) partial to shared memory.  Non-inlined for the same
  // reason as gemv_loop.
  __device__ __noinline__ Stream attn_loop(Stream S, const PD& d, int seg, long long u, long long run_end, int Lk,
                                           int sn_, bool own_new) const {
    const RingCtx R = ringctx();
    const int* st = sst(d.type);
    const int GQ = P.nq / P.nkv;
    constexpr int PW = MAX_GQ * (HD + 2);
    const int g = lane >> 2, t = lane & 3;
    const uint4* qfr = qf();
    float m = -INFINITY, lsum = 0.f;
    // O^T tiles: o[j] covers dims [16 j, 16 j + 16) x query heads 0..7 of the group
    float o[HD / 16][4];
#pragma unroll
    for (int j = 0; j < HD / 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    for (long long jc = u; jc < run_end; ++jc) {
      const int key0 = int(jc - st[seg]) * ATT_CTA_KEYS + warp * ATT_KEYS;
      if (key0 >= Lk) continue;
      uint8_t* slot = const_cast<uint8_t*>(wait_slot(R, S));
      uint8_t* Ks = slot;
      uint8_t* Vs = slot + ATT_KEYS * HD * 2;
      const bool patch = own_new && sn_ >= key0 && sn_ < key0 + ATT_KEYS;
      if (patch) {
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
      // S = Q K^T: rows = query heads (g), columns = the 8 keys (2t, 2t+1)
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
      // this lane's O^T columns are heads 2t and 2t+1: fetch their rescale factors
      const float a_lo = __shfl_sync(0xffffffffu, alpha, (2 * t) * 4);
      const float a_hi = __shfl_sync(0xffffffffu, alpha, (2 * t + 1) * 4);
#pragma unroll
      for (int j = 0; j < HD / 16; ++j) {
        o[j][0] *= a_lo;
        o[j][1] *= a_hi;
        o[j][2] *= a_lo;
        o[j][3] *= a_hi;
      }
      // O^T += V^T P^T: A = V^T from transposed 8x8 loads, B = (p0, p1) as hi + lo bf16
      uint32_t pa, pl;
      split_bf16x2(p0, p1, pa, pl);
#pragma unroll
      for (int q4 = 0; q4 < HD / 32; ++q4) {
        uint32_t v0, v1, v2, v3;
        ldsm_x4_t(v0, v1, v2, v3, Vs + r * HD * 2 + (((4 * q4 + mi) ^ r) << 4));
        mma_1688(o[2 * q4], v0, v1, pa);
        mma_1688(o[2 * q4], v0, v1, pl);
        mma_1688(o[2 * q4 + 1], v2, v3, pa);
        mma_1688(o[2 * q4 + 1], v2, v3, pl);
      }
      release_slot(R, S, patch);
    }
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
    float* wp = apw() + warp * PW;
#pragma unroll
    for (int j = 0; j < HD / 16; ++j) {
      if (2 * t < GQ) {
        wp[(2 * t) * (HD + 2) + 16 * j + g] = o[j][0];
        wp[(2 * t) * (HD + 2) + 16 * j + 8 + g] = o[j][2];
      }
      if (2 * t + 1 < GQ) {
        wp[(2 * t + 1) * (HD + 2) + 16 * j + g] = o[j][1];
        wp[(2 * t + 1) * (HD + 2) + 16 * j + 8 + g] = o[j][3];
      }
    }
    if (g < GQ && t == 0) {
      wp[g * (HD + 2) + HD] = m;
      wp[g * (HD + 2) + HD + 1] = lsum;
    }
    return S;
  }

  __device__ __noinline__ void attn_combine(const PD& d, int seg, long long a, long long b, int nca) {
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
    cbar();
    const long long total = st[P.B * P.nkv];
    const int c0 = owner(total, nca, st[seg]);
    const int c1 = owner(total, nca, st[seg + 1] - 1);
    if (tid == 0) {
      const uint32_t old = atomicAdd(P.ws.seg_ctr + seg, 1u);
      flags()[1] = (int(old) == c1 - c0) ? 1 : 0;
    }
    cbar();
    if (!flags()[1]) return;
    __threadfence();
    // warp h combines query head h over the pieces c0..c1 (one piece per lane
    // for the max and the denominators; shuffled weights for the outputs)
    if (warp < GQ) {
      const int h = warp;
      auto piece_of = [&](int c) {
        const int sl = (st[seg] < rstart(total, nca, c)) ? 0 : 1;
        return P.ws.apart + ((size_t)c * 2 + sl) * PW + h * (HD + 2);
      };
      float M = -INFINITY;
      for (int c = c0 + lane; c <= c1; c += 32) M = fmaxf(M, __ldcg(piece_of(c) + HD));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      constexpr int DPL = HD / 32;  // dims per lane
      float acc[DPL];
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
      float Lsum = 0.f;
      for (int cb = c0; cb <= c1; cb += 32) {
        const int cl = cb + lane;
        float ev = 0.f;
        if (cl <= c1) {
          const float* pc = piece_of(cl);
          ev = exp2f(__ldcg(pc + HD) - M);
          Lsum = fmaf(ev, __ldcg(pc + HD + 1), Lsum);
        }
        const int n = min(32, c1 - cb + 1);
#pragma unroll 4
        for (int i = 0; i < n; ++i) {
          const float w = __shfl_sync(0xffffffffu, ev, i);
          const float* pc = piece_of(cb + i) + lane * DPL;
#pragma unroll
          for (int e = 0; e < DPL; ++e) acc[e] = fmaf(w, __ldcg(pc + e), acc[e]);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, o);
      const float inv = 1.f / Lsum;
#pragma unroll
      for (int e = 0; e < DPL; ++e) {
        const float v = acc[e] * inv;
        out[h * HD + lane * DPL + e] = d.out_f16 ? f32_to_f16(v) : f32_to_bf16(v);
      }
    }
    if (tid == 0) P.ws.seg_ctr[seg] = 0u;
  }

  // ---- argmax phase (and the sum of the lm_head slabs when K was split) ----
  __device__ __noinline__ void run_argmax(const PD& d) {
    const int V = P.vocab, B = P.B;
    const int r0 = int(rstart(V, P.nc, cta)), r1 = int(rstart(V, P.nc, cta + 1));
    if (d.lpart != nullptr) {
      for (int bq = 0; bq < B; ++bq)
        for (int r = r0 + tid; r < r1; r += NT) {
          float y = 0.f;
          for (int s0 = 0; s0 < d.lns; s0 += 4) {
            float t[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              t[i] = (s0 + i < d.lns) ? __ldcg(d.lpart + ((size_t)(s0 + i) * B + bq) * V + r) : 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i)
              if (s0 + i < d.lns) y += t[i];
          }
          P.logits[(size_t)bq * V + r] = y;
        }
      cbar();
    }
    if (P.next_token == nullptr) return;
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
      cbar();
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
      cbar();
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
  __device__ __noinline__ void setup() {
    if (lane == 0) {
      for (int s = 0; s < NSLOT; ++s) mbar_init(fullb(warp, s), 1u);
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
    Stream S = loader_start();
    for (int p = P.phase_begin; p < P.phase_end; ++p) {
      if (p != P.phase_begin) {
        if (!grid_wait(uint32_t(p - P.phase_begin) * uint32_t(P.nc))) break;
      }
      cur_phase = p;
      mark(0);
      // the phase descriptor lives in shared memory (read by every warp)
      PD& d = *reinterpret_cast<PD*>(sm + L::PDS);
      if (tid == 0) get_phase(p, d);
      cbar();
      if (d.kind == PK_GEMV_W4 || d.kind == PK_GEMV_BF16)
        run_gemv(d, S);
      else if (d.kind == PK_ATTN)
        run_attn(d, S);
      else if (d.kind == PK_REDUCE)
        run_reduce();
      else
        run_argmax(d);
      grid_arrive();
      mark(3);
    }
    drain(S);
    cbar();
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

}  // namespace w4a
