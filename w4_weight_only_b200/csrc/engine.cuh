// The persistent decode engine.
//
// One CTA per SM, 16 warps: 15 math warps and a copy warp.  A launch runs a
// list of phases (decode: per layer QKV GEMV, GQA attention, O GEMV, gate/up
// GEMV, down GEMV; then lm_head and argmax) separated by grid-wide barriers.
// Every math warp consumes its own contiguous range of ~4 KB "units" (16
// weight rows x 512 int4 columns, 16 rows x 128 bf16 columns, or 8 keys of K
// and V) from a two-slot ring of shared memory; lane w of the copy warp walks
// math warp w's unit stream and issues each unit's bulk asynchronous copy
// (completing on an mbarrier) as soon as its slot is free, which the math
// warp signals once it has copied the unit into registers.  The stream runs
// across phase boundaries: weights and old KV entries do not depend on the
// activations, so the copies for phase p + 1 are in flight while the CTA
// waits at the barrier that ends phase p.
//
// Phase descriptors (what a phase reads, computes and writes) are built on the
// device at launch, in parallel by one thread per phase, into a table in the
// workspace; the CTA copies each descriptor into one of four shared-memory
// slots two phases before it runs, so the unit streams can look ahead.
//
// GEMV math: the int4 codes of a unit are laid out as mma.sync A fragments.
// A LOP3 turns each nibble q into the fp16 value 1024 + q (rows g) or
// 1024 + 16 q (rows g + 8, no shift needed), the tensor core accumulates
// sum_k (1024 + q) x_k in fp32 per 128-group, and the group is closed in fp32
// with s * (acc - (1024 + z) * sum_k x_k) (the 16x rows with s / 16 and
// 1024 + 16 z).  Within a unit the 512 columns are ordered so that each
// thread's activation fragments are 16 contiguous bytes of x: the activations
// are staged in shared memory in plain order, fp16 after an exact
// power-of-two range scaling that is undone when a partial leaves the warp.
// The bf16 lm_head takes bf16 x.
//
// Work split of a GEMV phase: K is cut into `ns` slabs; a "segment" is one
// 16-row block of one slab.  Every CTA owns whole segments; its warps split
// the CTA's units and the pieces of a segment held by different warps are
// summed in warp order in shared memory.  With one slab the CTA finishes the
// rows (plain store or SiLU * up); with several it stores one partial row per
// slab and the phase that consumes the vector adds the slabs in order
// (computing any RMSNorm over the whole vector itself).  Every sum has a fixed
// order, so results are bit-reproducible.
//
// Attention splits each (sequence, KV head) over CTAs by keys.  When every
// segment has the same number of CTAs, each CTA posts its piece, waits on the
// segment's counter and merges its share of the segment's outputs; otherwise
// the last CTA to arrive merges the whole segment (no waiting).  Pieces are
// folded in a fixed order.
//
// State that outlives a function (ring cursors, descriptors, launch
// constants, unit tables) is kept in shared memory; the hot loops keep theirs
// in registers and touch no local memory.  The helpers on the phase
// boundaries and the copy warp's cursor walk are inlined: a call to a
// non-inlined device function there costs far more than its body.  The
// phase bodies, the launch setup and the rare paths stay out of line.
#pragma once
#include <float.h>
#include <math.h>

#include "ptx.cuh"
#include "w4a_internal.h"

namespace w4a {

constexpr long long WAIT_CYCLES = 4000000000LL;  // bound on any single wait (~2 s)
constexpr int MAX_SEG = MAX_B * 16;              // attention segments (batch x kv heads)
constexpr int NS_MAX = 8;                        // k-slabs a GEMV phase may choose

__host__ __device__ inline long long rstart(long long U, int n, int i) { return (U * i) / n; }
// CTA (of n) whose range [rstart(c), rstart(c+1)) contains unit u.
__host__ __device__ inline int owner(long long U, int n, long long u) {
  return int(((u + 1) * n + U - 1) / U) - 1;
}

// x of klen columns for B rows fits the staging buffers (values and the
// per-group sums).
__host__ __device__ inline bool x_fits(long long klen, int B, int nb) {
  return B * (klen * 2 + 64) <= xs_cap(nb) && (klen / GROUP) * 8 * nb * 4 <= XSUM_BYTES;
}

// Largest k-chunks per slab whose x fits the shared-memory budget (one slab
// when it fits whole, else two slabs must fit); 0 when none does.
__host__ __device__ inline int choose_kps(int nkc, int kcw, int B, int nb) {
  if (x_fits((long long)nkc * kcw, B, nb)) return nkc;
  for (int dv = nkc - 1; dv >= 1; --dv)
    if (nkc % dv == 0 && x_fits(2LL * dv * kcw, B, nb)) return dv;
  return 0;
}

// Chooses how many k-slabs a GEMV phase uses.  The phase lasts as long as its
// busiest CTA, i.e. ceil(segments / CTAs) segments of kps units each; every
// slab beyond the first makes the consuming phase read one more copy of the
// output vector from L2 (`readers` CTAs read all of it).  Both are counted in
// bytes moved per SM: an L2 byte costs 1 / L2_VS_SM_HBM of an HBM byte on one
// SM (an estimate: ~12 TB/s of L2 against 6.5 TB/s of HBM shared by the SMs).
constexpr double L2_VS_SM_HBM = 270.0;
inline Geo gemv_geo(long long n, long long k, int kcw, int B, int nb, int nc, int readers) {
  // a consumer reading the whole vector loads at most four slabs per round trip
  const int ns_cap = readers > 1 ? 4 : NS_MAX;
  Geo g;
  g.nrb = int((n + RB - 1) / RB);
  g.nkc = int(k / kcw);
  g.ns = g.kps = g.nseg = g.nca = g.aligned = 0;
  const int kmax = choose_kps(g.nkc, kcw, B, nb);
  if (kmax <= 0 || nc <= 0) return g;
  const int ns0 = g.nkc / kmax;
  const int ub = kcw == W4_KC ? W4_UNIT : (kcw == S32_KC ? S32_UNIT : BF_UNIT);
  const double slab_cost = double(readers) * B * double(n) * 4.0 / L2_VS_SM_HBM;
  double best = 0.0;
  for (int ns = ns0; ns <= g.nkc && (ns == ns0 || ns <= ns_cap); ++ns) {
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
  // slab-aligned CTA groups when that keeps the busiest CTA's segment count
  if (g.ns > 1 && g.nca >= g.ns) {
    const long long per = (g.nseg + g.nca - 1) / g.nca;
    long long per_al = 0;
    for (int s = 0; s < g.ns; ++s) {
      const long long cnt = rstart(g.nca, g.ns, s + 1) - rstart(g.nca, g.ns, s);
      per_al = per_al > (g.nrb + cnt - 1) / cnt ? per_al : (g.nrb + cnt - 1) / cnt;
    }
    if (per_al <= per) g.aligned = 1;
  }
  return g;
}

// ---------------------------------------------------------------------------
// Phase descriptor (256 bytes; one per phase in the workspace plan)
// ---------------------------------------------------------------------------
struct alignas(16) PD {
  int kind, layer, n, k;         // PK_*, layer, GEMV rows / columns
  int kcw, ub, xsrc, epi;        // k per unit, unit bytes, XS_*, EPI_*
  Geo g;                         // GEMV geometry (24 bytes)
  int rows_valid, ostride;       // rows that exist; row stride of `out`
  const uint8_t* blob;           // GEMV units
  const uint16_t* xbf;           // 16-bit input rows (XS_BF16 / XS_F16; standalone attention: q)
  const float* xres;             // residual (XS_RESID / XS_FINAL)
  const float* vpart;            // producer slabs [vns][B][vstride] (XS_RESID / XS_FINAL / XS_SILU / reduce)
  const float* gain;             // RMSNorm gain of the branch
  const float* gain2;            // final RMSNorm gain (XS_FINAL)
  float* xdst;                   // new residual copy
  float* dump;                   // per-layer hidden dump
  void* out;                     // EPI_PART: fp32 slab base [ns][B][ostride]; EPI_SILU: 16-bit [B][ostride]
  float* aux;                    // reduce: per-16-row sums of squares
  int xbf_stride, vns, vstride, out_f16;
  int type, newkv, slots, seqoff;  // attention: layer type, append new k/v, cache slots, first sequence
  const uint8_t* kc;             // attention K region; a GEMV summing its own slabs: its row-block counters
  const uint8_t* vc;             // attention V region
  uint16_t* aout;                // attention output [B][nq][hd]
  union {
    const float* qpart;          // attention: QKV slabs [qns][B][qkv_dim]
    const float* vsq;            // XS_RESID / XS_FINAL GEMV above 8 rows: the branch's sums of squares
                                 // per (row, 16-row block) [B][nrb], published by a producer that sums
                                 // its own slabs (null otherwise)
  };
  const float* lpart;            // lm_head slabs [lns][B][vocab]; a GEMV summing its own slabs: the sums [B][ostride]
  const float* qnorm;            // QK-norm gains
  const float* knorm;
  int qns, lns, red_epi;
  int gi;                        // GEMV: index of its geometry in the launch's table
};
static_assert(sizeof(PD) == 256, "phase descriptor size");

__host__ __device__ __forceinline__ bool is_gemv_kind(int k) { return unsigned(k) <= unsigned(PK_GEMV_S32); }

// Launch constants (shared memory).
struct LC {
  int B, d, nq, nkv, ffn, vocab, window, nc;
  int mode, begin, end, n_layers, seq0, pos_const, trace_phases, max_ctx;
  float eps, mscale0, mscale1;
  int cur_phase;
  int scaled;  // some x row of this phase is range-scaled
  int final_norm;
  int stop;  // the math warps have left the phase loop
  uint32_t seg_target;  // arrivals each equal-split attention segment counter has reached
  long long wait_bar;   // bound (cycles) on a wait for other CTAs: grid barrier, attention segment
  int pd_hi;            // last phase whose descriptor copy was issued (thread 0)
  uint32_t* ctl;
  uint32_t* seg_ctr;
  float* apart;
  float* amax_val;
  int32_t* amax_idx;
  PD* plan;
  uint64_t* trace;
  const int32_t* tokens;
  const uint16_t* embed;
  float* logits;
  int32_t* next_token;
  const int32_t* pos;
};
static_assert(sizeof(LC) <= 256, "launch constants");

// A warp's position in its unit stream.
//   GEMV:      p0 = units, x0 = unit bytes, x1 = k-chunks per row block, x2 =
//              k-chunks per slab, x3 = row blocks, x4 / x5 / x6 = slab / row
//              block / k-chunk of unit i
//   attention: p0 / p1 = K / V regions, x0 = slots, x1 = first sequence, x2 =
//              layer type, x3 = segment of unit i
// kind: PK_* of phase p; CUR_DONE past the launch; CUR_WAIT when phase p's
// descriptor is not in shared memory yet.
constexpr int CUR_DONE = -1, CUR_WAIT = -2;
struct alignas(16) Cursor {
  int p, kind, i, end;
  const uint8_t* p0;
  const uint8_t* p1;
  int x0, x1, x2, x3, x4, x5, x6, pad_;
};
struct alignas(16) Ring {
  uint32_t consumed, pad0, pad1;  // units the math warp has taken
  int bad;    // a wait of the math warp timed out: stop waiting
  Cursor ld;  // the copy warp's cursor for this ring (its slow path)
};
static_assert(sizeof(Cursor) == 64 && sizeof(Ring) == 80, "ring state layout");

// ---------------------------------------------------------------------------
// Shared memory map
// ---------------------------------------------------------------------------
constexpr int SM_RING = 0;
constexpr int SM_MBAR = SM_RING + NW * NSLOT * SLOT_BYTES;
constexpr int PD_SLOTS = 4;                        // descriptor slots (phase p in slot p % 4)
constexpr int PD_LEAD = 2;                         // descriptor p is copied at the start of phase p - 2
constexpr int SM_EBAR = SM_MBAR + NW * NSLOT * 8;  // slot free again [NW][NSLOT]
constexpr int SM_PDBAR = SM_EBAR + NW * NSLOT * 8;
constexpr int SM_XS = ((SM_PDBAR + PD_SLOTS * 8 + 127) / 128) * 128;
constexpr int X_REGION = xs_cap(1) + XSUM_BYTES + wsp_bytes(1);
static_assert(xs_cap(1) + wsp_bytes(1) == xs_cap(2) + wsp_bytes(2), "x region");
__host__ __device__ constexpr int sm_xsum(int nb) { return SM_XS + xs_cap(nb); }
__host__ __device__ constexpr int sm_wsp(int nb) { return sm_xsum(nb) + XSUM_BYTES; }
constexpr int SM_QS = SM_XS + X_REGION;            // q of a head group, fp32 [MAX_GQ][128]
constexpr int SM_KNV = SM_QS + MAX_GQ * 128 * 4;    // new k / v, bf16 [2][128]
constexpr int SM_RED = SM_KNV + 512;                // 64 floats of block reductions
constexpr int SM_POSB = SM_RED + 256;               // positions [MAX_B]
constexpr int SM_LB = SM_POSB + MAX_B * 4;          // attended keys [2][MAX_B]
constexpr int SM_SNEW = SM_LB + 2 * MAX_B * 4;      // slot of the new key [2][MAX_B]
constexpr int SM_SST = SM_SNEW + 2 * MAX_B * 4;     // segment starts [2][MAX_SEG + 1]
constexpr int SM_FLAGS = SM_SST + ((2 * (MAX_SEG + 1) * 4 + 15) / 16) * 16;
constexpr int SM_LC = SM_FLAGS + 64;
constexpr int SM_ROPE = SM_LC + 256;                // inverse frequencies, fp64 [2][64]
constexpr int SM_PD = SM_ROPE + 2 * 64 * 8;         // descriptor slots
constexpr int SM_WST = SM_PD + PD_SLOTS * (int)sizeof(PD);  // ring state per warp
constexpr int SM_CTAB = SM_WST + NW * (int)sizeof(Ring);  // GEMV unit ranges [5 geometries][NW][4] int4
constexpr int SM_TOTAL = SM_CTAB + 5 * NW * 64;
static_assert(SM_TOTAL <= 232448, "shared memory budget");
// attention views of the x region
constexpr int ATT_PW = MAX_GQ * (128 + 2);                // floats of one warp's partial
constexpr int SM_APW = SM_XS;                             // warp partials [NW][ATT_PW]
constexpr int SM_QF = SM_XS + NW * ATT_PW * 4;            // q fragments (4 KB)
constexpr int SM_ASCR = SM_QF + 4096;                     // k, v rows fp32 [2][128], sums [2][NW]
static_assert(NW * 64 * 3 * 4 <= NW * ATT_PW * 4, "piece-merge scratch inside the warp partials");
static_assert(SM_ASCR + 2 * 128 * 4 + 2 * NW * 4 <= SM_XS + X_REGION, "attention scratch");


extern __shared__ __align__(128) uint8_t w4a_smem[];

template <class T>
__device__ __forceinline__ T* sm_at(int off) {
  return reinterpret_cast<T*>(w4a_smem + off);
}
__device__ __forceinline__ LC& lc() { return *sm_at<LC>(SM_LC); }
__device__ __forceinline__ PD& pd_slot(int p) {
  return *sm_at<PD>(SM_PD + (p & (PD_SLOTS - 1)) * (int)sizeof(PD));
}
__device__ __forceinline__ uint64_t* pd_bar(int p) { return sm_at<uint64_t>(SM_PDBAR) + (p & (PD_SLOTS - 1)); }
__device__ __forceinline__ Ring* ring_state(int w) { return sm_at<Ring>(SM_WST) + w; }
// Unit range of math warp w under GEMV geometry gi, computed once per launch:
// [0] = (first unit, end, slab, row block of the first unit), [1] = (its
// k-chunk, the CTA's first unit, the CTA's end, 0), [2] = the segment this
// warp closes for the CTA: (1 + first warp holding a piece of it, or 0 when
// the warp closes none; bit i: piece of warp first + i sits in that warp's
// second park slot, bit 16 + i: warp first + i has no units; its slab; its
// row block), [3] = (first column of the CTA's x range, its length, 0, 0).
__device__ __forceinline__ const int4* ctab(int gi, int w) { return sm_at<int4>(SM_CTAB) + (gi * NW + w) * 4; }
__device__ __forceinline__ uint64_t* ring_bar(int w, int s) { return sm_at<uint64_t>(SM_MBAR) + w * NSLOT + s; }
__device__ __forceinline__ uint64_t* ring_ebar(int w, int s) { return sm_at<uint64_t>(SM_EBAR) + w * NSLOT + s; }
__device__ __forceinline__ uint8_t* ring_slot(int w, int s) {
  return sm_at<uint8_t>(SM_RING + (w * NSLOT + s) * SLOT_BYTES);
}
__device__ __forceinline__ float* red() { return sm_at<float>(SM_RED); }
__device__ __forceinline__ int* posb() { return sm_at<int>(SM_POSB); }
__device__ __forceinline__ int* Lb(int type) { return sm_at<int>(SM_LB) + type * MAX_B; }
__device__ __forceinline__ int* snew(int type) { return sm_at<int>(SM_SNEW) + type * MAX_B; }
__device__ __forceinline__ int* sst(int type) { return sm_at<int>(SM_SST) + type * (MAX_SEG + 1); }
__device__ __forceinline__ int* flags() { return sm_at<int>(SM_FLAGS); }
__device__ __forceinline__ const double* rope_f(int type) { return sm_at<double>(SM_ROPE) + type * 64; }

// Warp barrier that is also a compiler memory barrier: shared-memory state
// written by one lane (under `if (lane == 0)`) must be re-read by the others
// after it, never forwarded from a load the compiler hoisted above it.
__device__ __forceinline__ void warp_sync() {
  asm volatile("" ::: "memory");
  __syncwarp();
  asm volatile("" ::: "memory");
}

// barrier over the CTA's warps (named barrier 1)
__device__ __forceinline__ void cbar() { asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory"); }
__device__ __forceinline__ void set_error(uint32_t bits) { atomicOr(lc().ctl + 2, bits); }

// A phase output carried between phases as 16 bits: bf16, or fp16 (the
// SwiGLU output h and the attention output o of the decode step).  fp16 holds
// |v| < 65504; a value beyond it (or a NaN) sets EW_RANGE instead of passing
// an infinity on silently.
__device__ __forceinline__ uint16_t out16(float v, bool f16) {
  if (!f16) return f32_to_bf16(v);
  const uint16_t h = f32_to_f16(v);
  if ((h & 0x7c00u) == 0x7c00u) set_error(EW_RANGE);
  return h;
}

__device__ __forceinline__ void mark(int slot) {
  const LC& L = lc();
  if (L.trace != nullptr && threadIdx.x == 0 && L.cur_phase < L.trace_phases)
    L.trace[((size_t)L.cur_phase * L.nc + blockIdx.x) * 8 + slot] = globaltimer();
}

// cos / sin of the rotation angle pos * f, times the attention factor: the
// angle is formed and reduced to [-pi, pi] in fp64, then evaluated in fp32.
__device__ __forceinline__ float2 rope_cs2(int pos, double f, float ms) {
  const double a = double(pos) * f;
  const double r = a - 6.283185307179586 * rint(a * 0.15915494309189535);
  float sn, cs;
  sincosf(float(r), &sn, &cs);
  return make_float2(cs * ms, sn * ms);
}
__device__ __forceinline__ void rope_cs(int pos, double f, float ms, float& c, float& s) {
  const float2 r = rope_cs2(pos, f, ms);
  c = r.x;
  s = r.y;
}

__device__ __forceinline__ uint32_t u4_word(const uint4& v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// ---------------------------------------------------------------------------
// Phase descriptors, built on the device from the launch parameters
// ---------------------------------------------------------------------------
__device__ __noinline__ void build_pd(const EngineParams& P, int p, PD* out) {
  uint4* z = reinterpret_cast<uint4*>(out);
#pragma unroll 1
  for (int i = 0; i < (int)(sizeof(PD) / 16); ++i) z[i] = make_uint4(0u, 0u, 0u, 0u);
  PD& d = *out;
  const int B = P.B;
  if (P.mode == MODE_GEMV) {
    d.kind = (p == 0) ? (P.fmt == FMT_SYM32 ? PK_GEMV_S32 : PK_GEMV_W4) : PK_REDUCE;
    d.blob = P.g_blob;
    d.n = P.g_n;
    d.k = P.g_k;
    d.kcw = fmt_kc(P.fmt);
    d.ub = fmt_unit(P.fmt);
    d.xsrc = XS_BF16;
    d.xbf = P.g_x;
    d.xbf_stride = P.g_k;
    d.rows_valid = P.g_n;
    d.g = P.geo[0];
    d.gi = 0;
    const bool direct_silu = P.g_epi == W4A_EPI_SILU_MUL && d.g.ns == 1;
    const bool direct = P.g_epi == W4A_EPI_NONE && d.g.ns == 1;
    if (direct_silu) {
      d.epi = EPI_SILU;
      d.out = P.g_out;
      d.ostride = P.g_n / 2;
    } else {
      d.epi = EPI_PART;
      d.out = direct ? P.g_out : P.ws.g_part;
      d.ostride = P.g_n;
    }
    if (p == 1) {  // sum the slabs, then the requested epilogue
      d.vpart = P.ws.g_part;
      d.vns = d.g.ns;
      d.out = P.g_out;
      d.aux = P.g_aux;
      d.red_epi = P.g_epi;
    }
    return;
  }
  if (P.mode == MODE_ATTN) {
    d.kind = PK_ATTN;
    d.slots = P.a_slots;
    d.kc = reinterpret_cast<const uint8_t*>(P.a_k);
    d.vc = reinterpret_cast<const uint8_t*>(P.a_v);
    d.aout = P.a_out;
    d.xbf = P.a_q;
    return;
  }
  const int nl = P.n_layers, dm = P.d;
  const int qd = P.nq * P.hd, qkv_dim = (P.nq + 2 * P.nkv) * P.hd;
  const Geo& g_qkv = P.geo[0];
  const Geo& g_o = P.geo[1];
  const Geo& g_gu = P.geo[2];
  const Geo& g_dn = P.geo[3];
  const Geo& g_lm = P.geo[4];
  // the O and down phases sum their own slabs when K is cut into many
  const bool red_o = g_o.ns > RED_NS, red_dn = g_dn.ns > RED_NS;
  const float* f_src = red_dn ? P.ws.f_red : P.ws.f_part;
  const int f_ns = red_dn ? 1 : g_dn.ns;
  if (p == 5 * nl) {
    d.kind = PK_GEMV_BF16;
    d.blob = P.lm_head;
    d.n = (P.vocab + RB - 1) / RB * RB;
    d.k = dm;
    d.kcw = BF_KC;
    d.ub = BF_UNIT;
    d.g = g_lm;
    d.gi = 4;
    d.xsrc = XS_FINAL;
    d.xres = P.ws.xB;
    d.vpart = f_src;
    d.vns = f_ns;
    d.vsq = red_dn ? P.ws.f_red + (size_t)B * dm : nullptr;
    d.vstride = dm;
    d.gain = P.layers[nl - 1].ffn_norm;
    d.gain2 = P.final_norm ? P.final_gain : nullptr;
    d.dump = P.dump ? P.dump + (size_t)nl * B * dm : nullptr;
    d.rows_valid = P.vocab;
    d.epi = EPI_PART;
    d.out = (g_lm.ns == 1) ? P.logits : P.ws.lg_part;
    d.ostride = P.vocab;
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
    d.vc = d.kc + (size_t)P.kv_batch * P.nkv * d.slots * P.hd * 2;
    d.aout = P.ws.o;
    d.out_f16 = 1;
    d.qpart = P.ws.y_part;
    d.qns = g_qkv.ns;
    d.qnorm = lw.q_norm;
    d.knorm = lw.k_norm;
    return;
  }
  d.kind = P.fmt == FMT_SYM32 ? PK_GEMV_S32 : PK_GEMV_W4;
  d.kcw = fmt_kc(P.fmt);
  d.ub = fmt_unit(P.fmt);
  d.rows_valid = 1 << 30;
  d.epi = EPI_PART;
  if (sub == 0) {
    d.blob = lw.qkv;
    d.n = qkv_dim;
    d.k = dm;
    d.g = g_qkv;
    d.gi = 0;
    if (l == 0) {
      d.xsrc = XS_EMBED;
    } else {
      d.xsrc = XS_RESID;
      d.xres = P.ws.xB;
      d.vpart = f_src;
      d.vns = f_ns;
      d.vsq = red_dn ? P.ws.f_red + (size_t)B * dm : nullptr;
      d.vstride = dm;
      d.gain = P.layers[l - 1].ffn_norm;
    }
    d.xdst = P.ws.xA;
    d.dump = P.dump ? P.dump + (size_t)l * B * dm : nullptr;
    d.out = P.ws.y_part;
    d.ostride = qkv_dim;
  } else if (sub == 2) {
    d.blob = lw.o;
    d.n = dm;
    d.k = qd;
    d.g = g_o;
    d.gi = 1;
    d.xsrc = XS_F16;
    d.xbf = P.ws.o;
    d.xbf_stride = qd;
    d.out = P.ws.a_part;
    d.ostride = dm;
    if (red_o) {
      d.kc = reinterpret_cast<const uint8_t*>(P.ws.rb_ctr);
      d.lpart = P.ws.a_red;
      d.aux = P.ws.a_red + (size_t)B * dm;  // its blocks' sums of squares (above 8 rows)
    }
  } else if (sub == 3) {
    d.blob = lw.gu;
    d.n = 2 * P.ffn;
    d.k = dm;
    d.g = g_gu;
    d.gi = 2;
    d.xsrc = XS_RESID;
    d.xres = P.ws.xA;
    d.vpart = red_o ? P.ws.a_red : P.ws.a_part;
    d.vns = red_o ? 1 : g_o.ns;
    d.vsq = red_o ? P.ws.a_red + (size_t)B * dm : nullptr;
    d.vstride = dm;
    d.gain = lw.attn_norm;
    d.xdst = P.ws.xB;
    if (d.g.ns == 1) {
      d.epi = EPI_SILU;
      d.out = P.ws.h;
      d.ostride = P.ffn;
      d.out_f16 = 1;
    } else {
      d.out = P.ws.gu_part;
      d.ostride = 2 * P.ffn;
    }
  } else {
    d.blob = lw.down;
    d.n = dm;
    d.k = P.ffn;
    d.g = g_dn;
    d.gi = 3;
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
    d.out = P.ws.f_part;
    d.ostride = dm;
    if (red_dn) {
      d.kc = reinterpret_cast<const uint8_t*>(P.ws.rb_ctr + MAX_RBC);
      d.lpart = P.ws.f_red;
      d.aux = P.ws.f_red + (size_t)B * dm;  // its blocks' sums of squares (above 8 rows)
    }
  }
}

// ---------------------------------------------------------------------------
// Ranges
// ---------------------------------------------------------------------------
// A GEMV CTA owns whole segments: units [a, b) of the phase order.
__host__ __device__ inline void gemv_cta_range(const Geo& g, int cta, int& a, int& b) {
  if (cta >= g.nca) {
    a = b = 0;
  } else if (g.aligned) {
    // CTA group s of slab s: its CTAs share the slab's row blocks
    int s = 0;
    while (s + 1 < g.ns && rstart(g.nca, g.ns, s + 1) <= cta) ++s;
    const int c0 = int(rstart(g.nca, g.ns, s)), cnt = int(rstart(g.nca, g.ns, s + 1)) - c0;
    a = (s * g.nrb + int(rstart(g.nrb, cnt, cta - c0))) * g.kps;
    b = (s * g.nrb + int(rstart(g.nrb, cnt, cta - c0 + 1))) * g.kps;
  } else {
    a = int(rstart(g.nseg, g.nca, cta)) * g.kps;
    b = int(rstart(g.nseg, g.nca, cta + 1)) * g.kps;
  }
}
// A CTA's GEMV units split over its math warps.  Warp w runs on SM
// sub-partition w % 4; the copy warp (warp NW = 15) shares sub-partition 3
// with only three math warps, which run a unit ~1.09x faster than the math
// warps of the full sub-partitions (per-warp finish times of the 64-layer
// decode step).  Shares: 11 parts per warp, 12 on sub-partition 3, of 168;
// warp w starts at 11 w + floor(w / 4).
static_assert(NW == 15, "warp shares assume 15 math warps");
__device__ __forceinline__ int warp_part(int w) { return 11 * w + (w >> 2); }
__device__ __forceinline__ void warp_range(int a, int b, int w, int& wa, int& wb) {
  wa = a + (b - a) * warp_part(w) / 168;
  wb = a + (b - a) * warp_part(w + 1) / 168;
}
// Attention work split over CTAs.  When every segment (sequence, KV head)
// has the same number of 128-key units n (the usual case: equal lengths),
// each segment gets m = nc / segments CTAs of its own (at most n of them) and
// no CTA spans two segments; otherwise the units are split contiguously.
// amode / am / ameff per layer type live in flags()[4 + 3 type ..].
__device__ __forceinline__ void attn_cta_range(int type, int cta, int& a, int& b, int& nca) {
  const LC& L = lc();
  const int* st = sst(type);
  const int S = L.B * L.nkv;
  const int total = st[S];
  const int* am = flags() + 4 + 3 * type;
  if (am[0]) {
    const int m = am[1], meff = am[2], n = st[1] - st[0];
    const int s = cta / m, j = cta - s * m;
    nca = S * m;
    if (s < S && j < meff) {
      a = st[s] + n * j / meff;
      b = st[s] + n * (j + 1) / meff;
    } else {
      a = b = 0;
    }
    return;
  }
  nca = total < L.nc ? total : L.nc;
  if (nca > 0 && cta < nca) {
    a = int(rstart(total, nca, cta));
    b = int(rstart(total, nca, cta + 1));
  } else {
    a = b = 0;
  }
}
// CTAs c0 .. c1 holding the pieces of segment seg.
__device__ __forceinline__ void attn_seg_ctas(int type, int seg, int nca, int& c0, int& c1) {
  const int* st = sst(type);
  const int* am = flags() + 4 + 3 * type;
  if (am[0]) {
    c0 = seg * am[1];
    c1 = c0 + am[2] - 1;
    return;
  }
  const int total = st[lc().B * lc().nkv];
  c0 = owner(total, nca, st[seg]);
  c1 = owner(total, nca, st[seg + 1] - 1);
}

// ---------------------------------------------------------------------------
// Unit streams: cursors, the ring, the L2 prefetch
// ---------------------------------------------------------------------------
// Is phase q's descriptor in shared memory?  Descriptors begin .. begin +
// PD_LEAD are built in shared memory at launch; descriptor q after them is
// copied at the start of phase q - PD_LEAD (the k-th copy into its slot
// completes mbarrier phase k).  `block`: wait for a copy under way (bounded);
// else only test it.
__device__ __forceinline__ bool pd_ready(int q, bool block) {
  const LC& L = lc();
  if (q <= L.begin + PD_LEAD) return true;
  if (*reinterpret_cast<const volatile int*>(&L.cur_phase) < q - PD_LEAD) return false;  // copy not issued yet
  const uint32_t par = uint32_t((q - L.begin - PD_LEAD - 1) / PD_SLOTS) & 1u;
  if (mbar_try_wait(pd_bar(q), par)) return true;
  if (!block) return false;
  const long long t0 = clock64();
  while (!mbar_try_wait(pd_bar(q), par)) {
    if (clock64() - t0 > WAIT_CYCLES) {
      set_error(EW_MBAR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Position cursor c at the first unit of warp w in phase q.
__device__ __forceinline__ void cur_enter(Cursor* c, int q, int w) {
  const LC& L = lc();
  c->p = q;
  c->i = c->end = 0;
  if (q >= L.end) {
    c->kind = CUR_DONE;
    return;
  }
  if (!pd_ready(q, false)) {
    c->kind = CUR_WAIT;
    return;
  }
  const PD& d = pd_slot(q);
  c->kind = d.kind;
  if (is_gemv_kind(d.kind)) {
    const int4* e = ctab(d.gi, w);
    const int4 e0 = e[0], e1 = e[1];
    c->p0 = d.blob;
    c->x0 = d.ub;
    c->x1 = d.g.nkc;
    c->x2 = d.g.kps;
    c->x3 = d.g.nrb;
    c->i = e0.x;
    c->end = e0.y;
    c->x4 = e0.z;
    c->x5 = e0.w;
    c->x6 = e1.x;
  } else if (d.kind == PK_ATTN) {
    int a, b, nca;
    attn_cta_range(d.type, blockIdx.x, a, b, nca);
    c->i = a;
    c->end = b;
    c->p0 = d.kc;
    c->p1 = d.vc;
    c->x0 = d.slots;
    c->x1 = d.seqoff;
    c->x2 = d.type;
    c->x3 = 0;
  }
}

// Move c to warp w's next unit at or after its position (possibly in a later
// phase).  Stops on CUR_DONE or CUR_WAIT.
__device__ __forceinline__ void cur_normalize(Cursor* c, int w) {
  const LC& L = lc();
#pragma unroll 1
  for (;;) {
    const int kind = c->kind;
    if (kind == CUR_DONE) return;
    if (kind == CUR_WAIT) {
      if (!pd_ready(c->p, false)) return;
      cur_enter(c, c->p, w);
      continue;
    }
    if (is_gemv_kind(kind)) {
      if (c->i < c->end) return;
    } else if (kind == PK_ATTN) {
      const int* st = sst(c->x2);
#pragma unroll 1
      while (c->i < c->end) {
        while (st[c->x3 + 1] <= c->i) ++c->x3;
        const int key0 = (c->i - st[c->x3]) * ATT_CTA_KEYS + w * ATT_KEYS;
        if (key0 < Lb(c->x2)[c->x3 / L.nkv]) return;
        ++c->i;
      }
    }
    cur_enter(c, c->p + 1, w);
  }
}

__device__ __forceinline__ void cur_load(Cursor& c, const Cursor* s) {
  const uint4* q = reinterpret_cast<const uint4*>(s);
  const uint4 v0 = q[0], v1 = q[1], v2 = q[2], v3 = q[3];
  c.p = int(v0.x);
  c.kind = int(v0.y);
  c.i = int(v0.z);
  c.end = int(v0.w);
  c.p0 = reinterpret_cast<const uint8_t*>((uint64_t(v1.y) << 32) | v1.x);
  c.p1 = reinterpret_cast<const uint8_t*>((uint64_t(v1.w) << 32) | v1.z);
  c.x0 = int(v2.x);
  c.x1 = int(v2.y);
  c.x2 = int(v2.z);
  c.x3 = int(v2.w);
  c.x4 = int(v3.x);
  c.x5 = int(v3.y);
  c.x6 = int(v3.z);
  c.pad_ = 0;
}
__device__ __forceinline__ void cur_store(Cursor* s, const Cursor& c) {
  uint4* q = reinterpret_cast<uint4*>(s);
  const uint64_t a = reinterpret_cast<uint64_t>(c.p0), b = reinterpret_cast<uint64_t>(c.p1);
  q[0] = make_uint4(uint32_t(c.p), uint32_t(c.kind), uint32_t(c.i), uint32_t(c.end));
  q[1] = make_uint4(uint32_t(a), uint32_t(a >> 32), uint32_t(b), uint32_t(b >> 32));
  q[2] = make_uint4(uint32_t(c.x0), uint32_t(c.x1), uint32_t(c.x2), uint32_t(c.x3));
  q[3] = make_uint4(uint32_t(c.x4), uint32_t(c.x5), uint32_t(c.x6), 0u);
}

// Next unit of a copy-warp lane's cursor: the common GEMV step in registers,
// everything else through the lane's shared-memory copy.
__device__ __forceinline__ void cur_adv(Cursor& c, int w) {
  if (is_gemv_kind(c.kind)) {
    ++c.i;
    if (++c.x6 == c.x2) {
      c.x6 = 0;
      if (++c.x5 == c.x3) {
        c.x5 = 0;
        ++c.x4;
      }
    }
    if (c.i < c.end) return;
  } else {
    ++c.i;
  }
  Cursor* s = &ring_state(w)->ld;
  cur_store(s, c);
  cur_normalize(s, w);
  cur_load(c, s);
}

// Source range(s) of the unit under a cursor.
__device__ __forceinline__ void cur_src(const Cursor& c, int warp, const uint8_t*& s1, const uint8_t*& s2,
                                        uint32_t& bytes, int hd) {
  if (is_gemv_kind(c.kind)) {
    const uint32_t idx = uint32_t(c.x5 * c.x1 + c.x4 * c.x2 + c.x6);
    s1 = c.p0 + (size_t)idx * uint32_t(c.x0);
    s2 = nullptr;
    bytes = uint32_t(c.x0);
  } else {
    const LC& L = lc();
    const int* st = sst(c.x2);
    const int bq = c.x3 / L.nkv, g = c.x3 - bq * L.nkv;
    const int key0 = (c.i - st[c.x3]) * ATT_CTA_KEYS + warp * ATT_KEYS;
    const size_t row = ((size_t)(c.x1 + bq) * L.nkv + g) * c.x0 + key0;
    bytes = ATT_KEYS * hd * 2;
    s1 = c.p0 + row * hd * 2;
    s2 = c.p1 + row * hd * 2;
  }
}

// ---- consumer side of a warp's ring ----------------------------------------
// Math warp w takes its units in order from slots w.0, w.1: it waits for the
// slot's copy (full barrier) and hands the slot back (empty barrier) once its
// lanes are done with it.  The copy warp refills it.
struct Cons {
  uint32_t consumed;
  int bad;  // a wait of this warp timed out: stop waiting
};
__device__ __forceinline__ void cons_load(Cons& C, int warp) {
  const Ring* s = ring_state(warp);
  C.consumed = s->consumed;
  C.bad = s->bad;
}
__device__ __forceinline__ void cons_store(const Cons& C, int warp, int lane) {
  warp_sync();  // all lanes are done reading the shared copy
  if (lane == 0) {
    Ring* s = ring_state(warp);
    s->consumed = C.consumed;
    s->bad = C.bad;
  }
  warp_sync();
}
__device__ __forceinline__ uint8_t* cons_wait(Cons& C, int warp, int lane) {
  const int sl = C.consumed % NSLOT;
  const uint32_t par = (C.consumed / NSLOT) & 1u;
  uint64_t* bar = ring_bar(warp, sl);
  int late = 0;
  if (!C.bad && !mbar_try_wait(bar, par)) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, par)) {
      if (clock64() - t0 > WAIT_CYCLES) {
        late = 1;
        break;
      }
    }
  }
  if (__any_sync(0xffffffffu, late)) {  // keep the warp's state uniform
    if (lane == 0) set_error(EW_MBAR_TIMEOUT);
    C.bad = 1;
  }
  return ring_slot(warp, sl);
}
// Hand the slot back.  Lanes that wrote into it order those writes before
// the copy engine's refill.
__device__ __forceinline__ void cons_release(Cons& C, int warp, int lane, bool wrote_slot) {
  if (wrote_slot) fence_proxy_async();
  warp_sync();  // every lane is done with the slot
  if (lane == 0) mbar_arrive(ring_ebar(warp, C.consumed % NSLOT));
  ++C.consumed;
}

// ---- the copy warp -----------------------------------------------------------
// Lane w (< NW) walks math warp w's unit stream through the phases of the
// launch and issues each unit's bulk copy as soon as its slot is free; the
// math warps never compute addresses or issue copies.  It stops past the last
// phase, or when the math warps have left (error paths), and then waits for
// its copies in flight so that none lands after the CTA has exited.
template <int HD>
__device__ __noinline__ void copy_warp() {
  const int lane = threadIdx.x & 31;
  if (lane >= NW) return;
  const int w = lane;
  Cursor c;
  cur_load(c, &ring_state(w)->ld);
  uint32_t issued = 0;
  // weights and old keys are read once per token: evict them first, so that
  // the activations, residuals and gains the phase prologues read stay in L2
  const uint64_t once = policy_evict_first();
  long long idle0 = clock64();
#pragma unroll 1
  for (;;) {
    if (c.kind == CUR_DONE) break;
    bool progress = false;
    if (c.kind == CUR_WAIT) {
      if (pd_ready(c.p, false)) {
        Cursor* s = &ring_state(w)->ld;
        cur_store(s, c);
        cur_normalize(s, w);
        cur_load(c, s);
        progress = true;
      }
    } else {
      const int sl = issued % NSLOT;
      const uint32_t n = issued / NSLOT;
      if (n == 0 || mbar_test_wait(ring_ebar(w, sl), (n - 1u) & 1u)) {
        const uint8_t *s1, *s2;
        uint32_t bytes;
        cur_src(c, w, s1, s2, bytes, HD);
        // the math warp's accesses of the slot (seen through the empty
        // barrier) before the copy engine overwrites it
        fence_proxy_async();
        uint64_t* bar = ring_bar(w, sl);
        uint8_t* dst = ring_slot(w, sl);
        mbar_expect_tx(bar, s2 ? 2 * bytes : bytes);
        bulk_g2s_hint(dst, s1, bytes, bar, once);
        if (s2) bulk_g2s_hint(dst + bytes, s2, bytes, bar, once);
        ++issued;
        cur_adv(c, w);
        progress = true;
      }
    }
    if (progress) {
      idle0 = clock64();
      continue;
    }
    if (*reinterpret_cast<volatile int*>(&lc().stop) != 0) break;
    if (clock64() - idle0 > 2 * WAIT_CYCLES) {
      set_error(EW_MBAR_TIMEOUT);
      break;
    }
  }
  // copies in flight land before the lane leaves
#pragma unroll 1
  for (uint32_t j = issued > uint32_t(NSLOT) ? issued - NSLOT : 0u; j < issued; ++j) {
    const long long t0 = clock64();
    while (!mbar_try_wait(ring_bar(w, j % NSLOT), (j / NSLOT) & 1u)) {
      if (clock64() - t0 > WAIT_CYCLES) {
        set_error(EW_DRAIN_TIMEOUT);
        return;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Grid barrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool grid_wait(uint32_t target) {
  if (threadIdx.x == 0) {
    const LC& L = lc();
    int ok = 1;
    const long long t0 = clock64();
    while (ld_acquire(L.ctl) < target) {
      if (ld_volatile_u32(L.ctl + 2) != 0u) {
        ok = 0;
        break;
      }
      if (clock64() - t0 > L.wait_bar) {
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
// The CTA barrier orders every thread's writes of the phase before thread
// 0's release, and the release makes them visible to the acquiring CTAs.
__device__ __forceinline__ void grid_arrive() {
  cbar();
  if (threadIdx.x == 0) red_release_add(lc().ctl, 1u);
}

// Deterministic per-batch-row totals of per-warp partial sums wsum[warp][b].
// Warp 0 sums the NW partials of each row with a fixed shuffle tree.
__device__ __forceinline__ void block_rows_total(const float* wsum, float* out, int B) {
  cbar();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
#pragma unroll 1
    for (int b = 0; b < B; ++b) {
      float s = lane < NW ? wsum[lane * MAX_B + b] : 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) out[b] = s;
    }
  }
  cbar();
}

// ---------------------------------------------------------------------------
// GEMV input staging
// ---------------------------------------------------------------------------
__device__ __forceinline__ float4 ldcg4(const float* p) { return __ldcg(reinterpret_cast<const float4*>(p)); }

struct F8 {
  float v[8];
};
__device__ __forceinline__ F8 f8(const float (&a)[8]) {
  F8 r;
#pragma unroll
  for (int i = 0; i < 8; ++i) r.v[i] = a[i];
  return r;
}

// Sum of `ns` slabs (stride sstride floats) at p[0 .. 8), in slab order, the
// loads of up to eight slabs in flight at once.
__device__ __noinline__ F8 slab_sum8v(const float* p, size_t sstride, int ns) {
  F8 r;
  float* v = r.v;
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = 0.f;
#pragma unroll 1
  for (int s0 = 0; s0 < ns; s0 += 8) {
    float4 a[8], b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      a[i] = b[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (s0 + i < ns) {
        a[i] = ldcg4(p + (s0 + i) * sstride);
        b[i] = ldcg4(p + (s0 + i) * sstride + 4);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (s0 + i < ns) {
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
  return r;
}
// The same for two chunks at once (p1 used when has1), four slabs of each in
// flight per round.
struct F16v {
  float v[16];
};
__device__ __forceinline__ F16v slab_sum8x2(const float* p0, const float* p1, bool has1, size_t sstride, int ns) {
  F16v r;
  float* v = r.v;
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = 0.f;
#pragma unroll 1
  for (int s0 = 0; s0 < ns; s0 += 4) {
    float4 a[2][4], b[2][4];
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[c][i] = b[c][i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (s0 + i < ns && (c == 0 || has1)) {
          const float* p = (c ? p1 : p0) + (s0 + i) * sstride;
          a[c][i] = ldcg4(p);
          b[c][i] = ldcg4(p + 4);
        }
      }
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (s0 + i < ns) {
          v[8 * c + 0] += a[c][i].x;
          v[8 * c + 1] += a[c][i].y;
          v[8 * c + 2] += a[c][i].z;
          v[8 * c + 3] += a[c][i].w;
          v[8 * c + 4] += b[c][i].x;
          v[8 * c + 5] += b[c][i].y;
          v[8 * c + 6] += b[c][i].z;
          v[8 * c + 7] += b[c][i].w;
        }
      }
  }
  return r;
}
__device__ __forceinline__ void slab_sum8(const float* p, size_t sstride, int ns, float (&v)[8]) {
  const F8 r = slab_sum8v(p, sstride, ns);
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = r.v[i];
}

__device__ __forceinline__ void cvt16(bool f16, const uint4& u, float (&v)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint16_t lo = uint16_t(w[i] & 0xffffu), hi = uint16_t(w[i] >> 16);
    v[2 * i] = f16 ? half_bits_to_f32(lo) : bf16_to_f32(lo);
    v[2 * i + 1] = f16 ? half_bits_to_f32(hi) : bf16_to_f32(hi);
  }
}

// Store eight activations x[bb][kl0 .. kl0 + 8) (kl0 relative to the staged
// range) as fp16 (f16) or bf16, times `scale`.  The 16 lanes of a half-warp
// hold one 128-group, whose sum (of the stored, rounded values) and max |x|
// they reduce here.  Warp-uniform: every lane calls it.
template <int NB>
__device__ __forceinline__ void put8(bool valid, int bb, int kl0, int xrow_b, F8 vv, bool f16, float scale,
                                  bool track_max) {
  const float* v = vv.v;
  const int lane = threadIdx.x & 31;
  float s8 = 0.f, m8 = 0.f;
  if (valid) {
    uint32_t w[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float a = v[2 * t] * scale, b = v[2 * t + 1] * scale;
      if (f16) {
        const uint16_t ha = f32_to_f16(a), hb = f32_to_f16(b);
        w[t] = uint32_t(ha) | (uint32_t(hb) << 16);
        s8 += half_bits_to_f32(ha) + half_bits_to_f32(hb);
      } else {
        const uint16_t ha = f32_to_bf16(a), hb = f32_to_bf16(b);
        w[t] = uint32_t(ha) | (uint32_t(hb) << 16);
        s8 += bf16_to_f32(ha) + bf16_to_f32(hb);
      }
      m8 = fmaxf(m8, fmaxf(fabsf(v[2 * t]), fabsf(v[2 * t + 1])));
    }
    *sm_at<uint4>(SM_XS + bb * xrow_b + kl0 * 2) = make_uint4(w[0], w[1], w[2], w[3]);
  }
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) s8 += __shfl_xor_sync(0xffffffffu, s8, o);
  if (valid && (lane & 15) == 0) sm_at<float>(sm_xsum(NB))[(kl0 >> 7) * (8 * NB) + bb] = s8;
  // the row maximum matters only once it reaches the fp16 guard, so only the
  // lanes past it post theirs (rare; shared atomics on one word serialise)
  if (track_max && __any_sync(0xffffffffu, valid && m8 >= 32768.f) && valid && m8 >= 32768.f)
    atomicMax(reinterpret_cast<uint32_t*>(red() + 32) + bb, __float_as_uint(m8));
}

// Two fp16 chunks of eight at once (the residual paths hold up to two chunks
// per thread): the conversions and the two group-sum reductions interleave.
template <int NB>
__device__ __forceinline__ void put8x2(bool va, int ba, int ka, const float (&xa)[8], bool vb, int bb, int kb,
                                       const float (&xb)[8], int xrow_b) {
  const int lane = threadIdx.x & 31;
  float sa = 0.f, sb = 0.f, ma = 0.f, mb = 0.f;
  uint32_t wa[4], wb[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint16_t a0 = f32_to_f16(xa[2 * t]), a1 = f32_to_f16(xa[2 * t + 1]);
    const uint16_t b0 = f32_to_f16(xb[2 * t]), b1 = f32_to_f16(xb[2 * t + 1]);
    wa[t] = uint32_t(a0) | (uint32_t(a1) << 16);
    wb[t] = uint32_t(b0) | (uint32_t(b1) << 16);
    sa += half_bits_to_f32(a0) + half_bits_to_f32(a1);
    sb += half_bits_to_f32(b0) + half_bits_to_f32(b1);
    ma = fmaxf(ma, fmaxf(fabsf(xa[2 * t]), fabsf(xa[2 * t + 1])));
    mb = fmaxf(mb, fmaxf(fabsf(xb[2 * t]), fabsf(xb[2 * t + 1])));
  }
  if (!va) sa = 0.f;
  if (!vb) sb = 0.f;
  if (va) *sm_at<uint4>(SM_XS + ba * xrow_b + ka * 2) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
  if (vb) *sm_at<uint4>(SM_XS + bb * xrow_b + kb * 2) = make_uint4(wb[0], wb[1], wb[2], wb[3]);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) {
    sa += __shfl_xor_sync(0xffffffffu, sa, o);
    sb += __shfl_xor_sync(0xffffffffu, sb, o);
  }
  if ((lane & 15) == 0) {
    if (va) sm_at<float>(sm_xsum(NB))[(ka >> 7) * (8 * NB) + ba] = sa;
    if (vb) sm_at<float>(sm_xsum(NB))[(kb >> 7) * (8 * NB) + bb] = sb;
  }
  const bool pa = va && ma >= 32768.f, pb = vb && mb >= 32768.f;
  if (__any_sync(0xffffffffu, pa || pb)) {  // rare: the fp16 guard
    if (pa) atomicMax(reinterpret_cast<uint32_t*>(red() + 32) + ba, __float_as_uint(ma));
    if (pb) atomicMax(reinterpret_cast<uint32_t*>(red() + 32) + bb, __float_as_uint(mb));
  }
}

__device__ __forceinline__ void store8f(float* p, const float (&x)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
}
__device__ __forceinline__ void load8f(const float* p, float (&v)[8], bool ro) {
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

// Eight inputs of a 16-bit source or the SiLU(gate) * up source at k0.
__device__ __noinline__ F8 src16_or_silu_v(const PD& d, int bb, int k0) {
  F8 r;
  float* v = r.v;
  const LC& L = lc();
  if (d.xsrc == XS_SILU) {
    float ga[8], gb[8];
    // tiled rows 2j (gate j), 2j + 1 (up j): columns [2 k0, 2 k0 + 16)
    slab_sum8(d.vpart + (size_t)bb * d.vstride + 2 * k0, (size_t)L.B * d.vstride, d.vns, ga);
    slab_sum8(d.vpart + (size_t)bb * d.vstride + 2 * k0 + 8, (size_t)L.B * d.vstride, d.vns, gb);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[i] = ga[2 * i] / (1.f + expf(-ga[2 * i])) * ga[2 * i + 1];
      v[4 + i] = gb[2 * i] / (1.f + expf(-gb[2 * i])) * gb[2 * i + 1];
    }
    return r;
  }
  int tok = 0;
  if (d.xsrc == XS_EMBED) {
    tok = L.tokens[bb];
    tok = tok < 0 ? 0 : (tok >= L.vocab ? L.vocab - 1 : tok);
  }
  const uint4 u = (d.xsrc == XS_EMBED)
                      ? __ldg(reinterpret_cast<const uint4*>(L.embed + (size_t)tok * L.d + k0))
                      : __ldcg(reinterpret_cast<const uint4*>(d.xbf + (size_t)bb * d.xbf_stride + k0));
  float w[8];
  cvt16(d.xsrc == XS_F16, u, w);
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = w[i];
  return r;
}
__device__ __forceinline__ void src16_or_silu(const PD& d, int bb, int k0, float (&v)[8]) {
  const F8 r = src16_or_silu_v(d, bb, k0);
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = r.v[i];
}

// Residual update of one chunk: x = xres + v * r * gain.
__device__ __forceinline__ void resid8(const float (&v)[8], const float (&xr)[8], const float (&g)[8], float r,
                                       float (&x)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = fmaf(v[i] * r, g[i], xr[i]);
}

// Scratch a GEMV phase's staging starts from: group sums, row maxima, row
// scales, per-warp sums of squares.  Runs between phases (after the CTA's
// arrival at the grid barrier, before the wait's CTA sync), so the staging
// itself starts with loads.
template <int NB>
__device__ __forceinline__ void stage_reset() {
  const int tid = threadIdx.x;
  float* rd = red();
  float* xsm = sm_at<float>(sm_xsum(NB));
#pragma unroll 1
  for (int i = tid; i < XSUM_BYTES / 4; i += NT) xsm[i] = 0.f;
  if (tid < MAX_B) {
    reinterpret_cast<uint32_t*>(rd + 32)[tid] = 0u;
    rd[48 + tid] = 1.f;
  }
  float* wsum = sm_at<float>(sm_wsp(NB));
  if (tid < NW * MAX_B) wsum[tid] = 0.f;
  if (tid == 0) lc().scaled = 0;
}

// Stage x for the CTA's k-range [kbase, kbase + klen) of a GEMV phase.  The
// scratch was reset by stage_reset.
template <int NB>
__device__ __forceinline__ void stage_x(const PD& d, int kbase, int klen) {
  LC& L = lc();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = L.B, dm = L.d;
  const bool f16 = (d.kind == PK_GEMV_W4 || d.kind == PK_GEMV_S32);
  float* rd = red();
  float* wsum = sm_at<float>(sm_wsp(NB));  // [NW][MAX_B] per-warp sums of squares (reset by stage_reset)
  const int xrow_b = klen * 2 + 64;
  const bool has_out = (d.xdst != nullptr || d.dump != nullptr);
  const int nout = B * dm / 8;
  const int out_per = (nout + L.nc - 1) / L.nc;
  const int o0 = blockIdx.x * out_per, o1 = min(nout, o0 + out_per);

  if (d.xsrc == XS_RESID || d.xsrc == XS_FINAL) {
    // Residual update over the whole width: v = sum of the branch slabs,
    // x = xres + v * rsqrt(mean(v^2) + eps) * gain  [then the final norm].
    // Chunks of 8; a warp iteration covers 32 consecutive chunks of one batch
    // row (d % 256 == 0).  Up to two chunks per thread stay in registers.
    const int n8 = dm / 8, total8 = B * n8;
    const bool fin = (d.xsrc == XS_FINAL) && d.gain2 != nullptr;
    const bool two = NB == 1 && total8 <= 2 * NT;  // never above 8 rows (B * d / 8 > 2 NT)
    const size_t sstride = (size_t)B * d.vstride;
    const int c0 = warp * 32 + lane, c1 = c0 + NT;
    const bool h0 = warp * 32 < total8, h1 = two && warp * 32 + NT < total8;
    const int b0 = h0 ? (warp * 32) / n8 : 0, b1 = h1 ? (warp * 32 + NT) / n8 : 0;
    const int k00 = (c0 - b0 * n8) * 8, k01 = (c1 - b1 * n8) * 8;
    float v0[8], v1[8], x0[8], x1[8], g0[8], g1[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v0[i] = v1[i] = x0[i] = x1[i] = g0[i] = g1[i] = 0.f;
    // pass 1: branch sums (and, for up to two chunks, residual and gains in flight together)
    if (NB > 1 && d.vsq != nullptr) {
      // the producer published its blocks' sums of squares: warp w adds those
      // of rows w, w + NW, ... (eight loads in flight per lane, then a fixed
      // shuffle tree), so no CTA reads the whole branch output here
      const int nrb = (dm + RB - 1) / RB;
#pragma unroll 1
      for (int bb = warp; bb < B; bb += NW) {
        const float* q = d.vsq + (size_t)bb * nrb;
        float sq = 0.f;
#pragma unroll 1
        for (int r0 = 0; r0 < nrb; r0 += 8 * 32) {
          float t[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int rb = r0 + i * 32 + lane;
            t[i] = rb < nrb ? __ldcg(q + rb) : 0.f;
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) sq += t[i];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (lane == 0) wsum[warp * MAX_B + bb] = sq;
      }
    } else if (two) {
      // the residual and gain only where this CTA uses x: its k-range and
      // its share of the residual copy (all of it for the final norm); the
      // sums of squares need every branch value
      const bool u0 = fin || (k00 >= kbase && k00 < kbase + klen) || (c0 >= o0 && c0 < o1);
      const bool u1 = fin || (k01 >= kbase && k01 < kbase + klen) || (c1 >= o0 && c1 < o1);
      if (h0 && u0) {
        load8f(d.xres + (size_t)b0 * dm + k00, x0, false);
        load8f(d.gain + k00, g0, true);
      }
      if (h1 && u1) {
        load8f(d.xres + (size_t)b1 * dm + k01, x1, false);
        load8f(d.gain + k01, g1, true);
      }
      if (h0) {
        const F16v r = slab_sum8x2(d.vpart + (size_t)b0 * d.vstride + k00, d.vpart + (size_t)b1 * d.vstride + k01,
                                   h1, sstride, d.vns);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          v0[i] = r.v[i];
          v1[i] = r.v[8 + i];
        }
      }
      float sq0 = 0.f, sq1 = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        sq0 = fmaf(v0[i], v0[i], sq0);
        sq1 = fmaf(v1[i], v1[i], sq1);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        sq0 += __shfl_xor_sync(0xffffffffu, sq0, o);
        sq1 += __shfl_xor_sync(0xffffffffu, sq1, o);
      }
      if (lane == 0 && h0) wsum[warp * MAX_B + b0] += sq0;
      if (lane == 0 && h1) wsum[warp * MAX_B + b1] += sq1;
    } else {
#pragma unroll 1
      for (int j = 0; warp * 32 + j * NT < total8; ++j) {
        const int c = warp * 32 + j * NT + lane, bb = (warp * 32 + j * NT) / n8;
        float v[8];
        slab_sum8(d.vpart + (size_t)bb * d.vstride + (c - bb * n8) * 8, sstride, d.vns, v);
        float sq = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) sq = fmaf(v[i], v[i], sq);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (lane == 0) wsum[warp * MAX_B + bb] += sq;
      }
    }
    block_rows_total(wsum, rd, B);
    if (tid < B) rd[tid] = rsqrtf(rd[tid] / float(dm) + L.eps);
    cbar();
    mark(2);
    if (fin) {
      // the final norm's sums of squares
      if (tid < NW * MAX_B) wsum[tid] = 0.f;
      cbar();
#pragma unroll 1
      for (int j = 0; warp * 32 + j * NT < total8; ++j) {
        const int c = warp * 32 + j * NT + lane, bb = (warp * 32 + j * NT) / n8, k0 = (c - bb * n8) * 8;
        float x[8];
        if (two) {
          if (j == 0)
            resid8(v0, x0, g0, rd[bb], x);
          else
            resid8(v1, x1, g1, rd[bb], x);
        } else {
          float v[8], xr[8], g[8];
          slab_sum8(d.vpart + (size_t)bb * d.vstride + k0, sstride, d.vns, v);
          load8f(d.xres + (size_t)bb * dm + k0, xr, false);
          load8f(d.gain + k0, g, true);
          resid8(v, xr, g, rd[bb], x);
        }
        float sq = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) sq = fmaf(x[i], x[i], sq);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (lane == 0) wsum[warp * MAX_B + bb] += sq;
      }
      block_rows_total(wsum, rd + 16, B);
      if (tid < B) rd[16 + tid] = rsqrtf(rd[16 + tid] / float(dm) + L.eps);
      cbar();
    }
    // convert the k-range, write the residual copy / dump slice
    if (two && !fin) {
      // this thread's (up to) two chunks, indexed in pass 1
      float xa[8], xb[8];
      resid8(v0, x0, g0, h0 ? rd[b0] : 0.f, xa);
      resid8(v1, x1, g1, h1 ? rd[b1] : 0.f, xb);
      if (has_out) {
        if (h0 && c0 >= o0 && c0 < o1) {
          if (d.xdst) store8f(d.xdst + (size_t)b0 * dm + k00, xa);
          if (d.dump) store8f(d.dump + (size_t)b0 * dm + k00, xa);
        }
        if (h1 && c1 >= o0 && c1 < o1) {
          if (d.xdst) store8f(d.xdst + (size_t)b1 * dm + k01, xb);
          if (d.dump) store8f(d.dump + (size_t)b1 * dm + k01, xb);
        }
      }
      // half-warps are uniformly inside or outside (128-aligned k-range)
      put8x2<NB>(h0 && k00 >= kbase && k00 < kbase + klen, b0, k00 - kbase, xa,
                 h1 && k01 >= kbase && k01 < kbase + klen, b1, k01 - kbase, xb, xrow_b);
    } else
#pragma unroll 1
    for (int j = 0; warp * 32 + j * NT < total8; ++j) {
      const int c = warp * 32 + j * NT + lane, bb = (warp * 32 + j * NT) / n8, k0 = (c - bb * n8) * 8;
      if (!two) {
        // the warp's 32 chunks (256 columns of one row): skip them unless they
        // meet the CTA's k-range or its share of the residual copy (warp-uniform)
        const int cw = warp * 32 + j * NT, kw = (cw - bb * n8) * 8;
        const bool in_k = kw + 256 > kbase && kw < kbase + klen;
        const bool in_out = has_out && cw + 32 > o0 && cw < o1;
        if (!in_k && !in_out) continue;
      }
      float x[8];
      if (two) {
        if (j == 0)
          resid8(v0, x0, g0, rd[bb], x);
        else
          resid8(v1, x1, g1, rd[bb], x);
      } else {
        float v[8], xr[8], g[8];
        slab_sum8(d.vpart + (size_t)bb * d.vstride + k0, sstride, d.vns, v);
        load8f(d.xres + (size_t)bb * dm + k0, xr, false);
        load8f(d.gain + k0, g, true);
        resid8(v, xr, g, rd[bb], x);
      }
      if (has_out && c >= o0 && c < o1) {
        if (d.xdst) store8f(d.xdst + (size_t)bb * dm + k0, x);
        if (d.dump) store8f(d.dump + (size_t)bb * dm + k0, x);
      }
      if (fin) {
        float g2[8];
        load8f(d.gain2 + k0, g2, true);
        const float rf = rd[16 + bb];
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = x[i] * rf * g2[i];
      }
      // half-warps are uniformly inside or outside (128-aligned k-range)
      put8<NB>(k0 >= kbase && k0 < kbase + klen, bb, k0 - kbase, xrow_b, f8(x), f16, 1.f, f16);
    }
  } else {
    // 16-bit / SiLU sources: the k-range only
    const int n8 = klen / 8, total8 = B * n8;
    if (d.xsrc != XS_SILU) {
      constexpr int JU = 4;  // chunks per thread in flight
#pragma unroll 1
      for (int j0 = 0; warp * 32 + j0 * NT < total8; j0 += JU) {
        uint4 raw[JU];
#pragma unroll
        for (int jj = 0; jj < JU; ++jj) {
          const int c = warp * 32 + (j0 + jj) * NT + lane;
          raw[jj] = make_uint4(0u, 0u, 0u, 0u);
          if (c < total8) {
            const int bb = c / n8;
            const int k0 = kbase + (c - bb * n8) * 8;
            if (d.xsrc == XS_EMBED) {
              const int tok = max(0, min(L.vocab - 1, L.tokens[bb]));
              raw[jj] = __ldg(reinterpret_cast<const uint4*>(L.embed + (size_t)tok * dm + k0));
            } else {
              raw[jj] = __ldcg(reinterpret_cast<const uint4*>(d.xbf + (size_t)bb * d.xbf_stride + k0));
            }
          }
        }
#pragma unroll
        for (int jj = 0; jj < JU; ++jj) {
          const int cw = warp * 32 + (j0 + jj) * NT;
          if (cw < total8) {  // warp-uniform (total8 % 32 == 0)
            const int c = cw + lane, bb = cw / n8;
            float v[8];
            cvt16(d.xsrc == XS_F16, raw[jj], v);
            put8<NB>(true, bb, (c - bb * n8) * 8, xrow_b, f8(v), f16, 1.f, f16);
          }
        }
      }
    } else {
#pragma unroll 1
      for (int j = 0; warp * 32 + j * NT < total8; ++j) {
        const int cw = warp * 32 + j * NT, c = cw + lane, bb = cw / n8;
        float v[8];
        src16_or_silu(d, bb, kbase + (c - bb * n8) * 8, v);
        put8<NB>(true, bb, (c - bb * n8) * 8, xrow_b, f8(v), f16, 1.f, f16);
      }
    }
    mark(2);
    // residual copy / dump of the embedding (first layer)
    if (has_out) {
#pragma unroll 1
      for (int c = o0 + tid; c < o1; c += NT) {
        const int bb = (c * 8) / dm, k0 = c * 8 - bb * dm;
        float v[8];
        src16_or_silu(d, bb, k0, v);
        if (d.xdst) store8f(d.xdst + (size_t)bb * dm + k0, v);
        if (d.dump) store8f(d.dump + (size_t)bb * dm + k0, v);
      }
    }
    if (blockIdx.x == 0 && tid == 0 && d.xsrc == XS_EMBED) {
#pragma unroll 1
      for (int bb = 0; bb < B; ++bb)
        if (L.tokens[bb] < 0 || L.tokens[bb] >= L.vocab) set_error(EW_BAD_SHAPE);
    }
  }
  cbar();
}

// fp16 range guard: rows whose max |x| reaches 2^15 are re-staged scaled by an
// exact power of two, undone on the partial sums when they leave the warp.
template <int NB>
__device__ __noinline__ void restage_scaled(const PD& d, int kbase, int klen) {
  const LC& L = lc();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = L.B, dm = L.d;
  float* rd = red();
  const uint32_t* xmax = reinterpret_cast<const uint32_t*>(rd + 32);
  const int n8 = klen / 8, total8 = B * n8;
  const int xrow_b = klen * 2 + 64;
#pragma unroll 1
  for (int j = 0; warp * 32 + j * NT < total8; ++j) {
    const int cw = warp * 32 + j * NT, c = cw + lane, bb = cw / n8;  // one batch row per warp iteration
    const float mx = __uint_as_float(xmax[bb]);
    if (!(mx >= 32768.f)) continue;  // warp-uniform
    int ex;
    frexpf(mx, &ex);
    const int k0 = kbase + (c - bb * n8) * 8;
    float v[8];
    if (d.xsrc == XS_RESID || d.xsrc == XS_FINAL) {
      float br[8], xr[8], g[8];
      slab_sum8(d.vpart + (size_t)bb * d.vstride + k0, (size_t)B * d.vstride, d.vns, br);
      load8f(d.xres + (size_t)bb * dm + k0, xr, false);
      load8f(d.gain + k0, g, true);
      resid8(br, xr, g, rd[bb], v);
      if (d.xsrc == XS_FINAL && d.gain2 != nullptr) {
        load8f(d.gain2 + k0, g, true);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] *= rd[16 + bb] * g[i];
      }
    } else {
      src16_or_silu(d, bb, k0, v);
    }
    put8<NB>(true, bb, k0 - kbase, xrow_b, f8(v), true, ldexpf(1.f, 15 - ex), false);
  }
  cbar();
  if (tid < B) {
    const float mx = __uint_as_float(xmax[tid]);
    if (mx >= 32768.f) {
      int ex;
      frexpf(mx, &ex);
      rd[48 + tid] = ldexpf(1.f, ex - 15);
    }
  }
  if (tid == 0) lc().scaled = 1;
  cbar();
}

// ---------------------------------------------------------------------------
// Unit kernels (one warp, one unit)
// ---------------------------------------------------------------------------
// int4 unit: codes [grp 4][half 2][lane 32][4 words], scales at +4096 ordered
// [row % 8][grp][row / 8], zeros at +4224 [grp][row / 8] (nibble row % 8).
// A warp copies its share of a unit into registers (w4_load) and hands the
// ring slot back before the math (w4_math), so the slot refills while the
// tensor cores work.
struct W4Regs {
  uint4 q[8];   // codes of this lane: [grp][half]
  uint4 sc;     // scales of rows g, g + 8 for the four groups
  uint4 zA, zB; // zero words [grp][row / 8]
};
__device__ __forceinline__ void w4_load(const uint8_t* slot, int g, int lane, W4Regs& r) {
  const uint4* qw = reinterpret_cast<const uint4*>(slot) + lane;
#pragma unroll
  for (int i = 0; i < 8; ++i) r.q[i] = qw[i * 32];
  r.sc = *reinterpret_cast<const uint4*>(slot + 4096 + g * 16);
  r.zA = *reinterpret_cast<const uint4*>(slot + 4224);
  r.zB = *reinterpret_cast<const uint4*>(slot + 4240);
}
// xl: this lane's x bytes (batch row g, + 16 t, + 2 koff); xsg: per-group sums
// of x for the unit's first group, + 2 t.
template <int NB>
__device__ __forceinline__ void w4_math(const W4Regs& r, const uint8_t* xl, int xrow_b, const float* xsg,
                                        float (&acc)[NB][4], int B, int g) {
  const int sh = 4 * g;
#pragma unroll
  for (int grp = 0; grp < 4; ++grp) {
    const uint4 w0 = r.q[grp * 2];
    const uint4 w1 = r.q[grp * 2 + 1];
    uint4 xv[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int pr = 0; pr < 4; ++pr)
        xv[nb][pr] = (g + 8 * nb < B)
                         ? *reinterpret_cast<const uint4*>(xl + nb * 8 * xrow_b + grp * 256 + pr * 64)
                         : make_uint4(0u, 0u, 0u, 0u);
    float c[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) c[nb][0] = c[nb][1] = c[nb][2] = c[nb][3] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t w = u4_word(i < 4 ? w0 : w1, i & 3);
      const uint32_t a0 = lop3_and_or(w, 0x000F000Fu, 0x64006400u);       // rows g:     1024 + q
      const uint32_t a1 = lop3_and_or(w, 0x00F000F0u, 0x64006400u);       // rows g + 8: 1024 + 16 q
      const uint32_t w8 = w >> 8;
      const uint32_t a2 = lop3_and_or(w8, 0x000F000Fu, 0x64006400u);
      const uint32_t a3 = lop3_and_or(w8, 0x00F000F0u, 0x64006400u);
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const uint4& x = xv[nb][i >> 1];
        mma_16816_f16(c[nb], a0, a1, a2, a3, (i & 1) ? x.z : x.x, (i & 1) ? x.w : x.y);
      }
    }
    const uint32_t sw = u4_word(r.sc, grp);
    const float sl = half_bits_to_f32(uint16_t(sw & 0xffffu));
    const float shi = half_bits_to_f32(uint16_t(sw >> 16)) * 0.0625f;
    const uint32_t zl_w = u4_word(grp < 2 ? r.zA : r.zB, (grp * 2) & 3);
    const uint32_t zh_w = u4_word(grp < 2 ? r.zA : r.zB, (grp * 2 + 1) & 3);
    // 1024 + z and 1024 + 16 z built in the fp32 significand (2^23 + m - (2^23 - 1024))
    const float zl = __uint_as_float(0x4B000000u | ((zl_w >> sh) & 15u)) - 8387584.f;
    const float zh = __uint_as_float(0x4B000000u | (((zh_w >> sh) & 15u) << 4)) - 8387584.f;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const float2 xs2 = *reinterpret_cast<const float2*>(xsg + grp * (8 * NB) + nb * 8);
      acc[nb][0] = fmaf(sl, fmaf(-zl, xs2.x, c[nb][0]), acc[nb][0]);
      acc[nb][1] = fmaf(sl, fmaf(-zl, xs2.y, c[nb][1]), acc[nb][1]);
      acc[nb][2] = fmaf(shi, fmaf(-zh, xs2.x, c[nb][2]), acc[nb][2]);
      acc[nb][3] = fmaf(shi, fmaf(-zh, xs2.y, c[nb][3]), acc[nb][3]);
    }
  }
}
template <int NB>
__device__ __forceinline__ void w4_unit(const uint8_t* slot, const uint8_t* xl, int xrow_b, const float* xsg,
                                        float (&acc)[NB][4], int B, int g, int lane) {
  W4Regs r;
  w4_load(slot, g, lane, r);
  w4_math<NB>(r, xl, xrow_b, xsg, acc, B, g);
}

// Symmetric group-32 unit (16 rows x 256 columns): codes [grp 2][half 2]
// [lane 32][4 words] as in the int4 unit, then bf16 scales at +2048 ordered
// [row % 8][32-column group 8][row / 8] (a lane's 16 scales are 32 contiguous
// bytes).  The zero point is 8 for every group, so the LOP3 forms 1024 + q
// (rows g) / 1024 + 16 q (rows g + 8) are moved to q - 8 / 16 (q - 8) by one
// exact fp16 subtraction, and every 32-column group (two k-steps) closes as
// s * acc (s / 16 for the 16x rows); no per-group sums of x are needed.
struct S32Regs {
  uint4 q[4];   // codes of this lane: [grp][half]
  uint4 s0, s1; // scales of rows g, g + 8: groups 0..3, 4..7
};
__device__ __forceinline__ void s32_load(const uint8_t* slot, int g, int lane, S32Regs& r) {
  const uint4* qw = reinterpret_cast<const uint4*>(slot) + lane;
#pragma unroll
  for (int i = 0; i < 4; ++i) r.q[i] = qw[i * 32];
  r.s0 = *reinterpret_cast<const uint4*>(slot + 2048 + g * 32);
  r.s1 = *reinterpret_cast<const uint4*>(slot + 2048 + g * 32 + 16);
}
__device__ __forceinline__ uint32_t hsub2_bits(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
template <int NB>
__device__ __forceinline__ void s32_math(const S32Regs& r, const uint8_t* xl, int xrow_b, float (&acc)[NB][4], int B,
                                         int g) {
  constexpr uint32_t Z_LO = 0x64086408u;  // fp16 pair 1032 = 1024 + 8
  constexpr uint32_t Z_HI = 0x64806480u;  // fp16 pair 1152 = 1024 + 16 * 8
#pragma unroll
  for (int grp = 0; grp < 2; ++grp) {
    const uint4 w0 = r.q[grp * 2];
    const uint4 w1 = r.q[grp * 2 + 1];
    uint4 xv[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int pr = 0; pr < 4; ++pr)
        xv[nb][pr] = (g + 8 * nb < B)
                         ? *reinterpret_cast<const uint4*>(xl + nb * 8 * xrow_b + grp * 256 + pr * 64)
                         : make_uint4(0u, 0u, 0u, 0u);
    const uint4 sv = grp ? r.s1 : r.s0;
#pragma unroll
    for (int sub = 0; sub < 4; ++sub) {
      float c[NB][4];
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) c[nb][0] = c[nb][1] = c[nb][2] = c[nb][3] = 0.f;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = 2 * sub + e;
        const uint32_t w = u4_word(i < 4 ? w0 : w1, i & 3);
        const uint32_t a0 = hsub2_bits(lop3_and_or(w, 0x000F000Fu, 0x64006400u), Z_LO);
        const uint32_t a1 = hsub2_bits(lop3_and_or(w, 0x00F000F0u, 0x64006400u), Z_HI);
        const uint32_t w8 = w >> 8;
        const uint32_t a2 = hsub2_bits(lop3_and_or(w8, 0x000F000Fu, 0x64006400u), Z_LO);
        const uint32_t a3 = hsub2_bits(lop3_and_or(w8, 0x00F000F0u, 0x64006400u), Z_HI);
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          const uint4& x = xv[nb][i >> 1];
          mma_16816_f16(c[nb], a0, a1, a2, a3, (i & 1) ? x.z : x.x, (i & 1) ? x.w : x.y);
        }
      }
      // scales of group grp * 4 + sub: rows g (low half) and g + 8 (high half)
      const uint32_t sw = u4_word(sv, sub);
      const float sl = bf16_to_f32(uint16_t(sw & 0xffffu));
      const float shi = bf16_to_f32(uint16_t(sw >> 16)) * 0.0625f;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        acc[nb][0] = fmaf(sl, c[nb][0], acc[nb][0]);
        acc[nb][1] = fmaf(sl, c[nb][1], acc[nb][1]);
        acc[nb][2] = fmaf(shi, c[nb][2], acc[nb][2]);
        acc[nb][3] = fmaf(shi, c[nb][3], acc[nb][3]);
      }
    }
  }
}
template <int NB>
__device__ __forceinline__ void s32_unit(const uint8_t* slot, const uint8_t* xl, int xrow_b, float (&acc)[NB][4],
                                         int B, int g, int lane) {
  S32Regs r;
  s32_load(slot, g, lane, r);
  s32_math<NB>(r, xl, xrow_b, acc, B, g);
}

// bf16 unit: A fragments [k-step 8][lane 32][4 words].
struct BfRegs {
  uint4 a[8];
};
__device__ __forceinline__ void bf_load(const uint8_t* slot, int lane, BfRegs& r) {
  const uint4* aw = reinterpret_cast<const uint4*>(slot) + lane;
#pragma unroll
  for (int i = 0; i < 8; ++i) r.a[i] = aw[i * 32];
}
template <int NB>
__device__ __forceinline__ void bf_math(const BfRegs& r, const uint8_t* xl, int xrow_b, float (&acc)[NB][4], int B,
                                        int g) {
  uint4 xv[NB][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb)
#pragma unroll
    for (int pr = 0; pr < 4; ++pr)
      xv[nb][pr] = (g + 8 * nb < B) ? *reinterpret_cast<const uint4*>(xl + nb * 8 * xrow_b + pr * 64)
                                    : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4& a = r.a[i];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const uint4& x = xv[nb][i >> 1];
      mma_16816(acc[nb], a.x, a.y, a.z, a.w, (i & 1) ? x.z : x.x, (i & 1) ? x.w : x.y);
    }
  }
}
template <int NB>
__device__ __forceinline__ void bf_unit(const uint8_t* slot, const uint8_t* xl, int xrow_b, float (&acc)[NB][4],
                                        int B, int g, int lane) {
  BfRegs r;
  bf_load(slot, lane, r);
  bf_math<NB>(r, xl, xrow_b, acc, B, g);
}

// ---------------------------------------------------------------------------
// GEMV outputs
// ---------------------------------------------------------------------------
// Rows of 16-row block rb of slab s; fragment v[nb][0..3] = (row g, batch
// nb*8 + 2t), (g, 2t+1), (g+8, 2t), (g+8, 2t+1).
template <int NB>
struct Acc {
  float v[NB][4];
};
template <int NB>
__device__ __forceinline__ Acc<NB> acc_of(const float (&a)[NB][4]) {
  Acc<NB> r;
#pragma unroll
  for (int nb = 0; nb < NB; ++nb)
#pragma unroll
    for (int j = 0; j < 4; ++j) r.v[nb][j] = a[nb][j];
  return r;
}

template <int NB>
__device__ __forceinline__ void emit_rows(const PD& d, int s, int rb, Acc<NB> A, int B, int lane) {
  const float (&v)[NB][4] = A.v;
  const int g = lane >> 2, t = lane & 3;
  if (d.epi == EPI_SILU) {
    // rows 2j (gate) and 2j + 1 (up) sit in lanes g and g + 1 of a thread column
    uint16_t* h = reinterpret_cast<uint16_t*>(d.out);
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      float u[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) u[j] = __shfl_down_sync(0xffffffffu, v[nb][j], 4);
      if ((g & 1) == 0) {
        const int j0 = rb * 8 + g / 2, j1 = j0 + 4;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int b = nb * 8 + 2 * t + (e & 1), j = (e & 2) ? j1 : j0;
          const float x = v[nb][e];
          const float hv = __fdividef(x, 1.f + __expf(-x)) * u[e];
          if (b < B) h[(size_t)b * d.ostride + j] = out16(hv, d.out_f16);
        }
      }
    }
    return;
  }
  float* base = reinterpret_cast<float*>(d.out) + (size_t)s * B * d.ostride;
  const int r0 = rb * RB + g, r1 = r0 + 8;
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    const int b0 = nb * 8 + 2 * t, b1 = b0 + 1;
    if (r0 < d.rows_valid) {
      if (b0 < B) base[(size_t)b0 * d.ostride + r0] = v[nb][0];
      if (b1 < B) base[(size_t)b1 * d.ostride + r0] = v[nb][1];
    }
    if (r1 < d.rows_valid) {
      if (b0 < B) base[(size_t)b0 * d.ostride + r1] = v[nb][2];
      if (b1 < B) base[(size_t)b1 * d.ostride + r1] = v[nb][3];
    }
  }
}

// Sum of the ns slabs of outputs (b, r) of a GEMV that sums its own slabs,
// in slab order, eight L2 loads in flight.
__device__ __forceinline__ float slab_total(const PD& d, int b, int r, int B) {
  const float* p = reinterpret_cast<const float*>(d.out) + (size_t)b * d.ostride + r;
  const size_t sstride = (size_t)B * d.ostride;
  const int ns = d.g.ns;
  float v = 0.f;
  int sl = 0;
#pragma unroll 1
  for (; sl + 8 <= ns; sl += 8) {
    float t[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) t[i] = __ldcg(p + (sl + i) * sstride);
#pragma unroll
    for (int i = 0; i < 8; ++i) v += t[i];
  }
#pragma unroll 1
  for (; sl < ns; ++sl) v += __ldcg(p + sl * sstride);
  return v;
}

// After a warp has written the partial rows of segment (slab, row block rb)
// of a GEMV that sums its own slabs: count the row block's arrivals (release:
// every lane's stores, a fence each, the warp barrier, one atomic add).
__device__ __forceinline__ void rb_sum(const PD& d, int rb, int B, int lane) {
  if (d.lpart == nullptr || d.epi != EPI_PART) return;
  uint32_t* ctr = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(d.kc)) + rb;
  __threadfence();
  __syncwarp();
  if (lane == 0) atomicAdd(ctr, 1u);
}

// At the phase end, CTA c sums row blocks c, c + nc, ... (all its math
// threads, each block's ns slabs in slab order, so the sums are the same
// whichever CTA runs them): thread 0 waits (bounded) until every slab of the
// block has arrived (acquire), then the block is summed and its counter
// cleared for the next layer.  A fixed share per CTA: the CTAs that emit a
// block's last slab are not the ones left to sum it, so no CTA gathers a long
// tail of blocks.  Above 8 rows the CTA also publishes the block's sum of
// squares per row (the 16 summed values of a row, squared and added by a fixed
// shuffle tree), so that the consumer's RMSNorm reads B * n / 16 floats
// instead of the whole B x n output.  Called by all math threads after a CTA
// barrier.
template <int NB>
__device__ __forceinline__ void rb_sum_pending(const PD& d) {
  const LC& L = lc();
  const int B = L.B, per = RB * B, nrb = d.g.nrb;
  uint32_t* ctr = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(d.kc));
  float* sum = const_cast<float*>(d.lpart);
#pragma unroll 1
  for (int rb = blockIdx.x; rb < nrb; rb += gridDim.x) {
    if (threadIdx.x == 0) {
      int ok = 1;
      const long long t0 = clock64();
      while (ld_acquire(ctr + rb) < uint32_t(d.g.ns)) {
        if (ld_volatile_u32(L.ctl + 2) != 0u) {  // another CTA gave up: its slab may never come
          ok = 0;
          break;
        }
        if (clock64() - t0 > L.wait_bar) {
          set_error(EW_BARRIER_TIMEOUT);
          ok = 0;
          break;
        }
      }
      flags()[2] = ok;
    }
    cbar();
    if (flags()[2]) {
      if constexpr (NB > 1) {
        static_assert(RB * MAX_B <= NT && RB == 16, "one (row, block row) per math thread");
        const int i = threadIdx.x;
        float v = 0.f;
        if (i < per) {
          const int r = rb * RB + (i & (RB - 1)), b = i / RB;
          if (r < d.rows_valid) {
            v = slab_total(d, b, r, B);
            sum[(size_t)b * d.ostride + r] = v;
          }
        }
        if (d.aux != nullptr && i < ((per + 31) & ~31)) {  // whole warps; a half-warp holds one row's block
          float q = v * v;
#pragma unroll
          for (int o = RB / 2; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
          if (i < per && (i & (RB - 1)) == 0) d.aux[(size_t)(i / RB) * nrb + rb] = q;
        }
      } else {
#pragma unroll 1
        for (int i = threadIdx.x; i < per; i += NT) {
          const int r = rb * RB + (i & (RB - 1)), b = i / RB;
          if (r < d.rows_valid) sum[(size_t)b * d.ostride + r] = slab_total(d, b, r, B);
        }
      }
    }
    cbar();
    if (threadIdx.x == 0) ctr[rb] = 0u;
  }
}

// A segment piece leaves the warp: undo the range scaling, then emit it
// (segment wholly inside this warp) or park it in the warp's slot.
// whole: the warp ran all of the segment's units; first: it is the warp's
// first segment (its piece goes to park slot 0, a later one to slot 1).
template <int NB>
__device__ __forceinline__ void seg_done(const PD& d, int s, int rb, bool whole, bool first, float (&acc)[NB][4],
                                         float* park, int B, int lane) {
  if (lc().scaled) {
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
  if (whole) {
    emit_rows<NB>(d, s, rb, acc_of<NB>(acc), B, lane);
    rb_sum(d, rb, B, lane);
  } else {
    float* q = park + (first ? 0 : 32 * 4 * NB);
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
      reinterpret_cast<float4*>(q)[nb] = make_float4(acc[nb][0], acc[nb][1], acc[nb][2], acc[nb][3]);
  }
}

// Segments of this CTA split between warps: the warp holding a segment's last
// unit sums its pieces in warp order and emits the rows.
template <int NB>
__device__ __forceinline__ void cta_combine(const PD& d) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int4 c = ctab(d.gi, warp)[2];
  if (c.x == 0) return;
  const int w0 = c.x - 1;
  const float* wsp = sm_at<float>(sm_wsp(NB));
  float sum[NB][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) sum[nb][0] = sum[nb][1] = sum[nb][2] = sum[nb][3] = 0.f;
#pragma unroll 1
  for (int w2 = w0; w2 <= warp; ++w2) {
    if ((c.y >> (16 + w2 - w0)) & 1) continue;
    const int sl = (c.y >> (w2 - w0)) & 1;
    const float* q = wsp + w2 * (2 * 32 * 4 * NB) + sl * (32 * 4 * NB) + lane * 4 * NB;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const float4 f = reinterpret_cast<const float4*>(q)[nb];
      sum[nb][0] += f.x;
      sum[nb][1] += f.y;
      sum[nb][2] += f.z;
      sum[nb][3] += f.w;
    }
  }
  emit_rows<NB>(d, c.z, c.w, acc_of<NB>(sum), lc().B, lane);
  rb_sum(d, c.w, lc().B, lane);
}

// The unit loop of a GEMV phase over this CTA's segments (S32: the
// symmetric group-32 units; else group-128 int4 or bf16 units).
template <int NB, bool S32>
__device__ __forceinline__ void gemv_units(const PD& d, int4 e0, int4 e1, int kbase, int klen) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int wa = e0.x, wb = e0.y;
  const int B = lc().B;
  Cons C;
  cons_load(C, warp);
  const int kps = d.g.kps, nrb = d.g.nrb, kcw = d.kcw;
  const bool w4 = (d.kind == PK_GEMV_W4);
  const int xrow_b = klen * 2 + 64;
  const uint8_t* xl = sm_at<uint8_t>(SM_XS + g * xrow_b + t * 16);
  const float* xsg = sm_at<float>(sm_xsum(NB)) + 2 * t;
  float* park = sm_at<float>(sm_wsp(NB)) + warp * (2 * 32 * 4 * NB) + lane * 4 * NB;
  int u = wa;
  int sl = e0.z, rb = e0.w, kci = e1.x;
  float acc[NB][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0.f;
  // the segment in progress: its slab and row block, units run, first?
  int cs = sl, crb = rb, cn = 0;
  bool cfirst = true;
#pragma unroll 1
  for (; u < wb; ++u) {
    if (sl != cs || rb != crb) {
      seg_done<NB>(d, cs, crb, cn == kps, cfirst, acc, park, B, lane);
      cs = sl;
      crb = rb;
      cn = 0;
      cfirst = false;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0.f;
    }
    ++cn;
    const int koff = (sl * kps + kci) * kcw - kbase;
    const uint8_t* slot = cons_wait(C, warp, lane);
    if (NB > 1) {
      // two batch tiles: the math reads the slot (registers are short)
      if (S32)
        s32_unit<NB>(slot, xl + koff * 2, xrow_b, acc, B, g, lane);
      else if (w4)
        w4_unit<NB>(slot, xl + koff * 2, xrow_b, xsg + (koff >> 7) * (8 * NB), acc, B, g, lane);
      else
        bf_unit<NB>(slot, xl + koff * 2, xrow_b, acc, B, g, lane);
      cons_release(C, warp, lane, false);
    } else if (S32) {
      S32Regs sr;
      s32_load(slot, g, lane, sr);
      cons_release(C, warp, lane, false);
      s32_math<NB>(sr, xl + koff * 2, xrow_b, acc, B, g);
    } else if (w4) {
      // copy the unit to registers and hand the slot back before the math
      W4Regs ur;
      w4_load(slot, g, lane, ur);
      cons_release(C, warp, lane, false);
      w4_math<NB>(ur, xl + koff * 2, xrow_b, xsg + (koff >> 7) * (8 * NB), acc, B, g);
    } else {
      BfRegs br;
      bf_load(slot, lane, br);
      cons_release(C, warp, lane, false);
      bf_math<NB>(br, xl + koff * 2, xrow_b, acc, B, g);
    }
    if (++kci == kps) {
      kci = 0;
      if (++rb == nrb) {
        rb = 0;
        ++sl;
      }
    }
  }
  seg_done<NB>(d, cs, crb, cn == kps, cfirst, acc, park, B, lane);
  cons_store(C, warp, lane);
}

// S32: the symmetric group-32 format's instantiation, a separate function,
// so that the group-128 / bf16 one carries none of its code.
template <int NB, int HD, bool S32>
__device__ __noinline__ void gemv_phase(const PD& d) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int4 e0 = ctab(d.gi, warp)[0], e1 = ctab(d.gi, warp)[1];
  int a = e1.y, b = e1.z;
  const int4 e3 = ctab(d.gi, warp)[3];
  int kbase = e3.x, klen = e3.y;
  if (!x_fits(klen, lc().B, NB)) {  // the host sizes slabs so this never happens
    if (tid == 0) set_error(EW_BAD_SHAPE);
    a = b = 0;
    klen = 0;
  }
  stage_x<NB>(d, kbase, klen);
  if (d.kind == PK_GEMV_W4 || d.kind == PK_GEMV_S32) {
    const uint32_t* xmax = reinterpret_cast<const uint32_t*>(red() + 32);
    bool any = false;
#pragma unroll 1
    for (int bb = 0; bb < lc().B; ++bb) any |= __uint_as_float(xmax[bb]) >= 32768.f;
    if (any) restage_scaled<NB>(d, kbase, klen);
  }
  mark(3);
  if (a < b) {
    gemv_units<NB, S32>(d, e0, e1, kbase, klen);
  }
  cbar();
  mark(4);
  if (a < b) cta_combine<NB>(d);
  if (d.lpart != nullptr && d.epi == EPI_PART) {
    cbar();
    rb_sum_pending<NB>(d);
  }
  mark(5);
}

// Standalone GEMV whose K was split into slabs (or with the SUMSQ epilogue):
// y = sum of the slab rows in order, then the requested epilogue.
__device__ __noinline__ void reduce_phase(const PD& d) {
  const LC& L = lc();
  const int B = L.B, n = d.n, ns = d.vns;
  const float* part = d.vpart;
  if (d.red_epi == W4A_EPI_SILU_MUL) {
    const int nh = n / 2, total = B * nh;
#pragma unroll 1
    for (int i = blockIdx.x * NT + threadIdx.x; i < total; i += L.nc * NT) {
      const int bb = i / nh, j = i - bb * nh;
      float gs = 0.f, us = 0.f;
#pragma unroll 1
      for (int s = 0; s < ns; ++s) {
        gs += __ldcg(part + ((size_t)s * B + bb) * n + 2 * j);
        us += __ldcg(part + ((size_t)s * B + bb) * n + 2 * j + 1);
      }
      reinterpret_cast<uint16_t*>(d.out)[(size_t)bb * nh + j] = f32_to_bf16(gs / (1.f + expf(-gs)) * us);
    }
    return;
  }
  // one thread per (batch row, 16-row block): rows and their sum of squares
  const int nrb = n / RB, total = B * nrb;
#pragma unroll 1
  for (int i = blockIdx.x * NT + threadIdx.x; i < total; i += L.nc * NT) {
    const int bb = i / nrb, rb = i - bb * nrb;
    float ss = 0.f;
#pragma unroll 1
    for (int r = rb * RB; r < rb * RB + RB; ++r) {
      float y = 0.f;
#pragma unroll 1
      for (int s = 0; s < ns; ++s) y += __ldcg(part + ((size_t)s * B + bb) * n + r);
      reinterpret_cast<float*>(d.out)[(size_t)bb * n + r] = y;
      ss = fmaf(y, y, ss);
    }
    if (d.red_epi == W4A_EPI_SUMSQ) d.aux[(size_t)rb * B + bb] = ss;
  }
}

// ---------------------------------------------------------------------------
// Attention
// ---------------------------------------------------------------------------
template <int HD>
__device__ __forceinline__ void attn_prologue(const PD& d, int seg, bool own_new) {
  const LC& L = lc();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bq = seg / L.nkv, g = seg % L.nkv;
  const int GQ = L.nq / L.nkv;
  float* q = sm_at<float>(SM_QS);
  float* rd = red();
  uint16_t* kn = sm_at<uint16_t>(SM_KNV);
  uint16_t* vn = kn + 128;
  const float qscale = 1.4426950408889634f * rsqrtf(float(HD));
  if (d.newkv) {
    // q, k, v of this sequence are the sums of the QKV slabs (four-row
    // chunks, several in flight per thread); the norms run over the whole Q
    // and K projections.  This group's k and v rows go to scratch.
    const int qd = L.nq * HD, kd = L.nkv * HD, qkv_dim = qd + 2 * kd;
    const float* ybase = d.qpart + (size_t)bq * qkv_dim;
    const size_t sstride = (size_t)L.B * qkv_dim;
    float* kraw = sm_at<float>(SM_ASCR);
    float* vraw = kraw + 128;
    float* wq = vraw + 128;
    const int nq4 = qd / 4, nk4 = kd / 4;
    const int total4 = nq4 + (own_new ? nk4 + HD / 4 : 0);
    float sq = 0.f, sk = 0.f;
    // the norm gains of this thread's first rotation pair, in flight with the
    // slab loads below
    constexpr int H2 = HD / 2;
    float qg1 = 0.f, qg2 = 0.f, kg1 = 0.f, kg2 = 0.f;
    if (tid < GQ * H2) {
      const int h = tid / H2, i = tid - h * H2, row = (g * GQ + h) * HD;
      qg1 = __ldg(d.qnorm + row + i);
      qg2 = __ldg(d.qnorm + row + i + H2);
    }
    if (own_new && tid < H2) {
      kg1 = __ldg(d.knorm + g * HD + tid);
      kg2 = __ldg(d.knorm + g * HD + tid + H2);
    }
    constexpr int JU = 4;
#pragma unroll 1
    for (int c0 = tid; c0 < total4; c0 += JU * NT) {
      int rows[JU];
      float4 v[JU];
#pragma unroll
      for (int j = 0; j < JU; ++j) {
        const int c = c0 + j * NT;
        rows[j] = c < nq4 + nk4 ? 4 * c : qd + kd + g * HD + 4 * (c - nq4 - nk4);
        v[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll 1
      for (int sl = 0; sl < d.qns; sl += 2) {  // two slabs' loads in flight together
        float4 t4[2][JU];
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
          for (int j = 0; j < JU; ++j)
            t4[e][j] = (c0 + j * NT < total4 && sl + e < d.qns) ? ldcg4(ybase + (sl + e) * sstride + rows[j])
                                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
          for (int j = 0; j < JU; ++j) {
            v[j].x += t4[e][j].x;
            v[j].y += t4[e][j].y;
            v[j].z += t4[e][j].z;
            v[j].w += t4[e][j].w;
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
        if (dst) *reinterpret_cast<float4*>(dst) = v[j];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sq += __shfl_xor_sync(0xffffffffu, sq, o);
      sk += __shfl_xor_sync(0xffffffffu, sk, o);
    }
    mark(2);
    if (lane == 0) {
      wq[warp] = sq;
      wq[NW + warp] = sk;
    }
    cbar();
    if (tid < 32) {  // fixed shuffle tree over the warps' sums
      float a = tid < NW ? wq[tid] : 0.f, c = tid < NW ? wq[NW + tid] : 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        c += __shfl_xor_sync(0xffffffffu, c, o);
      }
      if (tid == 0) {
        rd[32] = rsqrtf(a / float(qd) + L.eps);
        rd[33] = rsqrtf(c / float(kd) + L.eps);
      }
    }
    cbar();
    const float rq = rd[32], rk = rd[33];
    const int pos = posb()[bq];
    const double* fr = rope_f(d.type);
    const float ms = d.type ? L.mscale1 : L.mscale0;
#pragma unroll 1
    for (int idx = tid; idx < GQ * H2; idx += NT) {
      const int h = idx / H2, i = idx - h * H2;
      const int row = (g * GQ + h) * HD;
      const bool first = idx == tid;
      const float x1 = q[h * HD + i] * rq * (first ? qg1 : d.qnorm[row + i]);
      const float x2 = q[h * HD + i + H2] * rq * (first ? qg2 : d.qnorm[row + i + H2]);
      float c, s;
      rope_cs(pos, fr[i], ms, c, s);
      q[h * HD + i] = (x1 * c - x2 * s) * qscale;
      q[h * HD + i + H2] = (x2 * c + x1 * s) * qscale;
    }
    if (own_new) {
      if (tid < H2) {
        const int i = tid;
        const float x1 = kraw[i] * rk * kg1;
        const float x2 = kraw[i + H2] * rk * kg2;
        float c, s;
        rope_cs(pos, fr[i], ms, c, s);
        kn[i] = f32_to_bf16(x1 * c - x2 * s);
        kn[i + H2] = f32_to_bf16(x2 * c + x1 * s);
      }
      if (tid < HD) vn[tid] = f32_to_bf16(vraw[tid]);
      cbar();
      const int sn_ = snew(d.type)[bq];
      const size_t row = ((size_t)(d.seqoff + bq) * L.nkv + g) * d.slots + sn_;
      uint16_t* kd_ = reinterpret_cast<uint16_t*>(const_cast<uint8_t*>(d.kc)) + row * HD;
      uint16_t* vd_ = reinterpret_cast<uint16_t*>(const_cast<uint8_t*>(d.vc)) + row * HD;
      if (tid < HD) {
        const int i = tid;
        const int sw = (((i >> 3) ^ (sn_ & 7)) << 3) | (i & 7);
        kd_[sw] = kn[i];
        vd_[sw] = vn[i];
      }
    }
  } else {
    const uint16_t* qin = d.xbf + ((size_t)bq * L.nq + g * GQ) * HD;
#pragma unroll 1
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
    sm_at<uint4>(SM_QF)[tid] = f;
  }
  cbar();
}

// Outputs [lo, hi) of a split segment (head o / HD, dim o % HD) from the
// pieces of CTAs c0 .. c0 + np - 1, one round of loads per batch of PB
// pieces: every output's thread loads the batch's maxima, denominators and
// values together and folds them in piece order.  CTA c0 filed its piece in
// its second slot (the segment is its last), the others in their first.
template <int HD>
__device__ __forceinline__ void merge_pieces(const LC& L, int c0, int np, int lo, int hi, uint16_t* out, int out_f16) {
  constexpr int PB = 24;
#pragma unroll 1
  for (int o = lo + (int)threadIdx.x; o < hi; o += NT) {
    const int h = o / HD, dd = o - h * HD;
    float M = -INFINITY, acc = 0.f, Ls = 0.f;
#pragma unroll 1
    for (int cb = 0; cb < np; cb += PB) {
      float mv[PB], lv[PB], ov[PB];
#pragma unroll
      for (int j = 0; j < PB; ++j) {
        const bool ok = cb + j < np;
        const int c = ok ? c0 + cb + j : c0;
        const float* pc = L.apart + ((size_t)c * 2 + (c == c0 ? 1 : 0)) * ATT_PW + h * (HD + 2);
        mv[j] = ok ? __ldcg(pc + HD) : -INFINITY;
        lv[j] = ok ? __ldcg(pc + HD + 1) : 0.f;
        ov[j] = ok ? __ldcg(pc + dd) : 0.f;
      }
      float Mn = M;
#pragma unroll
      for (int j = 0; j < PB; ++j) Mn = fmaxf(Mn, mv[j]);
      const float rs = exp2f(M - Mn);  // 0 on the first batch (M = -inf)
      acc *= rs;
      Ls *= rs;
#pragma unroll
      for (int j = 0; j < PB; ++j) {
        const float w = exp2f(mv[j] - Mn);  // 0 for the padding
        acc = fmaf(w, ov[j], acc);
        Ls = fmaf(w, lv[j], Ls);
      }
      M = Mn;
    }
    const float v = acc / Ls;
    out[o] = out16(v, out_f16);
  }
}

// The same merge for a short output range (hi - lo <= 64, one to two
// outputs per lane): warp w takes pieces w, w + NW, ..., so the pieces'
// loads spread over all warps; each warp folds its pieces per output into
// shared memory and the range's threads fold the NW warp results in warp
// order.  Every thread of the CTA calls it (one CTA sync).
template <int HD>
__device__ __forceinline__ void merge_pieces_warps(const LC& L, int c0, int np, int lo, int hi, uint16_t* out,
                                                   int out_f16) {
  constexpr int RMAX = 64, PB = 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* sc = sm_at<float>(SM_APW);  // [NW][RMAX][3]: maximum, weighted sum, denominator
#pragma unroll
  for (int ob = 0; ob < RMAX; ob += 32) {
    const int o = lo + ob + lane;
    const bool live = o < hi;
    const int oc = live ? o : lo;
    const int h = oc / HD, dd = oc - h * HD;
    float M = -INFINITY, acc = 0.f, Ls = 0.f;
#pragma unroll 1
    for (int j0 = warp; j0 < np; j0 += PB * NW) {
      float mv[PB], lv[PB], vv[PB];
#pragma unroll
      for (int i = 0; i < PB; ++i) {
        const int j = j0 + i * NW;
        const bool ok = live && j < np;
        const int c = c0 + (j < np ? j : 0);
        const float* pc = L.apart + ((size_t)c * 2 + (c == c0 ? 1 : 0)) * ATT_PW + h * (HD + 2);
        mv[i] = ok ? __ldcg(pc + HD) : -INFINITY;
        lv[i] = ok ? __ldcg(pc + HD + 1) : 0.f;
        vv[i] = ok ? __ldcg(pc + dd) : 0.f;
      }
      float Mn = M;
#pragma unroll
      for (int i = 0; i < PB; ++i) Mn = fmaxf(Mn, mv[i]);
      if (Mn != -INFINITY) {
        const float rs = exp2f(M - Mn);  // 0 while M = -inf
        acc *= rs;
        Ls *= rs;
#pragma unroll
        for (int i = 0; i < PB; ++i) {
          const float w = exp2f(mv[i] - Mn);  // 0 for the padding
          acc = fmaf(w, vv[i], acc);
          Ls = fmaf(w, lv[i], Ls);
        }
        M = Mn;
      }
    }
    float* e = sc + (warp * RMAX + ob + lane) * 3;
    e[0] = M;
    e[1] = acc;
    e[2] = Ls;
  }
  cbar();
  const int t = threadIdx.x;
  if (t < hi - lo) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, sc[(w * RMAX + t) * 3]);
    float acc = 0.f, Ls = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float* e = sc + (w * RMAX + t) * 3;
      if (e[0] != -INFINITY) {
        const float f = exp2f(e[0] - M);
        acc = fmaf(f, e[1], acc);
        Ls = fmaf(f, e[2], Ls);
      }
    }
    const float v = acc / Ls;
    out[lo + t] = out16(v, out_f16);
  }
}

template <int HD>
__device__ __forceinline__ void attn_combine(const PD& d, int seg, int a, int b, int nca) {
  const LC& L = lc();
  const int tid = threadIdx.x;
  const int* st = sst(d.type);
  const int GQ = L.nq / L.nkv;
  const int bq = seg / L.nkv, g = seg % L.nkv;
  const bool split = (st[seg] < a) || (st[seg + 1] > b);
  const float* wp = sm_at<float>(SM_APW);
  uint16_t* out = d.aout + ((size_t)bq * L.nq + g * GQ) * HD;
  const int pslot = (st[seg] < a) ? 0 : 1;
  float* piece = L.apart + ((size_t)blockIdx.x * 2 + pslot) * ATT_PW;
#pragma unroll 1
  for (int idx = tid; idx < GQ * HD; idx += NT) {
    const int h = idx / HD, dd = idx - h * HD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, wp[w * ATT_PW + h * (HD + 2) + HD]);
    float ls = 0.f, os = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float e = exp2f(wp[w * ATT_PW + h * (HD + 2) + HD] - M);
      ls += e * wp[w * ATT_PW + h * (HD + 2) + HD + 1];
      os += e * wp[w * ATT_PW + h * (HD + 2) + dd];
    }
    if (!split) {
      out[h * HD + dd] = out16(os / ls, d.out_f16);
    } else {
      piece[h * (HD + 2) + dd] = os;
      if (dd == 0) {
        piece[h * (HD + 2) + HD] = M;
        piece[h * (HD + 2) + HD + 1] = ls;
      }
    }
  }
  if (!split) return;
  cbar();
  int c0, c1;
  attn_seg_ctas(d.type, seg, nca, c0, c1);
  const int* am = flags() + 4 + 3 * d.type;
  if (am[0]) {
    // Equal split (each CTA in one segment): every CTA of the segment
    // publishes its piece, waits until all of them have, then merges its
    // share of the outputs.  The counters only grow during a launch (the
    // target advances by the pieces per segment each attention phase) and
    // are cleared when the launch ends.
    if (tid == 0) {
      uint32_t* ctr = L.seg_ctr + MAX_SEG + seg;
      const uint32_t target = L.seg_target + uint32_t(c1 - c0 + 1);
      red_release_add(ctr, 1u);
      int ok = 1;
      const long long t0 = clock64();
      while (ld_acquire(ctr) < target) {
        if (ld_volatile_u32(L.ctl + 2) != 0u) {  // another CTA gave up: its piece may never come
          ok = 0;
          break;
        }
        if (clock64() - t0 > L.wait_bar) {
          set_error(EW_BARRIER_TIMEOUT);
          ok = 0;
          break;
        }
      }
      flags()[1] = ok;
    }
    cbar();
    if (!flags()[1]) return;
    const int np = c1 - c0 + 1, j = blockIdx.x - c0, nout = GQ * HD;
    const int lo = nout * j / np, hi = nout * (j + 1) / np;
    if (hi - lo <= 64)  // the same for every thread of the CTA
      merge_pieces_warps<HD>(L, c0, np, lo, hi, out, d.out_f16);
    else
      merge_pieces<HD>(L, c0, np, lo, hi, out, d.out_f16);
    return;
  }
  if (tid == 0) {
    // release this CTA's piece, acquire the others' (last arriver)
    const uint32_t old = atom_add_acqrel(L.seg_ctr + seg, 1u);
    flags()[1] = (int(old) == c1 - c0) ? 1 : 0;
  }
  cbar();
  if (!flags()[1]) return;
  merge_pieces<HD>(L, c0, c1 - c0 + 1, 0, GQ * HD, out, d.out_f16);
  if (tid == 0) L.seg_ctr[seg] = 0u;
}

template <int HD>
__device__ __noinline__ void attn_phase(const PD& d) {
  const LC& L = lc();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int a, b, nca;
  attn_cta_range(d.type, blockIdx.x, a, b, nca);
  if (a >= b) return;
  const int* st = sst(d.type);
  const int GQ = L.nq / L.nkv;
  int seg = 0;
#pragma unroll 1
  for (int u = a; u < b;) {
    while (st[seg + 1] <= u) ++seg;
    const int run_end = (b < st[seg + 1]) ? b : st[seg + 1];
    const int bq = seg / L.nkv;
    const int Lk = Lb(d.type)[bq];
    const int sn_ = d.newkv ? snew(d.type)[bq] : -1;
    const int jnew = st[seg] + (sn_ >= 0 ? sn_ / ATT_CTA_KEYS : 0);
    const bool own_new = d.newkv && sn_ >= 0 && jnew >= u && jnew < run_end;
    attn_prologue<HD>(d, seg, own_new);
    if (u == a) mark(3);
    {
      // this warp's keys of CTA units [u, run_end); its (m, l, o) partial goes
      // to shared memory
      Cons C;
      cons_load(C, warp);
      const int g = lane >> 2, t = lane & 3;
      const uint4* qfr = sm_at<uint4>(SM_QF);
      const uint16_t* kn = sm_at<uint16_t>(SM_KNV);
      const uint16_t* vn = kn + 128;
      float m = -INFINITY, lsum = 0.f;
      // O^T tiles: o[j] covers dims [16 j, 16 j + 16) x query heads 0..7 of the group
      float o[HD / 16][4];
#pragma unroll
      for (int j = 0; j < HD / 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
#pragma unroll 1
      for (int jc = u; jc < run_end; ++jc) {
        const int key0 = (jc - st[seg]) * ATT_CTA_KEYS + warp * ATT_KEYS;
        if (key0 >= Lk) continue;
        uint8_t* slot = cons_wait(C, warp, lane);
        uint8_t* Ks = slot;
        uint8_t* Vs = slot + ATT_KEYS * HD * 2;
        const bool patch = own_new && sn_ >= key0 && sn_ < key0 + ATT_KEYS;
        if (patch) {
          const int r = sn_ - key0;  // == sn_ & 7
          uint16_t* kr = reinterpret_cast<uint16_t*>(Ks + r * HD * 2);
          uint16_t* vr = reinterpret_cast<uint16_t*>(Vs + r * HD * 2);
#pragma unroll 1
          for (int i = lane; i < HD; i += 32) {
            const int sw = (((i >> 3) ^ r) << 3) | (i & 7);
            kr[sw] = kn[i];
            vr[sw] = vn[i];
          }
          warp_sync();
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
        cons_release(C, warp, lane, patch);
      }
      cons_store(C, warp, lane);
      lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
      lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
      float* wp = sm_at<float>(SM_APW) + warp * ATT_PW;
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
    }
    cbar();
    if (run_end == b) mark(4);
    attn_combine<HD>(d, seg, a, b, nca);
    cbar();
    if (run_end == b) mark(5);
    u = run_end;
  }
}

// ---------------------------------------------------------------------------
// Argmax (and the sum of the lm_head slabs when K was split)
// ---------------------------------------------------------------------------
__device__ __noinline__ void argmax_phase(const PD& d) {
  const LC& L = lc();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int V = L.vocab, B = L.B;
  const int r0 = int(rstart(V, L.nc, blockIdx.x)), r1 = int(rstart(V, L.nc, blockIdx.x + 1));
  const bool pick = L.next_token != nullptr;
  float* rv = red();
  int* ri = reinterpret_cast<int*>(red() + 32);
  // one pass over the CTA's rows: the logit (sum of the lm_head slabs, or
  // the finished row) and this CTA's greedy candidate (ties: lowest index)
#pragma unroll 1
  for (int bq = 0; bq < B; ++bq) {
    float best = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll 1
    for (int r = r0 + tid; r < r1; r += NT) {
      float y = 0.f;
      if (d.lpart != nullptr) {
#pragma unroll 1
        for (int s0 = 0; s0 < d.lns; s0 += 4) {
          float t[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            t[i] = (s0 + i < d.lns) ? __ldcg(d.lpart + ((size_t)(s0 + i) * B + bq) * V + r) : 0.f;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if (s0 + i < d.lns) y += t[i];
        }
        L.logits[(size_t)bq * V + r] = y;
      } else if (pick) {
        y = __ldcg(L.logits + (size_t)bq * V + r);
      }
      if (y > best || (y == best && r < bi)) {
        best = y;
        bi = r;
      }
    }
    if (!pick) continue;
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
#pragma unroll 1
      for (int w = 0; w < NW; ++w)
        if (rv[w] > bb || (rv[w] == bb && ri[w] < bbi)) {
          bb = rv[w];
          bbi = ri[w];
        }
      L.amax_val[(size_t)blockIdx.x * B + bq] = bb;
      L.amax_idx[(size_t)blockIdx.x * B + bq] = bbi;
    }
    cbar();
  }
  if (!pick || warp != 0) return;
  // the last CTA to file its candidates picks the token: warp 0 reduces
  // the CTAs' candidates (lanes over CTAs, then shuffles)
  int last = 0;
  if (lane == 0) last = int(atom_add_acqrel(L.ctl + 3, 1u)) == L.nc - 1;
  last = __shfl_sync(0xffffffffu, last, 0);
  __syncwarp();  // orders the lanes' reads after lane 0's acquire
  if (!last) return;
#pragma unroll 1
  for (int bq = 0; bq < B; ++bq) {
    float bb = -INFINITY;
    int bbi = 0x7fffffff;
#pragma unroll 1
    for (int c = lane; c < L.nc; c += 32) {
      const float v = __ldcg(L.amax_val + (size_t)c * B + bq);
      const int i = __ldcg(L.amax_idx + (size_t)c * B + bq);
      if (v > bb || (v == bb && i < bbi)) {
        bb = v;
        bbi = i;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bb, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bbi, o);
      if (ov > bb || (ov == bb && oi < bbi)) {
        bb = ov;
        bbi = oi;
      }
    }
    if (lane == 0) L.next_token[bq] = (bbi == 0x7fffffff) ? 0 : bbi;
  }
  if (lane == 0) L.ctl[3] = 0u;
}

// ---------------------------------------------------------------------------
// Launch setup, phase start, the kernel
// ---------------------------------------------------------------------------
__device__ __noinline__ void setup(const EngineParams& P) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, cta = blockIdx.x;
  LC& L = lc();
  if (tid == 0) {
    L.B = P.B;
    L.d = P.d;
    L.nq = P.nq;
    L.nkv = P.nkv;
    L.ffn = P.ffn;
    L.vocab = P.vocab;
    L.window = P.window;
    L.nc = P.nc;
    L.mode = P.mode;
    L.begin = P.phase_begin;
    L.end = P.phase_end;
    L.n_layers = P.n_layers;
    L.seq0 = P.seq0;
    L.pos_const = P.pos_const;
    L.trace_phases = P.trace_phases;
    L.max_ctx = P.max_ctx;
    L.eps = P.eps;
    L.mscale0 = P.mscale[0];
    L.mscale1 = P.mscale[1];
    L.cur_phase = P.phase_begin;
    L.scaled = 0;
    L.final_norm = P.final_norm;
    L.stop = 0;
    L.seg_target = 0u;
    L.wait_bar = P.wait_bar > 0 ? P.wait_bar : WAIT_CYCLES;
    L.pd_hi = P.phase_begin + PD_LEAD;
    L.ctl = P.ws.ctl;
    L.seg_ctr = P.ws.seg_ctr;
    L.apart = P.ws.apart;
    L.amax_val = P.ws.amax_val;
    L.amax_idx = P.ws.amax_idx;
    L.plan = reinterpret_cast<PD*>(P.ws.plan);
    L.trace = P.trace;
    L.tokens = P.tokens;
    L.embed = P.embed;
    L.logits = P.logits;
    L.next_token = P.next_token;
    L.pos = P.pos;
#pragma unroll 1
    for (int s = 0; s < PD_SLOTS; ++s) mbar_init(pd_bar(s), 1u);
  }
  if (lane == 0 && warp < NW) {
#pragma unroll 1
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(ring_bar(warp, s), 1u);
      mbar_init(ring_ebar(warp, s), 1u);
    }
    fence_mbar_init();
  }
  if (tid < 128) sm_at<double>(SM_ROPE)[tid] = P.inv_freq[tid >> 6][tid & 63];
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
  // phase descriptors: the first PD_LEAD + 1 into shared memory, the rest
  // (one thread each) into the workspace plan
  const int begin = P.phase_begin, end = P.phase_end;
  if (lane == 0 && warp <= PD_LEAD && begin + warp < end) build_pd(P, begin + warp, &pd_slot(begin + warp));
  if (lane == 0 && warp > PD_LEAD) {
    const int q = begin + PD_LEAD + 1 + cta + P.nc * (warp - PD_LEAD - 1);
    if (q < end) build_pd(P, q, reinterpret_cast<PD*>(P.ws.plan) + q);
  }
  __syncthreads();
  if (P.mode != MODE_GEMV && tid < 2) {
    int* st = sst(tid);
    st[0] = 0;
    bool equal = true;
    const int S = B * P.nkv;
#pragma unroll 1
    for (int s = 0; s < S; ++s) {
      const int Lk = Lb(tid)[s / P.nkv];
      st[s + 1] = st[s] + (Lk + ATT_CTA_KEYS - 1) / ATT_CTA_KEYS;
      equal &= (st[s + 1] - st[s]) == st[1];
    }
    int* am = flags() + 4 + 3 * tid;
    const int n = st[1];
    am[0] = (equal && n > 0 && S <= P.nc) ? 1 : 0;
    am[1] = S > 0 ? P.nc / S : 0;
    am[2] = min(am[1], n);
  }
  // GEMV unit ranges of this CTA and its warps, per geometry
  if (tid < 5 * NW) {
    const int gi = tid / NW, w = tid - gi * NW;
    const Geo& g = P.geo[gi];
    int a = 0, b = 0, wa = 0, wb = 0, x4 = 0, x5 = 0, x6 = 0;
    if (g.nca > 0 && g.kps > 0 && g.nrb > 0) {
      gemv_cta_range(g, cta, a, b);
      warp_range(a, b, w, wa, wb);
      const int upsl = g.nrb * g.kps;
      x4 = wa / upsl;
      const int r = wa - x4 * upsl;
      x5 = r / g.kps;
      x6 = r - x5 * g.kps;
    }
    // the CTA-level close of a segment split between warps (the warp holding
    // its last unit sums the pieces of warps w0..w in order)
    int cw0 = 0, cmask = 0, cs = 0, crb = 0;
    if (g.nca > 0 && g.kps > 0 && g.nrb > 0 && wa < wb && wa % g.kps != 0) {
      const int S = wa / g.kps;
      if ((S + 1) * g.kps <= wb) {
        int w0 = w;
        while (w0 > 0) {
          int pa, pb;
          warp_range(a, b, w0 - 1, pa, pb);
          if (pb <= S * g.kps) break;
          --w0;
        }
        for (int w2 = w0; w2 <= w; ++w2) {
          int a2, b2;
          warp_range(a, b, w2, a2, b2);
          if (a2 >= b2) cmask |= 1 << (16 + w2 - w0);
          else if (S != a2 / g.kps) cmask |= 1 << (w2 - w0);
        }
        cw0 = w0 + 1;
        cs = S / g.nrb;
        crb = S - cs * g.nrb;
      }
    }
    // the CTA's x range: the slabs its segments touch
    int kbase = 0, klen = 0;
    if (a < b) {
      const int upsl = g.nrb * g.kps, KS = g.kps * (gi == 4 ? BF_KC : fmt_kc(P.fmt));
      const int s0 = a / upsl, s1 = (b - 1) / upsl;
      kbase = s0 * KS;
      klen = (s1 - s0 + 1) * KS;
    }
    int4* e = sm_at<int4>(SM_CTAB) + (gi * NW + w) * 4;
    e[0] = make_int4(wa, wb, x4, x5);
    e[1] = make_int4(x6, a, b, 0);
    e[2] = make_int4(cw0, cmask, cs, crb);
    e[3] = make_int4(kbase, klen, 0, 0);
  }
  // ring state: nothing taken yet, the copy warp's cursor before the first phase
  if (lane == 0 && warp < NW) {
    Ring* s = ring_state(warp);
    *reinterpret_cast<uint4*>(s) = make_uint4(0u, 0u, 0u, 0u);
    s->ld.kind = CUR_WAIT;
    s->ld.p = begin;
  }
  __syncthreads();
}

// Copy descriptor q from the workspace plan into its shared-memory slot
// (thread 0).  The plan was written with generic stores by every CTA during
// setup and is read by the copy engine, so the first copy runs after the
// first grid barrier and behind one proxy fence.
__device__ __forceinline__ void pd_fetch(int q) {
  LC& L = lc();
  if (q == L.begin + PD_LEAD + 1) fence_proxy_async_all();
  mbar_expect_tx(pd_bar(q), (uint32_t)sizeof(PD));
  bulk_g2s(&pd_slot(q), L.plan + q, (uint32_t)sizeof(PD), pd_bar(q));
  L.pd_hi = q;
}
// Before the CTA exits (thread 0): the descriptor copies still in flight land
// first.  On the normal path every issued copy has been waited for already;
// a launch that leaves its phase loop early (a wait ran out) may have issued
// up to PD_LEAD copies that no phase consumed.  The last PD_SLOTS copies are
// one per slot, so each one's mbarrier phase is the one to wait for.
__device__ __noinline__ void pd_drain() {
  const LC& L = lc();
  const int q0 = max(L.begin + PD_LEAD + 1, L.pd_hi - PD_SLOTS + 1);
#pragma unroll 1
  for (int q = q0; q <= L.pd_hi; ++q) {
    const uint32_t par = uint32_t((q - L.begin - PD_LEAD - 1) / PD_SLOTS) & 1u;
    const long long t0 = clock64();
    while (!mbar_try_wait(pd_bar(q), par)) {
      if (clock64() - t0 > WAIT_CYCLES) {
        set_error(EW_DRAIN_TIMEOUT);
        return;
      }
    }
  }
}
// Before the barrier into phase p (thread 0, while the other CTAs finish):
// descriptor p ready in shared memory and the copy of descriptor p + PD_LEAD
// under way; the barrier's CTA sync then publishes descriptor p.  The copy
// for phase begin + 1 waits for the first barrier (see pd_fetch).
__device__ __forceinline__ void phase_prep(int p) {
  if (threadIdx.x == 0) {
    const LC& L = lc();
    pd_ready(p, true);
    const int q = p + PD_LEAD;
    if (q < L.end && q > L.begin + PD_LEAD + 1) pd_fetch(q);
  }
}

// NW math warps run the phases; warp NW is the copy warp.
template <int NB, int HD>
__global__ void __launch_bounds__(NTH, 1) w4a_engine_kernel(const __grid_constant__ EngineParams P) {
  const uint64_t t_entry = P.trace != nullptr ? globaltimer() : 0ull;
  setup(P);
  // trace: the CTA's start in stamp 7 of the first phase (setup = stamp 0 - stamp 7)
  if (threadIdx.x == 0 && P.trace != nullptr && P.phase_begin < P.trace_phases)
    P.trace[((size_t)P.phase_begin * P.nc + blockIdx.x) * 8 + 7] = t_entry;
  if (threadIdx.x >= NT) {
    copy_warp<HD>();
    return;
  }
  const int begin = lc().begin, end = lc().end;
  stage_reset<NB>();
  cbar();
#pragma unroll 1
  for (int p = begin; p < end; ++p) {
    if (p != begin) {
      if (!grid_wait(uint32_t(p - begin) * uint32_t(lc().nc))) break;
    }
    if (threadIdx.x == 0) {
      lc().cur_phase = p;
      if (p == begin + 1 && p + PD_LEAD < end) pd_fetch(p + PD_LEAD);
    }
    mark(0);
    mark(1);
    const PD& d = pd_slot(p);
    const int kind = d.kind;
    if (kind == PK_GEMV_S32)
      gemv_phase<NB, HD, true>(d);
    else if (is_gemv_kind(kind))
      gemv_phase<NB, HD, false>(d);
    else if (kind == PK_ATTN) {
      attn_phase<HD>(d);
      // every CTA advances the equal-split counters' target (see attn_combine);
      // segments of one CTA (meff = 1) are not split and touch no counter
      const int* am = flags() + 4 + 3 * d.type;
      if (threadIdx.x == 0 && am[0] && am[2] > 1) lc().seg_target += uint32_t(am[2]);
    }
    else if (kind == PK_REDUCE)
      reduce_phase(d);
    else
      argmax_phase(d);
    grid_arrive();
    mark(6);
    stage_reset<NB>();  // the phase's shared scratch is free once every warp has arrived
    if (p + 1 < end) phase_prep(p + 1);
  }
  cbar();
  if (threadIdx.x == 0) {
    pd_drain();
    *reinterpret_cast<volatile int*>(&lc().stop) = 1;
    uint32_t* ctl = lc().ctl;
    __threadfence();
    const uint32_t old = atomicAdd(ctl + 1, 1u);
    if (int(old) == lc().nc - 1) {
      ctl[0] = 0u;
      ctl[1] = 0u;
#pragma unroll 1
      for (int i = 0; i < MAX_SEG; ++i) lc().seg_ctr[MAX_SEG + i] = 0u;  // equal-split attention counters
      __threadfence();
    }
  }
}

}  // namespace w4a
