// C-ABI entry points (include/w4a.h): argument checks, workspace layout, launches.
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "engine.cuh"
#include "w4a_internal.h"

namespace w4a {
cudaError_t launch_pack(const void*, int, int64_t, int64_t, uint32_t*, uint16_t*, uint32_t*, cudaStream_t);
cudaError_t launch_tile(const uint32_t*, const uint16_t*, const uint32_t*, int64_t, int64_t, int, uint8_t*,
                        cudaStream_t);
cudaError_t launch_tile_bf16(const uint16_t*, int64_t, int64_t, uint8_t*, cudaStream_t);
cudaError_t launch_unpack(const uint32_t*, const uint16_t*, const uint32_t*, const uint8_t*, int64_t, int64_t, int,
                          float*, cudaStream_t);
cudaError_t launch_kv_copy(uint16_t*, const uint16_t*, int, int, int, int, int, int, int, cudaStream_t);
cudaError_t launch_qk_prep(int, int, int, int, float, const double*, float, const float*, const float*, const float*,
                           const float*, const float*, const int32_t*, uint16_t*, uint16_t*, uint16_t*, int,
                           cudaStream_t);
cudaError_t launch_sample(const float*, int, int, float, float, const float*, int32_t*, double*, cudaStream_t);
cudaError_t launch_dequant_f16(const uint8_t*, int64_t, int64_t, int, uint16_t*, cudaStream_t);
cudaError_t launch_tile_s32(const uint32_t*, const uint16_t*, int64_t, int64_t, int, uint8_t*, cudaStream_t);
cudaError_t launch_unpack_s32(const uint32_t*, const uint16_t*, const uint8_t*, int64_t, int64_t, int, float*, cudaStream_t);
cudaError_t launch_gemm_f16(const uint16_t*, const uint16_t*, int, int, int, int, void*, int, const float*, uint32_t*,
                            int, cudaStream_t, int, const uint8_t* const*, const int64_t*, const int64_t*, int,
                            uint16_t* const*);
cudaError_t launch_flash_prefill(const uint16_t*, const uint16_t*, const uint16_t*, const uint16_t*, const uint16_t*,
                                 uint16_t*, int, int, int, int, int, int, int, int, uint32_t*, cudaStream_t);
cudaError_t launch_kv_append(uint16_t*, uint16_t*, const uint16_t*, const uint16_t*, int, int, int, int, int, int, int,
                             cudaStream_t);
cudaError_t launch_embed_rows(const int32_t*, int, const uint16_t*, int, int, float*, uint16_t*, float*, uint32_t*,
                              cudaStream_t);
cudaError_t launch_resid_rows(const float*, const float*, int, int, float, float*, uint16_t*, float*, cudaStream_t);
cudaError_t launch_final_row(const float*, const float*, int, float, uint16_t*, cudaStream_t);
cudaError_t launch_head_gemv(const uint8_t*, int, int, const uint16_t*, float*, int*, int, cudaStream_t);
cudaError_t launch_qk_rows(const float*, const float*, const float*, uint16_t*, uint16_t*, uint16_t*, const double*,
                           float, float, int, int, int, int, int, cudaStream_t);
}  // namespace w4a

using namespace w4a;

static_assert(sizeof(EngineParams) <= 32000, "kernel parameters must fit the 32 KB launch limit");

// ---------------------------------------------------------------------------
// errors
// ---------------------------------------------------------------------------
static thread_local char g_err[512] = "";

static int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}
static int cuda_fail(cudaError_t e, const char* what) {
  return fail(W4A_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}
#define CK(call)                                        \
  do {                                                  \
    cudaError_t e_ = (call);                            \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
  } while (0)

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static cudaStream_t S(void* s) { return static_cast<cudaStream_t>(s); }

// ---------------------------------------------------------------------------
// device properties and engine launch
// ---------------------------------------------------------------------------
struct DevInfo {
  int ok = 0;
  int sms = 0;
  int cc = 0;
  int attr_set = 0;
};
static DevInfo g_dev[64];
static std::mutex g_dev_mu;

static int device_info(DevInfo** out) {
  int dev = 0;
  CK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(W4A_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& di = g_dev[dev];
  if (!di.ok) {
    cudaDeviceProp p;
    CK(cudaGetDeviceProperties(&p, dev));
    di.sms = p.multiProcessorCount;
    di.cc = p.major * 10 + p.minor;
    di.ok = 1;
  }
  if (di.cc != 100) return fail(W4A_ERR_UNSUPPORTED, "this library is built for sm_100a; device is sm_%d", di.cc);
  *out = &di;
  return W4A_OK;
}

static const void* engine_fn(int nb, int hd) {
  if (nb == 1 && hd == 64) return reinterpret_cast<const void*>(&w4a_engine_kernel<1, 64>);
  if (nb == 1 && hd == 128) return reinterpret_cast<const void*>(&w4a_engine_kernel<1, 128>);
  if (nb == 2 && hd == 64) return reinterpret_cast<const void*>(&w4a_engine_kernel<2, 64>);
  if (nb == 2 && hd == 128) return reinterpret_cast<const void*>(&w4a_engine_kernel<2, 128>);
  return nullptr;
}
static int engine_smem(int) { return SM_TOTAL; }
static int nb_for(int batch) { return batch <= 8 ? 1 : 2; }

static void* g_trace = nullptr;
static size_t g_trace_bytes = 0;

static int phases_per_launch() {
  const char* e = getenv("W4A_PHASES_PER_LAUNCH");
  if (!e || !*e) return 0;
  const int v = atoi(e);
  return v > 0 ? v : 0;
}

// Debugging knob: W4A_BARRIER_WAIT_CYCLES bounds every wait of a CTA for the
// other CTAs (the grid barrier, the attention segment merge); unset or <= 0
// keeps the default of ~2 s.  A wait that runs out sets the timeout bit of
// the workspace's error word and the launch unwinds.
static long long barrier_wait_cycles() {
  const char* e = getenv("W4A_BARRIER_WAIT_CYCLES");
  if (!e || !*e) return 0;
  const long long v = atoll(e);
  return v > 0 ? v : 0;
}

// Runs phases [P.phase_begin, P.phase_end).  Every launch is cooperative, so
// that all CTAs are resident together: the grid barriers between phases and
// the attention merge of a segment split over CTAs (which waits for the
// segment's other CTAs even inside one phase) depend on it.
static int launch_engine(EngineParams& P, int nb, int hd, cudaStream_t st) {
  DevInfo* di;
  int rc = device_info(&di);
  if (rc) return rc;
  const void* fn = engine_fn(nb, hd);
  if (!fn) return fail(W4A_ERR_UNSUPPORTED, "head_dim %d", hd);
  const int smem = engine_smem(nb);
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    const int bit = 1 << ((nb - 1) * 2 + (hd == 128 ? 1 : 0));
    if (!(di->attr_set & bit)) {
      CK(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
      int occ = 0;
      CK(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, NTH, smem));
      if (occ < 1) return fail(W4A_ERR_UNSUPPORTED, "engine kernel does not fit on an SM");
      di->attr_set |= bit;
    }
  }
  P.nc = di->sms;
  P.wait_bar = barrier_wait_cycles();
  P.trace = nullptr;
  P.trace_phases = 0;
  if (g_trace && P.mode == MODE_DECODE) {
    P.trace = static_cast<uint64_t*>(g_trace);
    P.trace_phases = int(g_trace_bytes / ((size_t)P.nc * 64));
  }
  const int begin = P.phase_begin, end = P.phase_end;
  int chunk = phases_per_launch();
  if (chunk <= 0) chunk = end - begin;
  for (int p0 = begin; p0 < end; p0 += chunk) {
    P.phase_begin = p0;
    P.phase_end = (p0 + chunk < end) ? p0 + chunk : end;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(P.nc);
    cfg.blockDim = dim3(NTH);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {&P};
    cudaError_t e = cudaLaunchKernelExC(&cfg, fn, args);
    if (e != cudaSuccess) {
      P.phase_begin = begin;
      P.phase_end = end;
      return cuda_fail(e, "engine launch");
    }
  }
  P.phase_begin = begin;
  P.phase_end = end;
  return W4A_OK;
}

// ---------------------------------------------------------------------------
// workspace layout
// ---------------------------------------------------------------------------
static size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
  size_t ctl, seg, apart, amax_v, amax_i, y_part, o, a_part, gu_part, h, f_part, lg_part, xA, xB, g_part, a_red,
      f_red, rb_ctr, plan, total;
};

struct Dims {
  int d, nq, nkv, hd, ffn, vocab, n_layers;
  int fmt;  // W4Fmt of the int4 matrices
};

// A GEMV geometry the engine can run: some k-split fits shared memory and no
// CTA's segments span more than two k-slabs.
static int geo_check(const Geo& g, long long n, long long k, int B) {
  if (g.ns <= 0) return fail(W4A_ERR_SHAPE, "no k-split of %lld x %lld fits shared memory at batch %d", n, k, B);
  const long long upsl = (long long)g.nrb * g.kps;
  for (int c = 0; c < g.nca; ++c) {
    int a, b;
    gemv_cta_range(g, c, a, b);
    if (a < b && (b - 1) / upsl - a / upsl > 1)
      return fail(W4A_ERR_SHAPE, "%lld x %lld at batch %d needs more k-slabs per CTA than fit", n, k, B);
  }
  return W4A_OK;
}

// Geometries of the decode step's GEMVs: qkv, o, gate/up, down, lm_head.
static int decode_geos(const Dims& dm, int B, int nc, Geo* g) {
  const int nb = nb_for(B);
  const long long qd = (long long)dm.nq * dm.hd, qkv = (long long)(dm.nq + 2 * dm.nkv) * dm.hd;
  const long long n[5] = {qkv, dm.d, 2LL * dm.ffn, dm.d, (dm.vocab + RB - 1) / RB * (long long)RB};
  const long long k[5] = {dm.d, qd, dm.d, dm.ffn, dm.d};
  // every CTA of the consuming phase reads the whole qkv, O, gate/up (counted
  // as whole: one slab keeps the fused SiLU epilogue) and down outputs;
  // argmax reads each logit once
  const int readers[5] = {nc, nc, nc, nc, 1};
  for (int i = 0; i < 5; ++i) {
    g[i] = gemv_geo(n[i], k[i], i == 4 ? BF_KC : fmt_kc(dm.fmt), B, nb, nc, readers[i]);
    const int rc = geo_check(g[i], n[i], k[i], B);
    if (rc) return rc;
  }
  return W4A_OK;
}

// decode != 0: the decode step's activations; attn != 0: attention pieces;
// gemv_n > 0: a standalone GEMV of gemv_n x gemv_k.
static int ws_layout(int B, int nc, const Dims& dm, int attn, int decode, long long gemv_n, long long gemv_k,
                     WsLayout* L) {
  Geo g[5] = {};
  if (decode) {
    const int rc = decode_geos(dm, B, nc, g);
    if (rc) return rc;
  }
  Geo gs = {};
  if (gemv_n > 0) {
    gs = gemv_geo(gemv_n, gemv_k, fmt_kc(dm.fmt), B, nb_for(B), nc, 1);
    const int rc = geo_check(gs, gemv_n, gemv_k, B);
    if (rc) return rc;
  }
  size_t off = 0;
  auto put = [&](size_t bytes) {
    const size_t o = off;
    off += al256(bytes);
    return o;
  };
  const size_t qkv = (size_t)(dm.nq + 2 * dm.nkv) * dm.hd;
  L->ctl = put(256);
  L->seg = put((size_t)2 * MAX_SEG * 4);  // last-arriver counters, then equal-split counters
  L->apart = put(attn ? (size_t)nc * 2 * MAX_GQ * (dm.hd + 2) * 4 : 0);
  L->amax_v = put(decode ? (size_t)nc * B * 4 : 0);
  L->amax_i = put(decode ? (size_t)nc * B * 4 : 0);
  L->y_part = put(decode ? (size_t)g[0].ns * B * qkv * 4 : 0);
  L->o = put(decode ? (size_t)B * dm.nq * dm.hd * 2 : 0);
  L->a_part = put(decode ? (size_t)g[1].ns * B * dm.d * 4 : 0);
  L->gu_part = put(decode && g[2].ns > 1 ? (size_t)g[2].ns * B * 2 * dm.ffn * 4 : 0);
  L->h = put(decode ? (size_t)B * dm.ffn * 2 : 0);
  L->f_part = put(decode ? (size_t)g[3].ns * B * dm.d * 4 : 0);
  L->lg_part = put(decode && g[4].ns > 1 ? (size_t)g[4].ns * B * dm.vocab * 4 : 0);
  L->xA = put(decode ? (size_t)B * dm.d * 4 : 0);
  L->xB = put(decode ? (size_t)B * dm.d * 4 : 0);
  L->g_part = put(gemv_n > 0 ? (size_t)gs.ns * B * gemv_n * 4 : 0);
  // summed rows [B][d], then the 16-row blocks' sums of squares [B][d / 16]
  const size_t red_bytes = (size_t)B * dm.d * 4 + (size_t)B * ((dm.d + RB - 1) / RB) * 4;
  L->a_red = put(decode && g[1].ns > RED_NS ? red_bytes : 0);
  L->f_red = put(decode && g[3].ns > RED_NS ? red_bytes : 0);
  L->rb_ctr = put(decode ? (size_t)2 * MAX_RBC * 4 : 0);
  // phase descriptors: every phase of a decode step (standalone ops use at most two)
  L->plan = put(decode ? (size_t)(5 * dm.n_layers + 2) * sizeof(PD) : 2 * sizeof(PD));
  L->total = off;
  return W4A_OK;
}

static void ws_bind(EngineParams& P, void* ws, const WsLayout& L) {
  uint8_t* b = static_cast<uint8_t*>(ws);
  P.ws.ctl = reinterpret_cast<uint32_t*>(b + L.ctl);
  P.ws.seg_ctr = reinterpret_cast<uint32_t*>(b + L.seg);
  P.ws.apart = reinterpret_cast<float*>(b + L.apart);
  P.ws.amax_val = reinterpret_cast<float*>(b + L.amax_v);
  P.ws.amax_idx = reinterpret_cast<int32_t*>(b + L.amax_i);
  P.ws.y_part = reinterpret_cast<float*>(b + L.y_part);
  P.ws.o = reinterpret_cast<uint16_t*>(b + L.o);
  P.ws.a_part = reinterpret_cast<float*>(b + L.a_part);
  P.ws.gu_part = reinterpret_cast<float*>(b + L.gu_part);
  P.ws.h = reinterpret_cast<uint16_t*>(b + L.h);
  P.ws.f_part = reinterpret_cast<float*>(b + L.f_part);
  P.ws.lg_part = reinterpret_cast<float*>(b + L.lg_part);
  P.ws.xA = reinterpret_cast<float*>(b + L.xA);
  P.ws.xB = reinterpret_cast<float*>(b + L.xB);
  P.ws.g_part = reinterpret_cast<float*>(b + L.g_part);
  P.ws.a_red = reinterpret_cast<float*>(b + L.a_red);
  P.ws.f_red = reinterpret_cast<float*>(b + L.f_red);
  P.ws.rb_ctr = reinterpret_cast<uint32_t*>(b + L.rb_ctr);
  P.ws.plan = b + L.plan;
}

static int nc_for_sizing(int* nc) {
  // Workspace sizes depend on the SM count of the current device; without a
  // device (size queries on a host) assume the B200's 148.
  int dev = 0, count = 0;
  if (cudaGetDeviceCount(&count) != cudaSuccess || count == 0 || cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    *nc = 148;
    return W4A_OK;
  }
  int sms = 0;
  CK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  *nc = sms;
  return W4A_OK;
}

// ---------------------------------------------------------------------------
// RoPE / YaRN tables (host)
// ---------------------------------------------------------------------------
// Plain: f_i = theta^(-2i/d).  YaRN (Peng et al., "YaRN: Efficient Context
// Window Extension of Large Language Models"): dims below the correction range
// keep f_i, dims above it use f_i / factor, a linear ramp blends in between;
// the range comes from the rotation counts beta_fast / beta_slow over the
// original context.  Attention factor 0.1 ln(factor) + 1.
static void rope_tables(const W4AConfig* c, double out[2][64], float ms[2]) {
  const int hd = c->head_dim, half = hd / 2;
  const double th = c->rope_theta;
  double lo = floor(hd * log(c->yarn_orig_ctx / (c->yarn_beta_fast * 2.0 * M_PI)) / (2.0 * log(th)));
  double hi = ceil(hd * log(c->yarn_orig_ctx / (c->yarn_beta_slow * 2.0 * M_PI)) / (2.0 * log(th)));
  if (lo < 0) lo = 0;
  if (hi > hd - 1) hi = hd - 1;
  double span = hi - lo;
  if (span == 0) span = 0.001;
  for (int i = 0; i < 64; ++i) {
    if (i >= half) {
      out[0][i] = out[1][i] = 0.0;
      continue;
    }
    const double f = pow(th, -2.0 * i / hd);
    double r = (i - lo) / span;
    r = r < 0 ? 0 : (r > 1 ? 1 : r);
    out[0][i] = f;
    out[1][i] = (c->yarn_factor > 1.0) ? (f / c->yarn_factor) * r + f * (1.0 - r) : f;
  }
  ms[0] = 1.0f;
  ms[1] = (c->yarn_factor > 1.0) ? float(0.1 * log(c->yarn_factor) + 1.0) : 1.0f;
}

// ---------------------------------------------------------------------------
// model
// ---------------------------------------------------------------------------
struct W4AModel {
  W4AConfig cfg;
  const uint16_t* embed;
  const uint8_t* lm_head;
  const float* final_norm;
  LayerPtrs layers[MAX_LAYERS];
  double inv_freq[2][64];
  float ms[2];
};

static int check_config(const W4AConfig* c) {
  if (!c) return fail(W4A_ERR_ARG, "null config");
  if (c->n_layers < 1 || c->n_layers > MAX_LAYERS) return fail(W4A_ERR_SHAPE, "n_layers %d", c->n_layers);
  if (c->head_dim != 64 && c->head_dim != 128) return fail(W4A_ERR_UNSUPPORTED, "head_dim %d", c->head_dim);
  if (c->n_kv_heads < 1 || c->n_heads % c->n_kv_heads || c->n_heads / c->n_kv_heads > MAX_GQ ||
      c->n_kv_heads > 16)
    return fail(W4A_ERR_SHAPE, "heads %d / kv heads %d", c->n_heads, c->n_kv_heads);
  if (c->group != GROUP && c->group != S32_GROUP)
    return fail(W4A_ERR_UNSUPPORTED, "group %d (128: asymmetric, 32: the symmetric checkpoint format)", c->group);
  const int qd = c->n_heads * c->head_dim;
  if (c->d_model % W4_KC || qd % W4_KC || c->ffn % W4_KC)
    return fail(W4A_ERR_SHAPE, "d_model, heads*head_dim and ffn must be multiples of 512");
  if (c->window < 16 || c->window % 16) return fail(W4A_ERR_SHAPE, "window %d (multiple of 16)", c->window);
  if (c->d_model / RB > MAX_RBC) return fail(W4A_ERR_SHAPE, "d_model %d (at most %d)", c->d_model, MAX_RBC * RB);
  if (c->vocab < 1) return fail(W4A_ERR_SHAPE, "vocab %d", c->vocab);
  return W4A_OK;
}

static Dims dims_of(const W4AConfig& c) {
  return Dims{c.d_model, c.n_heads, c.n_kv_heads, c.head_dim, c.ffn, c.vocab, c.n_layers,
              c.group == S32_GROUP ? FMT_SYM32 : FMT_ASYM128};
}

static int kv_regions(const W4AConfig* c, int batch, int max_ctx, uint64_t* off, int* slots, size_t* total) {
  size_t o = 0;
  for (int l = 0; l < c->n_layers; ++l) {
    const int s = c->full_layers[l] ? max_ctx : c->window;
    const size_t bytes = (size_t)batch * c->n_kv_heads * s * c->head_dim * 2;
    // the engine places V right after K: keep K's size a multiple of 256 bytes
    if (bytes % 256) return fail(W4A_ERR_SHAPE, "KV region of layer %d is not a multiple of 256 bytes", l);
    if (off) off[l] = o;
    if (slots) slots[l] = s;
    o += 2 * al256(bytes);
  }
  *total = o;
  return W4A_OK;
}

extern "C" {

const char* w4a_last_error(void) { return g_err; }
int w4a_version(void) { return 1; }

// ---- codec -------------------------------------------------------------------
int w4a_pack(const void* W, int w_dtype, int64_t n, int64_t k, int group, uint32_t* qweight, uint16_t* scales,
             uint32_t* qzeros, void* stream) {
  if (!W || !qweight || !scales || !qzeros) return fail(W4A_ERR_ARG, "null pointer");
  if (w_dtype != W4A_F32 && w_dtype != W4A_BF16) return fail(W4A_ERR_ARG, "w_dtype %d", w_dtype);
  if (group != GROUP) return fail(W4A_ERR_UNSUPPORTED, "group %d (only 128)", group);
  if (n <= 0 || k <= 0 || n % 8 || k % GROUP) return fail(W4A_ERR_SHAPE, "n %% 8 and k %% 128 must be 0");
  if (!aligned16(W) || !aligned16(qweight) || !aligned16(scales) || !aligned16(qzeros))
    return fail(W4A_ERR_ALIGN, "pointers must be 16-byte aligned");
  CK(launch_pack(W, w_dtype, n, k, qweight, scales, qzeros, S(stream)));
  return W4A_OK;
}

static int tensor_fmt(const W4ATensor* t) { return t->group == S32_GROUP ? FMT_SYM32 : FMT_ASYM128; }

static int check_tensor(const W4ATensor* t) {
  if (!t || !t->qweight) return fail(W4A_ERR_ARG, "null tensor");
  if (t->group != GROUP && t->group != S32_GROUP)
    return fail(W4A_ERR_UNSUPPORTED, "group %d (128: asymmetric, 32: the symmetric checkpoint format)", t->group);
  const int kc = fmt_kc(tensor_fmt(t));
  if (t->layout == W4A_LAYOUT_CANONICAL) {
    if (t->group != GROUP) return fail(W4A_ERR_ARG, "group 32 tensors use W4A_LAYOUT_SYM32");
    if (!t->scales || !t->qzeros) return fail(W4A_ERR_ARG, "canonical tensor needs scales and qzeros");
    if (t->n <= 0 || t->k <= 0 || t->n % 8 || t->k % GROUP) return fail(W4A_ERR_SHAPE, "bad canonical shape");
  } else if (t->layout == W4A_LAYOUT_SYM32) {
    if (t->group != S32_GROUP) return fail(W4A_ERR_ARG, "W4A_LAYOUT_SYM32 needs group 32");
    if (!t->scales) return fail(W4A_ERR_ARG, "the symmetric format needs its scales");
    if (t->n <= 0 || t->k <= 0 || t->n % 8 || t->k % S32_GROUP) return fail(W4A_ERR_SHAPE, "bad canonical shape");
  } else if (t->layout == W4A_LAYOUT_TILED) {
    if (t->n <= 0 || t->k <= 0 || t->n % RB || t->k % kc) return fail(W4A_ERR_SHAPE, "bad tiled shape");
    if (t->row_interleave && (t->n % (2 * RB))) return fail(W4A_ERR_SHAPE, "interleaved n must be a multiple of 32");
  } else {
    return fail(W4A_ERR_ARG, "layout %d", t->layout);
  }
  if (!aligned16(t->qweight)) return fail(W4A_ERR_ALIGN, "qweight not 16-byte aligned");
  return W4A_OK;
}

int w4a_unpack(const W4ATensor* t, float* out, void* stream) {
  int rc = check_tensor(t);
  if (rc) return rc;
  if (!out) return fail(W4A_ERR_ARG, "null output");
  if (t->layout == W4A_LAYOUT_CANONICAL)
    CK(launch_unpack(static_cast<const uint32_t*>(t->qweight), static_cast<const uint16_t*>(t->scales),
                     static_cast<const uint32_t*>(t->qzeros), nullptr, t->n, t->k, 0, out, S(stream)));
  else if (t->layout == W4A_LAYOUT_SYM32)
    CK(launch_unpack_s32(static_cast<const uint32_t*>(t->qweight), static_cast<const uint16_t*>(t->scales), nullptr,
                         t->n, t->k, 0, out, S(stream)));
  else if (t->group == S32_GROUP)
    CK(launch_unpack_s32(nullptr, nullptr, static_cast<const uint8_t*>(t->qweight), t->n, t->k, t->row_interleave,
                         out, S(stream)));
  else
    CK(launch_unpack(nullptr, nullptr, nullptr, static_cast<const uint8_t*>(t->qweight), t->n, t->k,
                     t->row_interleave, out, S(stream)));
  return W4A_OK;
}

int w4a_tiled_bytes(int64_t n, int64_t k, int group, size_t* bytes) {
  if (!bytes) return fail(W4A_ERR_ARG, "null output");
  if (group == S32_GROUP) {
    if (n <= 0 || k <= 0 || n % RB || k % S32_KC) return fail(W4A_ERR_SHAPE, "n %% 16 and k %% 256 must be 0");
    *bytes = (size_t)(n / RB) * (k / S32_KC) * S32_UNIT;
    return W4A_OK;
  }
  if (group != GROUP) return fail(W4A_ERR_UNSUPPORTED, "group %d (128 or 32)", group);
  if (n <= 0 || k <= 0 || n % RB || k % W4_KC) return fail(W4A_ERR_SHAPE, "n %% 16 and k %% 512 must be 0");
  *bytes = (size_t)(n / RB) * (k / W4_KC) * W4_UNIT;
  return W4A_OK;
}

int w4a_tile(const W4ATensor* c, int row_interleave, void* tiled, size_t tiled_bytes, void* stream) {
  int rc = check_tensor(c);
  if (rc) return rc;
  if (c->layout == W4A_LAYOUT_TILED) return fail(W4A_ERR_ARG, "w4a_tile takes a canonical tensor");
  if (!tiled) return fail(W4A_ERR_ARG, "null output");
  size_t need;
  rc = w4a_tiled_bytes(c->n, c->k, c->group, &need);
  if (rc) return rc;
  if (row_interleave && c->n % (2 * RB)) return fail(W4A_ERR_SHAPE, "interleaved n must be a multiple of 32");
  if (tiled_bytes < need) return fail(W4A_ERR_WORKSPACE, "tiled buffer %zu < %zu bytes", tiled_bytes, need);
  if (!aligned16(tiled)) return fail(W4A_ERR_ALIGN, "tiled buffer not 16-byte aligned");
  if (c->layout == W4A_LAYOUT_SYM32)
    CK(launch_tile_s32(static_cast<const uint32_t*>(c->qweight), static_cast<const uint16_t*>(c->scales), c->n, c->k,
                       row_interleave ? 1 : 0, static_cast<uint8_t*>(tiled), S(stream)));
  else
    CK(launch_tile(static_cast<const uint32_t*>(c->qweight), static_cast<const uint16_t*>(c->scales),
                   static_cast<const uint32_t*>(c->qzeros), c->n, c->k, row_interleave ? 1 : 0,
                   static_cast<uint8_t*>(tiled), S(stream)));
  return W4A_OK;
}

int w4a_tiled_bf16_bytes(int64_t n, int64_t k, size_t* bytes) {
  if (!bytes) return fail(W4A_ERR_ARG, "null output");
  if (n <= 0 || k <= 0 || k % BF_KC) return fail(W4A_ERR_SHAPE, "k %% 128 must be 0");
  *bytes = (size_t)((n + RB - 1) / RB) * (k / BF_KC) * BF_UNIT;
  return W4A_OK;
}

int w4a_tile_bf16(const uint16_t* W, int64_t n, int64_t k, void* tiled, size_t tiled_bytes, void* stream) {
  if (!W || !tiled) return fail(W4A_ERR_ARG, "null pointer");
  size_t need;
  int rc = w4a_tiled_bf16_bytes(n, k, &need);
  if (rc) return rc;
  if (tiled_bytes < need) return fail(W4A_ERR_WORKSPACE, "tiled buffer %zu < %zu bytes", tiled_bytes, need);
  if (!aligned16(tiled) || (reinterpret_cast<uintptr_t>(W) & 3u)) return fail(W4A_ERR_ALIGN, "misaligned pointer");
  CK(launch_tile_bf16(W, n, k, static_cast<uint8_t*>(tiled), S(stream)));
  return W4A_OK;
}

// ---- GEMV ----------------------------------------------------------------------
int w4a_gemv_workspace_bytes(const W4ATensor* W, int batch, size_t* bytes) {
  int rc = check_tensor(W);
  if (rc) return rc;
  if (!bytes) return fail(W4A_ERR_ARG, "null output");
  if (batch < 1 || batch > MAX_B) return fail(W4A_ERR_SHAPE, "batch %d (1..16)", batch);
  int nc;
  rc = nc_for_sizing(&nc);
  if (rc) return rc;
  WsLayout L;
  rc = ws_layout(batch, nc, Dims{0, 0, 0, 128, 0, 0, 0, tensor_fmt(W)}, 0, 0, W->n, W->k, &L);
  if (rc) return rc;
  *bytes = L.total;
  return W4A_OK;
}

int w4a_gemv(const W4ATensor* W, const uint16_t* x, int batch, void* out, int epilogue, float* aux, void* ws,
             size_t ws_bytes, void* stream) {
  int rc = check_tensor(W);
  if (rc) return rc;
  if (W->layout != W4A_LAYOUT_TILED) return fail(W4A_ERR_ARG, "w4a_gemv takes a tiled tensor (see w4a_tile)");
  if (!x || !out || !ws) return fail(W4A_ERR_ARG, "null pointer");
  if (batch < 1 || batch > MAX_B) return fail(W4A_ERR_SHAPE, "batch %d (1..16)", batch);
  if (epilogue == W4A_EPI_SUMSQ && !aux) return fail(W4A_ERR_ARG, "W4A_EPI_SUMSQ needs aux");
  if (epilogue == W4A_EPI_SILU_MUL && !W->row_interleave)
    return fail(W4A_ERR_ARG, "W4A_EPI_SILU_MUL needs a row-interleaved (gate/up) tensor");
  if (epilogue < W4A_EPI_NONE || epilogue > W4A_EPI_SILU_MUL) return fail(W4A_ERR_ARG, "epilogue %d", epilogue);
  if (!aligned16(x) || !aligned16(ws)) return fail(W4A_ERR_ALIGN, "x / ws not 16-byte aligned");
  DevInfo* di;
  rc = device_info(&di);
  if (rc) return rc;
  WsLayout L;
  const int fmt = tensor_fmt(W);
  rc = ws_layout(batch, di->sms, Dims{0, 0, 0, 128, 0, 0, 0, fmt}, 0, 0, W->n, W->k, &L);
  if (rc) return rc;
  if (ws_bytes < L.total) return fail(W4A_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
  static thread_local EngineParams P;
  memset(&P, 0, sizeof(P));
  P.mode = MODE_GEMV;
  P.fmt = fmt;
  P.phase_begin = 0;
  // with K split into slabs a second phase sums them and applies the epilogue
  P.geo[0] = gemv_geo(W->n, W->k, fmt_kc(fmt), batch, nb_for(batch), di->sms, 1);
  P.phase_end = (P.geo[0].ns > 1 || epilogue == W4A_EPI_SUMSQ) ? 2 : 1;
  P.B = batch;
  P.pos_const = -1;
  P.g_blob = static_cast<const uint8_t*>(W->qweight);
  P.g_x = x;
  P.g_n = int(W->n);
  P.g_k = int(W->k);
  P.g_epi = epilogue;
  P.g_out = out;
  P.g_aux = aux;
  ws_bind(P, ws, L);
  return launch_engine(P, nb_for(batch), 128, S(stream));
}

// ---- GEMV with library-owned scratch -------------------------------------------------
// A fixed scratch array per device (zero at module load) replaces the caller's
// workspace; its device address is looked up once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[W4A_NOALLOC_SCRATCH_BYTES];
static void* g_noalloc_ptr[64];
static std::mutex g_noalloc_mu;

int w4a_gemv_noalloc(const W4ATensor* W, const uint16_t* x, int batch, void* out, int epilogue, float* aux,
                     void* stream) {
  int rc = check_tensor(W);
  if (rc) return rc;
  size_t need = 0;
  rc = w4a_gemv_workspace_bytes(W, batch, &need);
  if (rc) return rc;
  if (need > (size_t)W4A_NOALLOC_SCRATCH_BYTES)
    return fail(W4A_ERR_WORKSPACE, "%lld x %lld at batch %d needs %zu bytes of scratch (fixed scratch: %d)",
                (long long)W->n, (long long)W->k, batch, need, W4A_NOALLOC_SCRATCH_BYTES);
  int dev = 0;
  CK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(W4A_ERR_UNSUPPORTED, "device index %d", dev);
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
      void* p = nullptr;
      CK(cudaGetSymbolAddress(&p, g_noalloc_scratch));  // with `dev` current
      g_noalloc_ptr[dev] = p;
    }
    scratch = g_noalloc_ptr[dev];
  }
  // the control words (barrier counters, error word) must start at zero
  CK(cudaMemsetAsync(scratch, 0, 256, S(stream)));
  return w4a_gemv(W, x, batch, out, epilogue, aux, scratch, W4A_NOALLOC_SCRATCH_BYTES, stream);
}

// ---- attention ---------------------------------------------------------------------
int w4a_attn_workspace_bytes(int batch, int n_heads, int n_kv_heads, int head_dim, size_t* bytes) {
  if (!bytes) return fail(W4A_ERR_ARG, "null output");
  if (batch < 1 || batch > MAX_B) return fail(W4A_ERR_SHAPE, "batch %d (1..16)", batch);
  if (head_dim != 64 && head_dim != 128) return fail(W4A_ERR_UNSUPPORTED, "head_dim %d", head_dim);
  (void)n_heads;
  (void)n_kv_heads;
  int nc;
  int rc = nc_for_sizing(&nc);
  if (rc) return rc;
  WsLayout L;
  rc = ws_layout(batch, nc, Dims{0, 0, 0, head_dim, 0, 0, 0, 0}, 1, 0, 0, 0, &L);
  if (rc) return rc;
  *bytes = L.total;
  return W4A_OK;
}

int w4a_attn_decode(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache, int batch, int n_heads,
                    int n_kv_heads, int head_dim, int slots, const int32_t* pos, int window, uint16_t* out, void* ws,
                    size_t ws_bytes, void* stream) {
  if (!q || !k_cache || !v_cache || !pos || !out || !ws) return fail(W4A_ERR_ARG, "null pointer");
  if (batch < 1 || batch > MAX_B) return fail(W4A_ERR_SHAPE, "batch %d (1..16)", batch);
  if (head_dim != 64 && head_dim != 128) return fail(W4A_ERR_UNSUPPORTED, "head_dim %d", head_dim);
  if (n_kv_heads < 1 || n_kv_heads > 16 || n_heads % n_kv_heads || n_heads / n_kv_heads > MAX_GQ)
    return fail(W4A_ERR_SHAPE, "heads %d / kv heads %d", n_heads, n_kv_heads);
  if (slots < 16 || slots % 16) return fail(W4A_ERR_SHAPE, "slots %d (multiple of 16)", slots);
  if (window != 0 && window != slots) return fail(W4A_ERR_SHAPE, "window must be 0 (full) or equal to slots");
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(ws)) return fail(W4A_ERR_ALIGN, "misaligned pointer");
  DevInfo* di;
  int rc = device_info(&di);
  if (rc) return rc;
  WsLayout L;
  rc = ws_layout(batch, di->sms, Dims{0, 0, 0, head_dim, 0, 0, 0, 0}, 1, 0, 0, 0, &L);
  if (rc) return rc;
  if (ws_bytes < L.total) return fail(W4A_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
  static thread_local EngineParams P;
  memset(&P, 0, sizeof(P));
  P.mode = MODE_ATTN;
  P.phase_begin = 0;
  P.phase_end = 1;
  P.B = batch;
  P.nq = n_heads;
  P.nkv = n_kv_heads;
  P.hd = head_dim;
  P.pos = pos;
  P.pos_const = -1;
  P.a_q = q;
  P.a_k = k_cache;
  P.a_v = v_cache;
  P.a_out = out;
  P.a_slots = slots;
  P.a_window = window;
  ws_bind(P, ws, L);
  return launch_engine(P, 1, head_dim, S(stream));
}

int w4a_qk_prep(const W4AConfig* cfg, int full, const float* q_raw, const float* k_raw, const float* v_raw,
                const float* q_gain, const float* k_gain, const int32_t* pos, int batch, uint16_t* q_out,
                uint16_t* k_cache, uint16_t* v_cache, int slots, void* stream) {
  if (!cfg || !q_raw || !k_raw || !v_raw || !q_gain || !k_gain || !pos || !q_out || !k_cache || !v_cache)
    return fail(W4A_ERR_ARG, "null pointer");
  if (cfg->head_dim != 64 && cfg->head_dim != 128) return fail(W4A_ERR_UNSUPPORTED, "head_dim %d", cfg->head_dim);
  if (batch < 1 || slots < 1) return fail(W4A_ERR_SHAPE, "batch %d slots %d", batch, slots);
  double tab[2][64];
  float ms[2];
  rope_tables(cfg, tab, ms);
  const int t = full ? 1 : 0;
  CK(launch_qk_prep(batch, cfg->n_heads, cfg->n_kv_heads, cfg->head_dim, float(cfg->eps), tab[t], ms[t], q_raw, k_raw,
                    v_raw, q_gain, k_gain, pos, q_out, k_cache, v_cache, slots, S(stream)));
  return W4A_OK;
}

// ---- KV cache -------------------------------------------------------------------
int w4a_kv_bytes(const W4AConfig* cfg, int batch, int max_ctx, size_t* bytes) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if (!bytes) return fail(W4A_ERR_ARG, "null output");
  if (batch < 1 || max_ctx < 16 || max_ctx % 16) return fail(W4A_ERR_SHAPE, "batch %d max_ctx %d", batch, max_ctx);
  return kv_regions(cfg, batch, max_ctx, nullptr, nullptr, bytes);
}

int w4a_kv_layer(const W4AConfig* cfg, int batch, int max_ctx, int layer, size_t* k_offset, size_t* v_offset,
                 int* slots) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if (layer < 0 || layer >= cfg->n_layers) return fail(W4A_ERR_ARG, "layer %d", layer);
  if (batch < 1 || max_ctx < 16 || max_ctx % 16) return fail(W4A_ERR_SHAPE, "batch %d max_ctx %d", batch, max_ctx);
  uint64_t off[MAX_LAYERS];
  int sl[MAX_LAYERS];
  size_t total;
  kv_regions(cfg, batch, max_ctx, off, sl, &total);
  const size_t kb = (size_t)batch * cfg->n_kv_heads * sl[layer] * cfg->head_dim * 2;
  if (k_offset) *k_offset = off[layer];
  if (v_offset) *v_offset = off[layer] + al256(kb);
  if (slots) *slots = sl[layer];
  return W4A_OK;
}

static int kv_copy(uint16_t* cache, const uint16_t* other, int batch, int nkv, int hd, int slots, int b, int slot0, int n,
                   int to_cache, void* stream) {
  if (n == 0 && slot0 >= 0 && slot0 <= slots && b >= 0 && b < batch) return W4A_OK;  // nothing to copy
  if (!cache || !other) return fail(W4A_ERR_ARG, "null pointer");
  if (b < 0 || b >= batch || slot0 < 0 || n < 0 || slot0 + n > slots || nkv < 1 || hd % 8)
    return fail(W4A_ERR_SHAPE, "rows [%d, %d) of sequence %d outside the region", slot0, slot0 + n, b);
  CK(launch_kv_copy(cache, other, nkv, hd, slots, b, slot0, n, to_cache, S(stream)));
  return W4A_OK;
}

int w4a_kv_write(uint16_t* k, uint16_t* v, int batch, int n_kv_heads, int head_dim, int slots, int b, int slot0, int n,
                 const uint16_t* k_src, const uint16_t* v_src, void* stream) {
  int rc = kv_copy(k, k_src, batch, n_kv_heads, head_dim, slots, b, slot0, n, 1, stream);
  if (rc) return rc;
  return kv_copy(v, v_src, batch, n_kv_heads, head_dim, slots, b, slot0, n, 1, stream);
}

int w4a_kv_read(const uint16_t* k, const uint16_t* v, int batch, int n_kv_heads, int head_dim, int slots, int b,
                int slot0, int n, uint16_t* k_dst, uint16_t* v_dst, void* stream) {
  int rc = kv_copy(const_cast<uint16_t*>(k), k_dst, batch, n_kv_heads, head_dim, slots, b, slot0, n, 0, stream);
  if (rc) return rc;
  return kv_copy(const_cast<uint16_t*>(v), v_dst, batch, n_kv_heads, head_dim, slots, b, slot0, n, 0, stream);
}

// ---- model ------------------------------------------------------------------------
int w4a_model_create(const W4AConfig* cfg, const W4AModelWeights* w, W4AModel** out) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if (!w || !out || !w->embed || !w->lm_head || !w->layers) return fail(W4A_ERR_ARG, "null pointer");
  if (cfg->final_norm && !w->final_norm) return fail(W4A_ERR_ARG, "final_norm gains missing");
  if (!aligned16(w->lm_head) || !aligned16(w->embed) || (w->final_norm && !aligned16(w->final_norm)))
    return fail(W4A_ERR_ALIGN, "embedding, lm_head and final norm must be 16-byte aligned");
  if ((cfg->d_model * 2) % 16) return fail(W4A_ERR_SHAPE, "d_model must be a multiple of 8");
  W4AModel* m = static_cast<W4AModel*>(calloc(1, sizeof(W4AModel)));
  if (!m) return fail(W4A_ERR_ARG, "out of host memory");
  m->cfg = *cfg;
  m->embed = w->embed;
  m->lm_head = static_cast<const uint8_t*>(w->lm_head);
  m->final_norm = w->final_norm;
  for (int l = 0; l < cfg->n_layers; ++l) {
    const W4ALayerWeights& L = w->layers[l];
    if (!L.qkv || !L.o || !L.gate_up || !L.down || !L.q_norm || !L.k_norm || !L.post_attn_norm || !L.post_ffn_norm) {
      free(m);
      return fail(W4A_ERR_ARG, "layer %d: null weight pointer", l);
    }
    if (!aligned16(L.qkv) || !aligned16(L.o) || !aligned16(L.gate_up) || !aligned16(L.down) ||
        !aligned16(L.q_norm) || !aligned16(L.k_norm) || !aligned16(L.post_attn_norm) ||
        !aligned16(L.post_ffn_norm)) {
      free(m);
      return fail(W4A_ERR_ALIGN, "layer %d: weights not 16-byte aligned", l);
    }
    m->layers[l] = LayerPtrs{static_cast<const uint8_t*>(L.qkv), static_cast<const uint8_t*>(L.o),
                             static_cast<const uint8_t*>(L.gate_up), static_cast<const uint8_t*>(L.down),
                             L.q_norm, L.k_norm, L.post_attn_norm, L.post_ffn_norm};
  }
  rope_tables(cfg, m->inv_freq, m->ms);
  *out = m;
  return W4A_OK;
}

int w4a_model_destroy(W4AModel* m) {
  free(m);
  return W4A_OK;
}

int w4a_decode_workspace_bytes(const W4AModel* m, int batch, size_t* bytes) {
  if (!m || !bytes) return fail(W4A_ERR_ARG, "null pointer");
  if (batch < 1 || batch > MAX_B) return fail(W4A_ERR_SHAPE, "batch %d (1..16)", batch);
  int nc;
  int rc = nc_for_sizing(&nc);
  if (rc) return rc;
  WsLayout L;
  rc = ws_layout(batch, nc, dims_of(m->cfg), 1, 1, 0, 0, &L);
  if (rc) return rc;
  *bytes = L.total;
  return W4A_OK;
}

static int decode_common(W4AModel* m, const int32_t* tokens, const W4AKVCache* kv, int seq0, int batch,
                         const int32_t* pos, int pos_const, float* logits, int32_t* next_token, float* dump,
                         int phase_end_kind, void* ws, size_t ws_bytes, cudaStream_t st) {
  const W4AConfig& c = m->cfg;
  if (!tokens || !kv || !kv->base || !ws) return fail(W4A_ERR_ARG, "null pointer");
  if (batch < 1 || batch > MAX_B || batch * c.n_kv_heads > MAX_SEG)
    return fail(W4A_ERR_SHAPE, "batch %d (1..16)", batch);
  if (seq0 < 0 || seq0 + batch > kv->batch) return fail(W4A_ERR_SHAPE, "sequences [%d, %d) outside a cache of %d", seq0,
                                                       seq0 + batch, kv->batch);
  if (kv->max_ctx < 16 || kv->max_ctx % 16) return fail(W4A_ERR_SHAPE, "max_ctx %d (multiple of 16)", kv->max_ctx);
  if (!aligned16(kv->base) || !aligned16(ws)) return fail(W4A_ERR_ALIGN, "kv / ws not 16-byte aligned");
  DevInfo* di;
  int rc = device_info(&di);
  if (rc) return rc;
  WsLayout L;
  rc = ws_layout(batch, di->sms, dims_of(c), 1, 1, 0, 0, &L);
  if (rc) return rc;
  if (ws_bytes < L.total) return fail(W4A_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, L.total);
  static thread_local EngineParams P;
  memset(&P, 0, sizeof(P));
  P.mode = MODE_DECODE;
  P.fmt = c.group == S32_GROUP ? FMT_SYM32 : FMT_ASYM128;
  P.d = c.d_model;
  P.nq = c.n_heads;
  P.nkv = c.n_kv_heads;
  P.hd = c.head_dim;
  P.ffn = c.ffn;
  P.vocab = c.vocab;
  P.window = c.window;
  P.n_layers = c.n_layers;
  P.eps = float(c.eps);
  P.final_norm = c.final_norm;
  memcpy(P.inv_freq, m->inv_freq, sizeof(P.inv_freq));
  P.mscale[0] = m->ms[0];
  P.mscale[1] = m->ms[1];
  for (int l = 0; l < c.n_layers; ++l) {
    P.full[l] = c.full_layers[l] ? 1 : 0;
    P.layers[l] = m->layers[l];
  }
  P.embed = m->embed;
  P.lm_head = m->lm_head;
  P.final_gain = m->final_norm;
  P.kv_base = static_cast<uint8_t*>(kv->base);
  P.kv_batch = kv->batch;
  P.max_ctx = kv->max_ctx;
  size_t total;
  rc = kv_regions(&c, kv->batch, kv->max_ctx, P.kv_off, P.kv_slots, &total);
  if (rc) return rc;
  P.tokens = tokens;
  P.pos = pos;
  P.pos_const = pos_const;
  P.B = batch;
  P.seq0 = seq0;
  P.logits = logits;
  P.next_token = next_token;
  P.dump = dump;
  ws_bind(P, ws, L);
  rc = decode_geos(dims_of(c), batch, di->sms, P.geo);
  if (rc) return rc;
  P.phase_begin = 0;
  P.phase_end = phase_end_kind;
  return launch_engine(P, nb_for(batch), c.head_dim, st);
}

int w4a_decode_step(W4AModel* m, const int32_t* token_ids, const W4AKVCache* kv, int seq0, int batch,
                    const int32_t* pos, float* logits, int32_t* next_token, float* hidden_dump, void* ws,
                    size_t ws_bytes, void* stream) {
  if (!m || !pos || !logits) return fail(W4A_ERR_ARG, "null pointer");
  const int nl = m->cfg.n_layers;
  // the last phase also sums the lm_head's k-slabs into the logits when it is split
  return decode_common(m, token_ids, kv, seq0, batch, pos, -1, logits, next_token, hidden_dump, 5 * nl + 2, ws,
                       ws_bytes, S(stream));
}

// ---- dense prefill -------------------------------------------------------------
// A second stream per device for the fp16 expansion of the next matrix, and
// the events that order it against the GEMMs (created once per device).
// Workspace: the batch-1 decode workspace (its control words, error word
// included, come first; prompts too short for the dense path run as decode
// steps), then the dense path's buffers for `rows` prompt tokens.
struct PfLayout {
  size_t dec, X, X16, scale, Y, Q16, O16, H16, Kn, Vn, XB, ctr, Wq, Wo, Wg, Wd, total;
};
static int pf_layout(const W4AConfig& c, int rows, int nc, PfLayout* P) {
  WsLayout L;
  int rc = ws_layout(1, nc, dims_of(c), 1, 1, 0, 0, &L);
  if (rc) return rc;
  const size_t Tp = rows > 0 ? (size_t)rows : 0;
  const size_t d = c.d_model, qd = (size_t)c.n_heads * c.head_dim, kvd = (size_t)c.n_kv_heads * c.head_dim;
  const size_t qkv = qd + 2 * kvd, ffn = c.ffn;
  size_t off = 0;
  auto put = [&](size_t bytes) {
    const size_t o = off;
    off += al256(bytes);
    return o;
  };
  P->dec = put(L.total);
  P->X = put(Tp * d * 4);
  P->X16 = put(Tp * d * 2);
  P->scale = put(Tp * 4);
  P->Y = put(Tp * (qkv > d ? qkv : d) * 4);
  P->Q16 = put(Tp * qd * 2);
  P->O16 = put(Tp * qd * 2);
  P->H16 = put(Tp * ffn * 2);
  P->Kn = put(Tp * kvd * 2);
  P->Vn = put(Tp * kvd * 2);
  P->XB = put(Tp ? d * 2 : 0);
  P->ctr = put(Tp ? 4 : 0);
  // each of a layer's four matrices expanded to fp16 in its own buffer
  P->Wq = put(Tp ? qkv * d * 2 : 0);
  P->Wo = put(Tp ? d * qd * 2 : 0);
  P->Wg = put(Tp ? 2 * ffn * d * 2 : 0);
  P->Wd = put(Tp ? d * ffn * 2 : 0);
  P->total = off;
  return W4A_OK;
}

// Prompts shorter than this run token by token through the decode launch
// (expanding the weights to fp16 costs about as much as a few decode steps).
static const int PF_MIN_DENSE = 8;

int w4a_prefill_workspace_bytes(const W4AModel* m, int T, size_t* bytes) {
  if (!m || !bytes) return fail(W4A_ERR_ARG, "null pointer");
  if (T < 0) return fail(W4A_ERR_SHAPE, "T %d", T);
  int nc;
  int rc = nc_for_sizing(&nc);
  if (rc) return rc;
  PfLayout P;
  rc = pf_layout(m->cfg, T - 1 >= PF_MIN_DENSE ? T : 0, nc, &P);
  if (rc) return rc;
  *bytes = P.total;
  return W4A_OK;
}

int w4a_prefill(W4AModel* m, const int32_t* tokens, int T, const W4AKVCache* kv, int seq, int start_pos,
                float* last_logits, void* ws, size_t ws_bytes, void* stream) {
  if (!m || !tokens || !kv || !kv->base || !ws) return fail(W4A_ERR_ARG, "null pointer");
  if (T < 0 || start_pos < 0) return fail(W4A_ERR_SHAPE, "T %d start_pos %d", T, start_pos);
  if (T == 0) return W4A_OK;
  const W4AConfig& c = m->cfg;
  if (seq < 0 || seq >= kv->batch) return fail(W4A_ERR_SHAPE, "sequence %d outside a cache of %d", seq, kv->batch);
  if ((long long)start_pos + T > kv->max_ctx && [&] {
        for (int l = 0; l < c.n_layers; ++l)
          if (c.full_layers[l]) return true;
        return false;
      }())
    return fail(W4A_ERR_SHAPE, "positions up to %d do not fit a cache of %d", start_pos + T - 1, kv->max_ctx);
  if (!aligned16(ws)) return fail(W4A_ERR_ALIGN, "workspace not 16-byte aligned");
  DevInfo* di;
  int rc = device_info(&di);
  if (rc) return rc;
  const int nl = c.n_layers;
  const bool dense = T - 1 >= PF_MIN_DENSE;
  const int Tp = T;  // the dense path runs every prompt token, the last one included
  PfLayout P;
  rc = pf_layout(c, dense ? T : 0, di->sms, &P);
  if (rc) return rc;
  if (ws_bytes < P.total) return fail(W4A_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, P.total);
  uint8_t* b = static_cast<uint8_t*>(ws);
  const size_t dec_bytes = P.X - P.dec;
  cudaStream_t st = S(stream);
  if (!dense) {
    for (int i = 0; i < T; ++i) {
      const bool last = (i == T - 1) && last_logits != nullptr;
      rc = decode_common(m, tokens + i, kv, seq, 1, nullptr, start_pos + i, last ? last_logits : nullptr, nullptr,
                         nullptr, last ? 5 * nl + 2 : 5 * nl, b + P.dec, dec_bytes, st);
      if (rc) return rc;
    }
    return W4A_OK;
  }
  uint32_t* err = reinterpret_cast<uint32_t*>(b + P.dec) + 2;  // the decode workspace's error word
  float* X = reinterpret_cast<float*>(b + P.X);
  uint16_t* X16 = reinterpret_cast<uint16_t*>(b + P.X16);
  float* scale = reinterpret_cast<float*>(b + P.scale);
  float* Y = reinterpret_cast<float*>(b + P.Y);
  uint16_t* Q16 = reinterpret_cast<uint16_t*>(b + P.Q16);
  uint16_t* O16 = reinterpret_cast<uint16_t*>(b + P.O16);
  uint16_t* H16 = reinterpret_cast<uint16_t*>(b + P.H16);
  uint16_t* Wbuf[4] = {reinterpret_cast<uint16_t*>(b + P.Wq), reinterpret_cast<uint16_t*>(b + P.Wo),
                       reinterpret_cast<uint16_t*>(b + P.Wg), reinterpret_cast<uint16_t*>(b + P.Wd)};
  uint16_t* Kn = reinterpret_cast<uint16_t*>(b + P.Kn);
  uint16_t* Vn = reinterpret_cast<uint16_t*>(b + P.Vn);
  uint16_t* XB = reinterpret_cast<uint16_t*>(b + P.XB);
  int* hctr = reinterpret_cast<int*>(b + P.ctr);
  const int d = c.d_model, nq = c.n_heads, nkv = c.n_kv_heads, hd = c.head_dim;
  const int qd = nq * hd, qkv = qd + 2 * nkv * hd, ffn = c.ffn;
  uint64_t off[MAX_LAYERS];
  int slots[MAX_LAYERS];
  size_t total;
  rc = kv_regions(&c, kv->batch, kv->max_ctx, off, slots, &total);
  if (rc) return rc;
  const float eps = float(c.eps);
  const Dims dm = dims_of(c);
  // The int4 matrices are expanded to fp16, each into its own buffer, by
  // spare warps of an earlier GEMM (memory-bound work under a tensor-bound
  // product): the gate/up GEMM of layer l expands its down matrix, the down
  // GEMM expands layer l + 1's QKV, O and gate/up; layer 0's first three are
  // expanded up front.  Matrix i (4 per layer) goes to buffer i % 4, last
  // read by the same matrix of the layer before, whose GEMM has finished.
  const int nmat = 4 * nl;
  auto mat = [&](int i, const uint8_t*& blob, int64_t& n, int64_t& k) {
    const LayerPtrs& L = m->layers[i / 4];
    switch (i % 4) {
      case 0: blob = L.qkv; n = qkv; k = d; break;
      case 1: blob = L.o; n = d; k = qd; break;
      case 2: blob = L.gu; n = 2LL * ffn; k = d; break;
      default: blob = L.down; n = d; k = ffn; break;
    }
  };
  auto gemm = [&](int i, const uint16_t* A, int epi, void* out, int ldo, const float* rsc) -> int {
    const uint8_t* blob;
    int64_t n, k;
    mat(i, blob, n, k);
    const uint8_t* nb[3];
    int64_t nn[3], nk[3];
    uint16_t* nd[3];
    int cnt = 0;
    auto add = [&](int j) {
      if (j >= nmat) return;
      mat(j, nb[cnt], nn[cnt], nk[cnt]);
      nd[cnt] = Wbuf[j % 4];
      ++cnt;
    };
    if (i % 4 == 2) add(i + 1);
    if (i % 4 == 3) {
      add(i + 1);
      add(i + 2);
      add(i + 3);
    }
    CK(launch_gemm_f16(A, Wbuf[i % 4], Tp, int(n), int(k), epi, out, ldo, rsc, err, di->sms, st, cnt, nb, nn, nk,
                       dm.fmt, nd));
    return W4A_OK;
  };
  for (int i = 0; i < 3 && i < nmat; ++i) {
    const uint8_t* blob;
    int64_t n, k;
    mat(i, blob, n, k);
    CK(launch_dequant_f16(blob, n, k, dm.fmt, Wbuf[i], st));
  }
  CK(launch_embed_rows(tokens, Tp, m->embed, c.vocab, d, X, X16, scale, err, st));
  for (int l = 0; l < nl; ++l) {
    const LayerPtrs& L = m->layers[l];
    const int full = c.full_layers[l] ? 1 : 0;
    const int win = full ? 0 : c.window;
    uint16_t* kc = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(kv->base) + off[l]);
    uint16_t* vc = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(kc) +
                                               al256((size_t)kv->batch * nkv * slots[l] * hd * 2));
    const int i = 4 * l;
    if ((rc = gemm(i, X16, 0, Y, qkv, scale))) return rc;
    CK(launch_qk_rows(Y, L.q_norm, L.k_norm, Q16, Kn, Vn, m->inv_freq[full], m->ms[full], eps, Tp, nq, nkv, hd,
                      start_pos, st));
    CK(launch_flash_prefill(Q16, kc, vc, Kn, Vn, O16, Tp, nq, nkv, hd, slots[l], win, start_pos, seq, err, st));
    CK(launch_kv_append(kc, vc, Kn, Vn, nkv, hd, slots[l], win, seq, start_pos, Tp, st));
    if ((rc = gemm(i + 1, O16, 0, Y, d, nullptr))) return rc;
    CK(launch_resid_rows(Y, L.attn_norm, Tp, d, eps, X, X16, scale, st));
    if ((rc = gemm(i + 2, X16, 1, H16, ffn, scale))) return rc;
    if ((rc = gemm(i + 3, H16, 0, Y, d, nullptr))) return rc;
    CK(launch_resid_rows(Y, L.ffn_norm, Tp, d, eps, X, X16, scale, st));
  }
  // the last token's logits: the final norm of its residual, then the lm_head
  if (last_logits != nullptr) {
    CK(launch_final_row(X + (size_t)(T - 1) * d, c.final_norm ? m->final_norm : nullptr, d, eps, XB, st));
    CK(launch_head_gemv(m->lm_head, c.vocab, d, XB, last_logits, hctr, di->sms, st));
  }
  return W4A_OK;
}

// ---- int4 GEMM (the prefill's projections) ---------------------------------------
int w4a_gemm_workspace_bytes(const W4ATensor* W, size_t* bytes) {
  int rc = check_tensor(W);
  if (rc) return rc;
  if (!bytes) return fail(W4A_ERR_ARG, "null output");
  *bytes = 256 + al256((size_t)W->n * W->k * 2);
  return W4A_OK;
}

int w4a_gemm(const W4ATensor* W, const uint16_t* x, int M, const float* row_scale, void* out, int epilogue, void* ws,
             size_t ws_bytes, void* stream) {
  int rc = check_tensor(W);
  if (rc) return rc;
  if (W->layout != W4A_LAYOUT_TILED) return fail(W4A_ERR_ARG, "w4a_gemm takes a tiled tensor (see w4a_tile)");
  if (!x || !out || !ws) return fail(W4A_ERR_ARG, "null pointer");
  if (M < 1) return fail(W4A_ERR_SHAPE, "M %d", M);
  if (epilogue != W4A_EPI_NONE && epilogue != W4A_EPI_SILU_MUL) return fail(W4A_ERR_ARG, "epilogue %d", epilogue);
  if (epilogue == W4A_EPI_SILU_MUL && !W->row_interleave)
    return fail(W4A_ERR_ARG, "W4A_EPI_SILU_MUL needs a row-interleaved (gate/up) tensor");
  if (!aligned16(x) || !aligned16(out) || !aligned16(ws)) return fail(W4A_ERR_ALIGN, "x / out / ws not 16-byte aligned");
  size_t need = 0;
  rc = w4a_gemm_workspace_bytes(W, &need);
  if (rc) return rc;
  if (ws_bytes < need) return fail(W4A_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
  DevInfo* di;
  rc = device_info(&di);
  if (rc) return rc;
  uint8_t* b = static_cast<uint8_t*>(ws);
  uint16_t* W16 = reinterpret_cast<uint16_t*>(b + 256);
  uint32_t* err = reinterpret_cast<uint32_t*>(b) + 2;
  cudaStream_t st = S(stream);
  CK(launch_dequant_f16(static_cast<const uint8_t*>(W->qweight), W->n, W->k, tensor_fmt(W), W16, st));
  const int silu = epilogue == W4A_EPI_SILU_MUL ? 1 : 0;
  CK(launch_gemm_f16(x, W16, M, int(W->n), int(W->k), silu, out, silu ? int(W->n / 2) : int(W->n), row_scale, err,
                     di->sms, st, 0, nullptr, nullptr, nullptr, 0, nullptr));
  return W4A_OK;
}

// ---- attention over a prompt ------------------------------------------------------
int w4a_attn_prefill(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache, int batch, int seq,
                     int n_heads, int n_kv_heads, int head_dim, int slots, int window, int start_pos, int T,
                     const uint16_t* k_new, const uint16_t* v_new, uint16_t* out, void* ws, size_t ws_bytes,
                     void* stream) {
  if (!q || !k_cache || !v_cache || !k_new || !v_new || !out || !ws) return fail(W4A_ERR_ARG, "null pointer");
  if (head_dim != 64 && head_dim != 128) return fail(W4A_ERR_UNSUPPORTED, "head_dim %d", head_dim);
  if (n_kv_heads < 1 || n_heads % n_kv_heads) return fail(W4A_ERR_SHAPE, "heads %d / kv heads %d", n_heads, n_kv_heads);
  if (batch < 1 || seq < 0 || seq >= batch || T < 1 || start_pos < 0)
    return fail(W4A_ERR_SHAPE, "batch %d seq %d T %d start %d", batch, seq, T, start_pos);
  if (window == 0) {
    if ((long long)start_pos + T > slots) return fail(W4A_ERR_SHAPE, "positions beyond the %d slots", slots);
  } else if (window != slots || window % 64) {
    return fail(W4A_ERR_SHAPE, "window must equal slots and be a multiple of 64");
  }
  if (slots < 16 || slots % 16) return fail(W4A_ERR_SHAPE, "slots %d (multiple of 16)", slots);
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(q) || !aligned16(out) || !aligned16(ws) ||
      !aligned16(k_new) || !aligned16(v_new))
    return fail(W4A_ERR_ALIGN, "misaligned pointer");
  if (ws_bytes < 256) return fail(W4A_ERR_WORKSPACE, "workspace %zu < 256 bytes", ws_bytes);
  uint32_t* err = static_cast<uint32_t*>(ws) + 2;
  CK(launch_flash_prefill(q, k_cache, v_cache, k_new, v_new, out, T, n_heads, n_kv_heads, head_dim, slots, window,
                          start_pos, seq, err, S(stream)));
  return W4A_OK;
}

int w4a_trace(void* buf, size_t bytes) {
  if (buf && !aligned16(buf)) return fail(W4A_ERR_ALIGN, "trace buffer not 16-byte aligned");
  g_trace = buf;
  g_trace_bytes = buf ? bytes : 0;
  return W4A_OK;
}

// ---- sampling ------------------------------------------------------------------------
int w4a_sample_workspace_bytes(int batch, int vocab, size_t* bytes) {
  if (!bytes) return fail(W4A_ERR_ARG, "null output");
  if (batch < 1 || vocab < 1) return fail(W4A_ERR_SHAPE, "batch %d vocab %d", batch, vocab);
  *bytes = (size_t)batch * vocab * sizeof(double);
  return W4A_OK;
}

int w4a_sample(const float* logits, int batch, int vocab, float temperature, float top_p, const float* u,
               int32_t* tokens, void* ws, size_t ws_bytes, void* stream) {
  if (!logits || !u || !tokens || !ws) return fail(W4A_ERR_ARG, "null pointer");
  if (batch < 1 || vocab < 1) return fail(W4A_ERR_SHAPE, "batch %d vocab %d", batch, vocab);
  if (!(temperature > 0.f) || !isfinite(temperature)) return fail(W4A_ERR_ARG, "temperature %g", temperature);
  if (!(top_p > 0.f && top_p <= 1.f)) return fail(W4A_ERR_ARG, "top_p %g", top_p);
  if (!aligned16(ws)) return fail(W4A_ERR_ALIGN, "workspace not 16-byte aligned");
  if (ws_bytes < (size_t)batch * vocab * sizeof(double))
    return fail(W4A_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, (size_t)batch * vocab * sizeof(double));
  CK(launch_sample(logits, batch, vocab, temperature, top_p, u, tokens, static_cast<double*>(ws), S(stream)));
  return W4A_OK;
}

int w4a_check(const void* ws, size_t ws_bytes, void* stream) {
  if (!ws) {
    // the fixed scratch of w4a_gemv_noalloc on the current device
    int dev = 0;
    CK(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return fail(W4A_ERR_UNSUPPORTED, "device index %d", dev);
    {
      std::lock_guard<std::mutex> lk(g_noalloc_mu);
      ws = g_noalloc_ptr[dev];
    }
    if (!ws) return fail(W4A_ERR_ARG, "no w4a_gemv_noalloc call on device %d yet", dev);
    ws_bytes = W4A_NOALLOC_SCRATCH_BYTES;
  }
  if (ws_bytes < 256) return fail(W4A_ERR_ARG, "short workspace");
  CK(cudaStreamSynchronize(S(stream)));
  uint32_t ctl[4];
  CK(cudaMemcpy(ctl, ws, sizeof(ctl), cudaMemcpyDeviceToHost));
  const uint32_t e = ctl[2];
  if (e & (EW_MBAR_TIMEOUT | EW_BARRIER_TIMEOUT | EW_DRAIN_TIMEOUT))
    return fail(W4A_ERR_TIMEOUT, "device wait timed out (error word 0x%x)", e);
  if (e & EW_RANGE)
    return fail(W4A_ERR_KERNEL, "an fp16 intermediate (SwiGLU or attention output) overflowed (error word 0x%x)", e);
  if (e) return fail(W4A_ERR_KERNEL, "device error word 0x%x", e);
  return W4A_OK;
}

}  // extern "C"
