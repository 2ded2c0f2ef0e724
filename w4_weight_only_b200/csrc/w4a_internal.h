// Internal definitions shared by the host entry points and the device engine.
// Not part of the public C ABI (see include/w4a.h).
#pragma once
#include <stddef.h>
#include <stdint.h>

#include "../../include/w4a.h"

namespace w4a {

// ---- engine geometry -------------------------------------------------------
constexpr int NW = 15;                 // math warps per CTA
constexpr int NT = NW * 32;            // threads of the math warps
constexpr int NTH = NT + 32;           // threads per CTA: the math warps and the copy warp
constexpr int ENGINE_REGS = 128;       // registers per thread (four warps per SM sub-partition)
static_assert(NTH * ENGINE_REGS <= 65536, "register file");
constexpr int NSLOT = 2;               // ring slots per warp
constexpr int SLOT_BYTES = 4352;       // one unit (>= the largest unit below)
constexpr int RB = 16;                 // output rows per unit (one m16 tile)
constexpr int W4_KC = 512;             // k per int4 unit
constexpr int BF_KC = 128;             // k per bf16 unit
constexpr int GROUP = 128;             // quantization group (the only one supported)
constexpr int W4_UNIT = RB * W4_KC / 2 + (W4_KC / GROUP) * RB * 2 + (W4_KC / GROUP) * RB / 2;  // 4256
constexpr int BF_UNIT = RB * BF_KC * 2;                                                      // 4096
// The model card's own checkpoint format: symmetric int4, group 32, bf16
// scales, stored nibble q + 8 (w = (nibble - 8) * s).  Its unit holds 16 rows
// x 256 columns: the codes in the same fragment order, then the 16 x 8 scales.
constexpr int S32_GROUP = 32;
constexpr int S32_KC = 256;
constexpr int S32_UNIT = RB * S32_KC / 2 + (S32_KC / S32_GROUP) * RB * 2;                    // 2304
constexpr int ATT_KEYS = 8;            // keys per warp unit
constexpr int ATT_CTA_KEYS = ATT_KEYS * NW;  // keys per CTA unit (120)
// Shared-memory budget per CTA (bytes).  x fragments shrink when two
// 8-column batch tiles are in use, to make room for their split-K slots.
__host__ __device__ constexpr int xs_cap(int nb) { return nb == 1 ? 58368 : 43008; }
constexpr int XSUM_BYTES = 6912;       // per-128-group sums of x: [groups][8 * NB]
__host__ __device__ constexpr int wsp_bytes(int nb) { return NW * 2 * 32 * 4 * nb * 4; }
constexpr int MAX_B = 16;
constexpr int MAX_LAYERS = 128;
constexpr int MAX_GQ = 8;              // query heads per KV head supported by the attention tile
// A GEMV phase whose K is split into more than RED_NS slabs (batch > 1) sums
// them itself: the last CTA to finish a row block adds the slabs in order, so
// the consuming phase reads one copy of the vector instead of ns.
constexpr int RED_NS = 4;
constexpr int MAX_RBC = 2048;          // row blocks with a counter (d <= 32,768)

static_assert(W4_UNIT == 4256, "int4 unit size");
static_assert(W4_UNIT <= SLOT_BYTES && BF_UNIT <= SLOT_BYTES && S32_UNIT <= SLOT_BYTES, "slot too small");
static_assert(S32_UNIT == 2304, "sym32 unit size");

// ---- device error word bits -----------------------------------------------
enum : uint32_t {
  EW_MBAR_TIMEOUT = 1u << 0,     // a ring slot never completed
  EW_BARRIER_TIMEOUT = 1u << 1,  // a grid barrier never completed
  EW_DRAIN_TIMEOUT = 1u << 2,    // in-flight copies did not land before exit
  EW_BAD_SHAPE = 1u << 3,        // device-side shape check failed
  EW_BAD_POS = 1u << 4,          // a position outside the cache
  EW_RANGE = 1u << 5,            // a value carried in fp16 (SwiGLU or attention output) overflowed
};

// ---- engine modes / phase kinds --------------------------------------------
enum Mode : int { MODE_DECODE = 0, MODE_GEMV = 1, MODE_ATTN = 2 };
// the GEMV kinds come first: "is a GEMV" is one unsigned comparison
enum PhaseKind : int { PK_GEMV_W4 = 0, PK_GEMV_BF16 = 1, PK_GEMV_S32 = 2, PK_ATTN = 3, PK_ARGMAX = 4, PK_REDUCE = 5 };
// int4 weight formats of a launch: asymmetric group 128 (fp16 scale, int4
// zero) or the symmetric group-32 checkpoint format (bf16 scale, zero 8)
enum W4Fmt : int { FMT_ASYM128 = 0, FMT_SYM32 = 1 };
__host__ __device__ constexpr int fmt_kc(int fmt) { return fmt == FMT_SYM32 ? S32_KC : W4_KC; }
__host__ __device__ constexpr int fmt_unit(int fmt) { return fmt == FMT_SYM32 ? S32_UNIT : W4_UNIT; }
enum XSrc : int { XS_BF16 = 0, XS_EMBED = 1, XS_RESID = 2, XS_FINAL = 3, XS_F16 = 4, XS_SILU = 5 };
enum Epi : int { EPI_Y = 0, EPI_Y_SUMSQ = 1, EPI_SILU = 2, EPI_PART = 3 };

// Geometry of a GEMV phase: 16-row blocks, k-chunks, k-chunks per slab,
// slabs, segments (= slabs x row blocks) and CTAs used.
struct Geo {
  int nrb, nkc, kps, ns, nseg, nca;
  // 1: the CTAs are split into ns groups, one per k-slab, so that no CTA's
  // segments span two slabs (it stages one slab of x)
  int aligned;
};

struct LayerPtrs {
  const uint8_t* qkv;
  const uint8_t* o;
  const uint8_t* gu;
  const uint8_t* down;
  const float* q_norm;
  const float* k_norm;
  const float* attn_norm;
  const float* ffn_norm;
};

// Workspace carve-up (device pointers), filled on the host.
struct Workspace {
  uint32_t* ctl;        // [0] barrier, [1] exit, [2] error word, [3] argmax counter
  uint32_t* seg_ctr;    // attention arrival counters [2][MAX_SEG]
  float* apart;         // attention pieces [NC][2][MAX_GQ * (HD + 2)]
  float* amax_val;      // argmax pieces [NC][B]
  int32_t* amax_idx;
  float* y_part;        // QKV output, per k-slab [ns][B][qkv_dim]
  uint16_t* o;          // attention output, fp16 [B][q_dim]
  float* a_part;        // O output [ns][B][d]
  float* gu_part;       // gate/up output when split [ns][B][2 ffn]
  uint16_t* h;          // SwiGLU output, fp16 [B][ffn]
  float* f_part;        // down output [ns][B][d]
  float* lg_part;       // lm_head output when split [ns][B][vocab]
  float* xA;            // residual at the layer input [B][d]
  float* xB;            // residual after attention [B][d]
  float* g_part;        // standalone GEMV output when split [ns][B][n]
  float* a_red;         // O output with its slabs summed by the producer [B][d] (many slabs), then the
                        // 16-row blocks' sums of squares [B][d / 16] (written above 8 rows)
  float* f_red;         // down output, the same layout
  uint32_t* rb_ctr;     // producer-side slab sums: arrivals per row block [2][MAX_RBC]
  void* plan;           // phase descriptors, one per phase of the launch
};

struct EngineParams {
  int mode;
  int phase_begin, phase_end;
  int nc;               // CTAs in the grid
  long long wait_bar;   // bound in cycles on waits for other CTAs (<= 0: the default, ~2 s)
  int fmt;              // W4Fmt of every int4 matrix of the launch
  // model dims
  int d, nq, nkv, hd, ffn, vocab, window, n_layers;
  float eps;
  int final_norm;
  double inv_freq[2][64];   // [0] sliding-window layers, [1] full layers
  float mscale[2];
  uint8_t full[MAX_LAYERS];
  // weights
  const uint16_t* embed;
  const uint8_t* lm_head;
  const float* final_gain;
  LayerPtrs layers[MAX_LAYERS];
  // KV cache
  uint8_t* kv_base;
  int kv_batch, max_ctx;
  uint64_t kv_off[MAX_LAYERS];   // byte offset of layer l's K region (V follows it)
  int kv_slots[MAX_LAYERS];
  // step inputs / outputs
  const int32_t* tokens;
  const int32_t* pos;
  int pos_const;        // >= 0: every sequence is at this position (prefill); else read pos[]
  int B, seq0;
  float* logits;
  int32_t* next_token;
  float* dump;
  Workspace ws;
  Geo geo[5];           // decode: qkv, o, gate/up, down, lm_head; GEMV: [0]
  // standalone GEMV
  const uint8_t* g_blob;
  const uint16_t* g_x;
  int g_n, g_k, g_epi;
  void* g_out;
  float* g_aux;
  // standalone attention
  const uint16_t* a_q;
  const uint16_t* a_k;
  const uint16_t* a_v;
  uint16_t* a_out;
  int a_slots, a_window;
  // optional trace: [phase][cta][4] %globaltimer stamps (start, prologue done, units done, arrived)
  uint64_t* trace;
  int trace_phases;
};

// Slots of a layer's ring / linear cache.
inline int64_t kv_slots(int full, int window, int max_ctx) { return full ? max_ctx : window; }

}  // namespace w4a
