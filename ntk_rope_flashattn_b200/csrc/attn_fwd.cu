// attn_fwd.cu -- fused RoPE + blockwise online-softmax causal attention prefill
// on sm_100a tensor cores (lcx_attn_fwd).
//
// What it computes ("Long Context: RoPE / YaRN / NTK / MLA", section 2.4
// rope_attention with the masks of 10.1/10.2 and the YaRN scale of 6.3-6.4):
//   o_i = sum_j softmax_j(c <q'_i, k'_j>) v_j over visible keys j,
// q', k' the rotated vectors (times mscale).  The blockwise evaluation with a
// running max and sum is the exact online softmax of "8.3 长上下文技术",
// section 8.3.4.
//
// Design (one CTA per work unit, 14 warps):
//   unit      = (batch b, two query heads of one GQA group, 128 query rows);
//               both query tiles read the same K/V tiles, so each K tile is
//               loaded and rotated once for 256 query rows.
//   warp 12   TMA producer: Q tiles once, then K tiles into a ring of stages;
//   warp 14   TMA producer of the V tiles (a V stage that frees late never
//             holds back the next K tile).
//   warps 8-11 rotation warpgroup: rotates the Q tiles and every K tile in
//               shared memory (bf16 -> fp32 -> rotate -> bf16) right after the
//               TMA lands, then hands the tile to the tensor core.
//   warp 13   MMA issuer: S_t = Q_t K^T (tcgen05.mma, fp32 accumulators in
//               TMEM), then O_t += P_t V with P_t read from TMEM.  The two
//               query tiles ping-pong so one tile's softmax overlaps the other
//               tile's matrix products.
//   warps 0-3 / 4-7  softmax for query tile 0 / 1: one thread per query row
//               reads its S row from TMEM, masks partial tiles, keeps the
//               running max/sum, writes P (bf16) back over S, rescales its O
//               row only when the max grew by more than 2^15, and finally
//               normalises O and stores it.
// Positions: query row i sits at q_offset + i and key j at j, so one kernel
// serves prefill (q_offset 0, Lk = L), chunked prefill and decode (the new
// queries against the whole key cache), and a StreamingLLM cache whose
// un-rotated keys are re-rotated at their cache index on every call.
// Tiles entirely hidden by the causal/window mask are never visited; tiles
// entirely visible skip the per-element mask.  Every barrier wait is bounded
// (wall-clock timeout); on expiry the CTA winds down, releases TMEM and
// reports LCX_ERR_TIMEOUT through the optional status word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstring>

#include "lcx_internal.h"
#include "rope_angle.cuh"
#include "sm100.cuh"

namespace lcx {
namespace {

constexpr int kThreads = 512;           // 16 warps = 4 warpgroups
// Registers per thread after the warpgroups re-balance (launch: 128 each;
// 176 + 176 + 96 + 64 = 4 x 128, so the file is exactly used).
constexpr int kRegsSoftmax = 176;       // warpgroups 0, 1: a whole S row in registers
constexpr int kRegsRotate = 96;         // warpgroup 2
constexpr int kRegsIssue = 64;          // warpgroup 3: TMA and MMA issuing warps
static_assert(2 * kRegsSoftmax + kRegsRotate + kRegsIssue == 4 * 128, "register file split");
constexpr int kBM = 128;                // query rows per tile
// Rescale O only if the row max grew by more than 2^15: until then the weights
// stay <= 2^15, inside the range of every P format used (bf16, fp16, tf32), and
// O and l stay far from fp32's.  (At 2^8, outlier-heavy inputs had a rescale
// in 53% of a warp's key tiles, N(0,1) inputs in 5%; at 2^15 36% and ~0%.)
constexpr float kRescaleLog2 = 15.0f;
// Build-time switches (-D...; the defaults are the measured-fastest choices):
//   LCX_EMU_EVERY       1 column pair in N takes 2^x on the FMA pipe (0: none)
//   LCX_D192_TWO_TILES  two query tiles and one K stage at D = 192 (0: one tile)
//   LCX_KSTAGES_D128    K ring depth at D = 128 without split QK^T (key-split launches: 3)
//   LCX_ROT_UNROLL      rows in flight per rotation thread
//   LCX_PHASOR_CARRY    reuse the phasor a K tile ends with for the next tile
#ifndef LCX_EMU_EVERY
#define LCX_EMU_EVERY 0
#endif
#ifndef LCX_D192_TWO_TILES
#define LCX_D192_TWO_TILES 1
#endif
#ifndef LCX_KSTAGES_D128
#define LCX_KSTAGES_D128 2
#endif
#ifndef LCX_ROT_UNROLL
#define LCX_ROT_UNROLL 2
#endif
// LCX_SPLIT_P_F16: the split mode's PV takes P and V in fp16 (V converted once
// by the rotate pass, or in shared memory by softmax warps 4-7 when keys are
// rotated on chip) rather than bf16
#ifndef LCX_SPLIT_P_F16
#define LCX_SPLIT_P_F16 1
#endif
#ifndef LCX_PHASOR_CARRY
#define LCX_PHASOR_CARRY 1
#endif
constexpr int kRotUnroll = LCX_ROT_UNROLL;  // rows in flight per rotation thread
// 1 column pair in kEmuEvery takes 2^x on the FMA pipe (0 = all on the MUFU:
// measured fastest here, since the MUFU is not the binding limit).
constexpr int kEmuEvery = LCX_EMU_EVERY;
constexpr int kWarpMma = 13;
constexpr int kWarpTma = 12;    // Q and K tiles
constexpr int kWarpTmaV = 14;   // V tiles
constexpr int kWarpRot0 = 8;

struct AttnParams {
    const char *q, *k, *v;             // raw pointers (fp32 operands path)
    char *o;
    float *lse;
    int *status;
    long long qs[3], ks[3], vs[3], os[3];  // element strides of B, H, L
    int B, Hq, Hkv, L, G;              // L: query rows
    int Lk, qoff;                      // key rows; position of query row 0
    int causal, window, sinks;
    int n_qb, heads_per_unit, units_per_qb;
    int qpair;                         // unit = two consecutive 128-row query blocks of one
                                       // head (odd G); n_qb then counts 256-row blocks
    int rotate_q, rotate_k;
    int n_split;                       // key-range splits per unit (1: plain output)
    int pack_lp, pack_hpt;             // head-packed query tiles (split-KV only): rows
    int pack_stride, pack_off;         // head k of tile t starts at row k stride + t off;
                                       // per head (multiple of 8), heads per tile; 0 = off
    int pack_ilv;                      // packed: both tiles hold all heads of the group, tile t
                                       // takes key tiles j = t mod 2, partial 2 split + t
    float split_recip;                 // 1 / n_split, rounded up
    float *part_o;                     // n_split > 1: [n_split, B, Hq, L, D] partial o
    float *part_lse;                   //              [n_split, B, Hq, L] partial lse
    int test_stall;                    // loader issues nothing (watchdog test hook)
    int rot_help;                      // head-packed split-KV with keys rotated on chip: the
                                       // softmax warps (bit w = warp w; 0 or 4 of them) whose
                                       // rows hold no query and that rotate key tiles with
                                       // warps 8-11
    int k_rope_shared;                 // rotated key columns come from one shared head
    int k_x8_tma;                      // split mode: the keys' 8-bit cross parts arrive by TMA
    int v_f16;                         // split mode: V arrives in fp16 (converted by a pass)
    int persist;                       // split mode: each CTA takes units blockIdx.x + k gridDim.x
    int n_units;                       //   of the n_units, one after the other
    float rot_ms;                      // factor on rotated values (partial rotary: mscale)
    float c_log2;                      // logit scale in log2 units
    unsigned long long timeout_ns;
    float theta[64];
};

// Shared-memory plan.  A tile of R rows x D 16-bit values is stored as D/64 TMA
// boxes of R rows x 128 bytes with the 128-byte swizzle.  D is the query/key
// head dim, DV the value/output head dim; at D = 192 (decoupled RoPE: 128 + 64)
// two query tiles (96 KB) leave room for one K stage (48 KB) and two V stages
// (32 KB each).  The K stage is released as soon as both S products of key
// tile j are done, so key tile j + 1 lands while the softmax of j runs; the
// second V stage lets V(j + 1) land while PV(j) still reads V(j).  That beats
// two K stages with one V stage (1038 vs 942 TFLOP/s on a 16-head L 16384
// prefill).
//
// Split QK^T mode: every rotated value x' is held as an fp16 part h = f16(x')
// and the rounding residual r = x' - h, and
//   S = Qh Kh^T + [e5m2(Qh) | e5m2(Qr)] [e5m2(Kr) | e5m2(Kh)]^T,
// one fp16 product (kind::f16) plus one e5m2 product over K = 2D
// (kind::f8f6f4: at M = N = 128 each instruction takes the same ~64 cycles as
// an fp16 one, so the cross product costs one more fp16 product).  The cross
// terms h r' are ~2^-11 of S, so their 3-bit e5m2 operands still leave the
// logits accurate to about 2^-15 relative; only the product of the two
// residuals (~2^-22) is dropped.  Each Q and K tile then has a second part,
// the 8-bit cross operand: 2D bytes per row, the size of a 16-bit part, stored
// as D/64 boxes of 128-byte rows ([h8 | r8] for a query row, [r8 | h8] for a
// key row).  One query tile per CTA, whose parts are TMEM A operands (their
// shared-memory staging is the last K stage); two K stages (64 KB each at
// D = 128) and three V stages of fp16.
//
// tf32 operands (fp32 inputs at D = 64): Q, K and V tiles hold fp32 values
// rounded to tf32, 32 per 128-byte row of a box (2 boxes per row at D = 64);
// P is written to TMEM as fp32 over the whole S buffer.  Two K and two V
// stages of 32 KB beside two 32 KB query tiles.
template <int D, int DV, bool kSplit, bool kTF = false, bool kKv = false>
struct Cfg {
    static constexpr int BN = 128;                      // keys per tile
    static constexpr int ES = kTF ? 4 : 2;              // bytes per operand element
    static constexpr int kParts = kSplit ? 2 : 1;       // 16-bit part (+ 8-bit cross part)
    // query tiles per CTA: two that ping-pong on the tensor core, or (split
    // mode, and D = 192 without LCX_D192_TWO_TILES) one
    static constexpr int kNTQ = (kSplit || (D > 128 && !LCX_D192_TWO_TILES)) ? 1 : 2;
    // S buffers per query tile: the single split-mode tile keeps two, so S(j + 2)
    // is computed while the softmax works on key tile j
    static constexpr int kNB = kSplit ? 2 : 1;
    static constexpr int kTileQ = kBM * D * ES;         // one part of a Q tile
    static constexpr int kTileK = BN * D * ES;          // one part of a K tile
    static constexpr int kTileV = BN * DV * ES;         // a V tile
    static constexpr int kBoxQ = kBM * 128;
    static constexpr int kBoxK = BN * 128;
    static constexpr int kKSteps = D * ES / 32;         // QK^T instructions over D (32 bytes each)
    static constexpr int kStagesK = kSplit ? (D == 64 ? 3 : 2)
                                  : kTF ? 2
                                  : (D == 64) ? 4
                                  : (D == 128) ? (kKv ? 3 : LCX_KSTAGES_D128)
                                  : (kNTQ == 2) ? 1 : 2;
    static constexpr int kStagesV = kSplit ? 3 : kTF ? 2 : (D == 64) ? 4 : 2;
    // Split mode: the query tile's two parts are the A operands of QK^T from
    // TMEM, so its shared-memory copy is only a staging area for the rotation
    // and the last K stage reuses it once the parts have moved to TMEM.
    static constexpr bool kQT = kSplit;
    static constexpr int kOffK = kQT ? 0 : kNTQ * kParts * kTileQ;
    static constexpr int kOffQ = kQT ? kOffK + (kStagesK - 1) * kParts * kTileK : 0;
    static constexpr int kOffV = kOffK + kStagesK * kParts * kTileK;
    static constexpr int kOffBar = kOffV + kStagesV * kTileV;
    static constexpr int kSmemBytes = kOffBar + 1024 + 1024;  // barriers + alignment slack
    // TMEM columns: S_t,b at (t kNB + b) BN (P_t,b aliased over its first BN/2
    // columns, or all of it with tf32), then O_t, then (split mode) the query
    // tile's fp16 part (D/2 columns, two values each) and its 8-bit cross part
    // (D/2 columns, four bytes each).
    // With as many K stages as S buffers, the completion of S(j) (s_ready of
    // buffer j mod kNB) is also the release of K stage j mod kStagesK.
    static constexpr bool kKFreeOnS = kNB > 1 && kStagesK == kNB;
    static constexpr int kColO = kNTQ * kNB * BN;
    static constexpr int kColQ = kColO + kNTQ * DV;
    static_assert(!kQT || (kNTQ == 1 && kTileQ == kTileK), "query staging in a K stage");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(kColQ + (kQT ? D : 0) <= 512, "TMEM budget");
};

template <int NSK, int NSV>
struct Bars {
    uint64_t full_q, ready_q;
    uint64_t full_k[NSK], ready_k[NSK], empty_k[NSK];
    uint64_t full_v[NSV], empty_v[NSV], fp16_v[NSV];
    uint64_t s_ready[2][2], p_ready[2][2], o_ready[2];
    uint64_t o_free;   // persistent split mode: the epilogue has read O
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

// ---------------------------------------------------------------- schedule
struct Unit {
    int b, g, hq0, nt, q0, split;
    int hpt;  // heads per query tile: 1, or pack_hpt when the tiles are head-packed
    // query tile t holds head hq0 + t hstep, rows q0 + t qstep (+ the row)
    int hstep, qstep;
    __device__ __forceinline__ int tq0(int t) const { return q0 + t * qstep; }
    __device__ __forceinline__ int th(int t) const { return hq0 + t * hstep; }
};

// Work units are grouped by (batch, kv head) and, inside a group, numbered
// heaviest first (query blocks from the end of the sequence, which see the
// most keys).  The block scheduler therefore runs many query blocks of the same
// kv head side by side -- they stream the same K/V tiles, which L2 then serves
// -- and still hands out the longest units of every group first.  With key
// splits (kKvSplit), the n_split CTAs of a unit are consecutive.
template <bool kKvSplit>
__device__ __forceinline__ Unit decode_unit(const AttnParams &p, int unit = -1) {
    const int u = unit >= 0 ? unit : kKvSplit ? int(blockIdx.x) / p.n_split : int(blockIdx.x);
    const int upq = p.G / p.heads_per_unit;          // units per query block of a group
    const int per_group = p.n_qb * upq;
    const int grp = u / per_group, rem = u % per_group;
    Unit r;
    r.b = grp / p.Hkv;
    r.g = grp % p.Hkv;
    const int rows = p.qpair ? 2 * kBM : kBM;   // query rows of a unit
    r.q0 = (p.n_qb - 1 - rem / upq) * rows;
    r.hq0 = r.g * p.G + p.heads_per_unit * (rem % upq);
    r.split = kKvSplit ? int(blockIdx.x) % p.n_split : 0;
    // Head-packed (split-KV decode): one unit per kv group, its heads spread over
    // the two query tiles.
    r.hpt = (kKvSplit && p.pack_lp) ? p.pack_hpt : 1;
    r.nt = (kKvSplit && p.pack_lp && p.pack_ilv) ? 2 : p.heads_per_unit / r.hpt;
    r.hstep = 1;
    r.qstep = 0;
    if (p.qpair) {
        // odd G: the two tiles are consecutive query blocks of head hq0 (one,
        // when the second would start past the last query)
        r.hstep = 0;
        r.qstep = kBM;
        r.nt = (r.q0 + kBM < p.L) ? 2 : 1;
    }
    return r;
}

// K tiles a query block visits: the sink tiles [0, ns) then the window tiles
// [jlo, jhi]; every listed tile has at least one visible key.  Query row i sits
// at position qoff + i, key j at position j.
// A key split takes the consecutive stretch [j0, j0 + n) of that list.
struct Tiles {
    int ns, jlo, n, j0;
    __device__ __forceinline__ int tile(int j) const {
        const int x = j + j0;
        return x < ns ? x : jlo + (x - ns);
    }
};

template <int BN, bool kKvSplit>
__device__ __forceinline__ Tiles make_tiles(int q0, int split, const AttnParams &p) {
    const int rows = p.qpair ? 2 * kBM : kBM;   // the unit's query rows from q0
    const int i1 = min(q0 + rows - 1, p.L - 1) + p.qoff;
    const int jhi = p.causal ? i1 / BN : (p.Lk - 1) / BN;
    int jlo = 0, ns = 0;
    if (p.causal && p.window > 0) {
        jlo = max(0, q0 + p.qoff - p.window + 1) / BN;
        if (p.sinks > 0) ns = min((p.sinks + BN - 1) / BN, jlo);
    }
    Tiles t;
    t.ns = ns;
    t.jlo = jlo;
    t.n = ns + (jhi - jlo + 1);
    t.j0 = 0;
    if constexpr (kKvSplit) {
        // split s of S takes tiles [s c, min(n, (s + 1) c)) with c >= n / S
        // (c = n / S rounded up in fp32, never below the exact quotient for
        // n < 2^24); the last splits may be empty.
        const int per = int(ceilf(float(t.n) * p.split_recip));
        const int jb = min(t.n, split * per);
        t.j0 = jb;
        t.n = min(t.n, jb + per) - jb;
    }
    return t;
}

// True when every (query row of the block, key of the tile) pair is visible.
template <int BN>
__device__ __forceinline__ bool tile_full(int q0, int jt, const AttnParams &p) {
    const int j0 = jt * BN, j1 = j0 + BN - 1;
    const int i0 = q0 + p.qoff, i1 = i0 + kBM - 1;
    if (j1 > p.Lk - 1) return false;
    if (!p.causal) return true;
    if (j1 > i0) return false;
    if (p.window > 0 && !(j0 >= i1 - p.window + 1 || j1 < p.sinks)) return false;
    return true;
}

// ---------------------------------------------------------------- smem tiles
// Byte offset of the 16-byte chunk fc (8 bf16 columns) of row r in a tile whose
// boxes are box_bytes long: the chunk c of row r sits at chunk c ^ (r & 7).
__device__ __forceinline__ uint32_t chunk_off(int r, int fc, int box_bytes) {
    return (fc >> 3) * box_bytes + r * 128 + (((fc & 7) ^ (r & 7)) << 4);
}

// The rotation's work split among NT threads (the rotation warpgroup's 128, or
// 256 when idle softmax warps of a decode launch help with the key tiles).
template <int D, bool kHalf, int NT = 128>
struct Rot {
    static constexpr int CPR = kHalf ? D / 16 : D / 8;  // jobs per row
    static constexpr int RP = NT / CPR;                  // rows per pass of the NT threads
    static constexpr int PPJ = kHalf ? 8 : 4;            // pairs per job
    static_assert(NT % CPR == 0 && 128 % RP == 0, "rotation work split");
};

// Rotate one job's pairs, two pairs per packed instruction: x1/x2 are the pair
// members, (c, s) the phasor: x1' = x1 c - x2 s, x2' = x1 s + x2 c.
template <int N>
__device__ __forceinline__ void rot_pairs(float (&x1)[N], float (&x2)[N], const float *c,
                                          const float *s) {
#pragma unroll
    for (int e = 0; e < N; e += 2) {
        const float2 a = make_float2(x1[e], x1[e + 1]), b = make_float2(x2[e], x2[e + 1]);
        const float2 cc = make_float2(c[e], c[e + 1]), ss = make_float2(s[e], s[e + 1]);
        const float2 nss = make_float2(-s[e], -s[e + 1]);
        const float2 y1 = fma2(b, nss, mul2(a, cc));
        const float2 y2 = fma2(a, ss, mul2(b, cc));
        x1[e] = y1.x;
        x1[e + 1] = y1.y;
        x2[e] = y2.x;
        x2[e + 1] = y2.y;
    }
}

__device__ __forceinline__ void unpack8(const uint4 &v, float (&x)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        x[2 * k] = bf16lo_to_f32(w[k]);
        x[2 * k + 1] = bf16hi_to_f32(w[k]);
    }
}
__device__ __forceinline__ uint4 pack8(const float (&y)[8]) {
    return make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]),
                      pack_bf16x2(y[4], y[5]), pack_bf16x2(y[6], y[7]));
}
// Byte offset of byte x of row r in a tile of 128-byte swizzled rows whose
// boxes are box_bytes long (x < 128 per box: box x / 128, 16-byte chunk x / 16
// of that box's row at chunk (x / 16) ^ (r & 7)).
__device__ __forceinline__ uint32_t byte_off(int r, int x, int box_bytes) {
    return (x >> 7) * box_bytes + r * 128 + ((((x >> 4) & 7) ^ (r & 7)) << 4) + (x & 15);
}

// Store the 8 rotated values of 16-byte chunk fc (columns 8 fc .. 8 fc + 7) of
// row r.  Plain mode: bf16 into the tile.  Split mode: the fp16 part h into the
// tile and, into the 8-bit cross part x8, e5m2(h) and e5m2(x' - h): a query row
// holds [h8 | r8] (column c at bytes c and D + c), a key row [r8 | h8].
template <bool kSplit, bool kKey, int D, int BOX, bool kTF = false>
__device__ __forceinline__ void store8(uint8_t *tile, uint8_t *x8, int r, int fc,
                                       const float (&y)[8]) {
    if constexpr (kTF) {
        // tf32 tile: the 8 values are two 16-byte chunks (columns 8 fc ..)
        *reinterpret_cast<float4 *>(tile + chunk_off(r, 2 * fc, BOX)) =
            make_float4(round_tf32(y[0]), round_tf32(y[1]), round_tf32(y[2]), round_tf32(y[3]));
        *reinterpret_cast<float4 *>(tile + chunk_off(r, 2 * fc + 1, BOX)) =
            make_float4(round_tf32(y[4]), round_tf32(y[5]), round_tf32(y[6]), round_tf32(y[7]));
        return;
    }
    const uint32_t off = chunk_off(r, fc, BOX);
    if constexpr (!kSplit) {
        *reinterpret_cast<uint4 *>(tile + off) = pack8(y);
    } else {
        const uint4 h = make_uint4(pack_f16x2(y[0], y[1]), pack_f16x2(y[2], y[3]),
                                   pack_f16x2(y[4], y[5]), pack_f16x2(y[6], y[7]));
        *reinterpret_cast<uint4 *>(tile + off) = h;
        const uint32_t hw[4] = {h.x, h.y, h.z, h.w};
        float hf[8], rr[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = f16x2_to_f32x2(hw[k]);
            hf[2 * k] = f.x;
            hf[2 * k + 1] = f.y;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) rr[e] = y[e] - hf[e];   // exact in fp32
        const uint2 h8 = make_uint2(pack_e5m2x4(hf[0], hf[1], hf[2], hf[3]),
                                    pack_e5m2x4(hf[4], hf[5], hf[6], hf[7]));
        const uint2 r8 = make_uint2(pack_e5m2x4(rr[0], rr[1], rr[2], rr[3]),
                                    pack_e5m2x4(rr[4], rr[5], rr[6], rr[7]));
        const int c = 8 * fc;
        *reinterpret_cast<uint2 *>(x8 + byte_off(r, kKey ? D + c : c, BOX)) = h8;
        *reinterpret_cast<uint2 *>(x8 + byte_off(r, kKey ? c : D + c, BOX)) = r8;
    }
}

// Copy row r of a split-mode query tile into TMEM lane r (taddr: the lane's
// address at the first query column): the fp16 part (128-byte swizzled rows,
// D/64 boxes) to D/2 columns of two values, then the 8-bit cross part (2 D
// bytes, as many boxes) to D/2 columns of four bytes, both in K order with the
// lower index in the lower bits -- the A-operand layout of the TMEM form of the
// MMA, 32 bytes of K (8 columns) per instruction.
template <int D, int BOX>
__device__ __forceinline__ void q_parts_to_tmem(const uint8_t *hi, const uint8_t *x8, int r,
                                                uint32_t taddr) {
#pragma unroll 1
    for (int part = 0; part < 2; ++part) {
        const uint8_t *src = part ? x8 : hi;
#pragma unroll 1
        for (int g = 0; g < D / 64; ++g) {
            uint32_t u[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 w =
                    *reinterpret_cast<const uint4 *>(src + chunk_off(r, g * 8 + c, BOX));
                u[4 * c] = w.x;
                u[4 * c + 1] = w.y;
                u[4 * c + 2] = w.z;
                u[4 * c + 3] = w.w;
            }
            tmem_st32_nowait(taddr + part * (D / 2) + g * 32, u);
        }
    }
    tmem_wait_st();
}

// Per-thread phasor state of the rotation warpgroup: the thread always handles
// the same pairs i0..i0+PPJ-1 and rows r0 + RP k, so it starts each tile at
// e^{i (pos0 + r0) theta} and steps by e^{i RP theta}.
template <int D, bool kHalf, int NT = 128>
struct Phasor {
    using R = Rot<D, kHalf, NT>;
    float sc[R::PPJ], ss[R::PPJ];  // step
    int q, r0, i0;
    __device__ __forceinline__ void init(int tw, const AttnParams &p) {
        q = tw % R::CPR;
        r0 = tw / R::CPR;
        i0 = q * R::PPJ;
#pragma unroll
        for (int e = 0; e < R::PPJ; ++e) rope_sincos(R::RP, p.theta[i0 + e], &sc[e], &ss[e]);
    }
    // kScaled: multiply by p.rot_ms (partial rotary, where mscale is not folded
    // into the logit scale).
    template <bool kScaled = false>
    __device__ __forceinline__ void start(long long pos0, const AttnParams &p, float (&c)[R::PPJ],
                                          float (&s)[R::PPJ]) const {
#pragma unroll
        for (int e = 0; e < R::PPJ; ++e) {
            rope_sincos_fast(pos0 + r0, p.theta[i0 + e], &c[e], &s[e]);
            if constexpr (kScaled) {
                c[e] *= p.rot_ms;
                s[e] *= p.rot_ms;
            }
        }
    }
    __device__ __forceinline__ void step(float (&c)[R::PPJ], float (&s)[R::PPJ]) const {
#pragma unroll
        for (int e = 0; e < R::PPJ; e += 2) {
            const float2 cc = make_float2(c[e], c[e + 1]), s2 = make_float2(s[e], s[e + 1]);
            const float2 stc = make_float2(sc[e], sc[e + 1]), sts = make_float2(ss[e], ss[e + 1]);
            const float2 nsts = make_float2(-ss[e], -ss[e + 1]);
            const float2 nc = fma2(cc, stc, mul2(s2, nsts));
            const float2 ns = fma2(cc, sts, mul2(s2, stc));
            c[e] = nc.x;
            c[e + 1] = nc.y;
            s[e] = ns.x;
            s[e + 1] = ns.y;
        }
    }
};

// The phasor a rotation thread ends a K tile with already points at the first
// row of the next tile; consecutive tiles reuse it, and every kReseed tiles
// (or after a jump, e.g. from the sink tiles to the window) it is evaluated
// afresh from the exact angle, which bounds the drift of the recurrence.
template <int PPJ>
struct PhasorCarry {
    float c[PPJ], s[PPJ];
    long long next = -1;
    int age = 0;
};
constexpr int kReseed = 16;

// Rotate (or, with rotate = false, only copy into the split mode's parts) this
// thread's pairs of row r of a tile whose boxes are BOX bytes long; (c, s) the
// phasor.  Only the last RD of the D columns are rotated.
template <int D, int RD, bool kHalf, bool kSplit, bool kKey, int BOX>
__device__ __forceinline__ void rotate_row(uint8_t *tile, uint8_t *x8, int r, int q,
                                           const float *c, const float *s, bool rotate) {
    constexpr int C0 = (D - RD) / 8;  // first rotated 16-byte chunk of a row
    if (kHalf) {
        const int fa = C0 + q, fb = C0 + q + RD / 16;
        float x1[8], x2[8];
        unpack8(*reinterpret_cast<const uint4 *>(tile + chunk_off(r, fa, BOX)), x1);
        unpack8(*reinterpret_cast<const uint4 *>(tile + chunk_off(r, fb, BOX)), x2);
        if (rotate) rot_pairs<8>(x1, x2, c, s);
        store8<kSplit, kKey, D, BOX>(tile, x8, r, fa, x1);
        store8<kSplit, kKey, D, BOX>(tile, x8, r, fb, x2);
    } else {
        const int fa = C0 + q;
        float x[8];
        unpack8(*reinterpret_cast<const uint4 *>(tile + chunk_off(r, fa, BOX)), x);
        if (rotate) {
            float x1[4], x2[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                x1[e] = x[2 * e];
                x2[e] = x[2 * e + 1];
            }
            rot_pairs<4>(x1, x2, c, s);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                x[2 * e] = x1[e];
                x[2 * e + 1] = x2[e];
            }
        }
        store8<kSplit, kKey, D, BOX>(tile, x8, r, fa, x);
    }
}

// A head-packed query tile (decode): row off + k stride + i holds query i
// (i < Lp) of the tile's k-th head (k < heads), at position pos0 + i; other
// rows hold no data.  Each row's phasor comes from its exact angle (once per
// CTA).
template <int D, int RD, bool kHalf, bool kSplit>
__device__ __forceinline__ void rotate_packed_q(uint8_t *tile, uint8_t *lo, long long pos0,
                                                int Lp, int stride, int off, int heads,
                                                const Phasor<RD, kHalf> &ph, const AttnParams &p,
                                                bool rotate) {
    using R = Rot<RD, kHalf>;
    constexpr int NJ = kBM / R::RP;
    for (int k = 0; k < NJ; ++k) {
        const int r = ph.r0 + k * R::RP;
        const int rel = r - off;
        if (rel < 0 || rel >= heads * stride || rel % stride >= Lp) continue;
        float c[R::PPJ], s[R::PPJ];
        if (rotate) ph.template start<(RD < D)>(pos0 + rel % stride - ph.r0, p, c, s);
        rotate_row<D, RD, kHalf, kSplit, false, kBM * 128>(tile, lo, r, ph.q, c, s, rotate);
    }
}

// Rotate a ROWS x D bf16 tile in place (row r at position pos0 + r); only its
// last RD columns are rotated (RD = D: all of them).  In the split mode the
// tile receives the fp16 parts and `lo` the 8-bit cross parts (kKey: the key
// order [r8 | h8]).
template <int D, int RD, bool kHalf, bool kSplit, bool kKey, int ROWS, int NT = 128>
__device__ __forceinline__ void rotate_tile_bf16(uint8_t *tile, uint8_t *lo, long long pos0,
                                                 const Phasor<RD, kHalf, NT> &ph,
                                                 const AttnParams &p, bool rotate,
                                                 PhasorCarry<Rot<RD, kHalf>::PPJ> *carry = nullptr) {
    using R = Rot<RD, kHalf, NT>;
    constexpr int NJ = ROWS / R::RP;
    constexpr int BOX = ROWS * 128;
    float c[R::PPJ], s[R::PPJ];
    if (rotate) {
        if (LCX_PHASOR_CARRY && carry && carry->next == pos0 && carry->age < kReseed) {
#pragma unroll
            for (int e = 0; e < R::PPJ; ++e) {
                c[e] = carry->c[e];
                s[e] = carry->s[e];
            }
            ++carry->age;
        } else {
            ph.template start<(RD < D)>(pos0, p, c, s);
            if (carry) carry->age = 0;
        }
    }
    // the split mode's stores take more registers: one row in flight
    constexpr int kUnroll = kSplit ? 1 : kRotUnroll;
#pragma unroll kUnroll
    for (int k = 0; k < NJ; ++k) {
        const int r = ph.r0 + k * R::RP;
        rotate_row<D, RD, kHalf, kSplit, kKey, BOX>(tile, lo, r, ph.q, c, s, rotate);
        if (rotate) ph.step(c, s);
    }
    if (LCX_PHASOR_CARRY && carry && rotate) {
#pragma unroll
        for (int e = 0; e < R::PPJ; ++e) {
            carry->c[e] = c[e];
            carry->s[e] = s[e];
        }
        carry->next = pos0 + ROWS;
    }
}

// fp32 operands: load ROWS rows from global (rows >= L read as zero), rotate in
// fp32 when asked (row r at position pos0 + r), round to bf16 (split mode: the
// fp16 part, and the 8-bit cross part into `lo`; kTF: to tf32, kept in fp32)
// into the tile.
template <int D, bool kHalf, bool kSplit, bool kKey, int ROWS, bool kTF = false>
__device__ __forceinline__ void load_tile_f32(uint8_t *tile, uint8_t *lo, const float *base,
                                              long long rs, int row0, int L, long long pos0,
                                              bool rotate, const Phasor<D, kHalf> &ph,
                                              const AttnParams &p) {
    using R = Rot<D, kHalf>;
    constexpr int NJ = ROWS / R::RP;
    constexpr int BOX = ROWS * 128;
    float c[R::PPJ], s[R::PPJ];
    if (rotate) ph.start(pos0, p, c, s);
    for (int k = 0; k < NJ; ++k) {
        const int r = ph.r0 + k * R::RP;
        const bool valid = row0 + r < L;
        const float *src = base + (long long)(row0 + r) * rs;
        if (kHalf) {
            float x1[8], x2[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                x1[e] = valid ? src[ph.i0 + e] : 0.f;
                x2[e] = valid ? src[ph.i0 + e + D / 2] : 0.f;
            }
            if (rotate) rot_pairs<8>(x1, x2, c, s);
            store8<kSplit, kKey, D, BOX, kTF>(tile, lo, r, ph.q, x1);
            store8<kSplit, kKey, D, BOX, kTF>(tile, lo, r, ph.q + D / 16, x2);
        } else {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = valid ? src[8 * ph.q + e] : 0.f;
            if (rotate) {
                float x1[4], x2[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x1[e] = x[2 * e];
                    x2[e] = x[2 * e + 1];
                }
                rot_pairs<4>(x1, x2, c, s);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x[2 * e] = x1[e];
                    x[2 * e + 1] = x2[e];
                }
            }
            store8<kSplit, kKey, D, BOX, kTF>(tile, lo, r, ph.q, x);
        }
        if (rotate) ph.step(c, s);
    }
}

// A bf16 tile converted to fp16 in place (exact for |x| in fp16's normal range;
// smaller values keep fp16's subnormal spacing, 2^-24), 16 bytes per thread
// and step.
template <int BYTES>
__device__ __forceinline__ void bf16_tile_to_f16(uint8_t *tile, int tw) {
    for (int i = tw; i < BYTES / 16; i += 128) {
        uint4 *c = reinterpret_cast<uint4 *>(tile) + i;
        const uint4 x = *c;
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        uint32_t h[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) h[k] = pack_f16x2(bf16lo_to_f32(w[k]), bf16hi_to_f32(w[k]));
        *c = make_uint4(h[0], h[1], h[2], h[3]);
    }
}

// fp32 V tile: convert only (to bf16, with kF16 to fp16, or with kTF round to
// tf32).  The tf32
// tile is stored transposed, K-major for the PV product: row d (output dim)
// holds the ROWS keys' values, 32 keys per 128-byte row of a box of D rows
// (ROWS / 32 boxes), 16-byte chunks swizzled by d; each thread gathers four
// consecutive keys of one dim into one chunk.
template <int D, int ROWS, bool kTF = false, bool kF16 = false>
__device__ __forceinline__ void load_v_f32(uint8_t *tile, const float *base, long long rs, int row0,
                                           int L, int tw) {
    if constexpr (kTF) {
        constexpr int VBOX = D * 128;   // one box: D rows of 32 keys
        for (int idx = tw; idx < D * (ROWS / 4); idx += 128) {
            const int d = idx % D, g = idx / D;    // dim, group of 4 keys
            float x[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = 4 * g + e;
                x[e] = row0 + r < L ? round_tf32(base[(long long)(row0 + r) * rs + d]) : 0.f;
            }
            *reinterpret_cast<float4 *>(tile + (g >> 3) * VBOX + d * 128 +
                                        (((g & 7) ^ (d & 7)) << 4)) =
                make_float4(x[0], x[1], x[2], x[3]);
        }
        return;
    }
    constexpr int CPR = D / 8;
    constexpr int BOX = ROWS * 128;
    for (int idx = tw; idx < ROWS * CPR; idx += 128) {
        const int r = idx / CPR, fc = idx % CPR;
        const bool valid = row0 + r < L;
        const float *src = base + (long long)(row0 + r) * rs + fc * 8;
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = valid ? src[e] : 0.f;
        *reinterpret_cast<uint4 *>(tile + chunk_off(r, fc, BOX)) =
            kF16 ? make_uint4(pack_f16x2(x[0], x[1]), pack_f16x2(x[2], x[3]),
                              pack_f16x2(x[4], x[5]), pack_f16x2(x[6], x[7]))
                 : pack8(x);
    }
}


// Max of N values (N % 8 == 0) with four independent chains of 3-input max:
// v[0..3] start the chains, v[4 .. N-5] are taken 8 at a time, v[N-4 .. N-1]
// close them.
template <int N>
__device__ __forceinline__ float row_max(const float (&v)[N]) {
    static_assert(N % 8 == 0 && N >= 16, "row_max layout");
    float m0 = v[0], m1 = v[1], m2 = v[2], m3 = v[3];
#pragma unroll
    for (int e = 4; e + 8 <= N - 4; e += 8) {
        m0 = max3(m0, v[e], v[e + 1]);
        m1 = max3(m1, v[e + 2], v[e + 3]);
        m2 = max3(m2, v[e + 4], v[e + 5]);
        m3 = max3(m3, v[e + 6], v[e + 7]);
    }
    m0 = max3(m0, v[N - 4], v[N - 3]);
    m1 = max3(m1, v[N - 2], v[N - 1]);
    return fmaxf(max3(m0, m1, m2), m3);
}

// Store 32 output columns [c*32, c*32+32) of query row i of head h, scaled by
// inv: fp32 into the partial buffer of the unit's key split when there is one,
// else rounded once to the output type.
template <int D, bool kF32, bool kKvSplit>
__device__ __forceinline__ void store_o32(const AttnParams &p, const Unit &U, int slot, int h,
                                          int i, int c, const float (&v)[32], float inv) {
    if constexpr (kKvSplit) {
        const long long prow = (((long long)slot * p.B + U.b) * p.Hq + h) * p.L + i;
        float4 *dst = reinterpret_cast<float4 *>(p.part_o + prow * D + c * 32);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(v[4 * e] * inv, v[4 * e + 1] * inv, v[4 * e + 2] * inv,
                                 v[4 * e + 3] * inv);
        return;
    }
    const long long ob = U.b * p.os[0] + (long long)h * p.os[1] + (long long)i * p.os[2] + c * 32;
    if (kF32) {
        float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.o) + ob);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(v[4 * e] * inv, v[4 * e + 1] * inv, v[4 * e + 2] * inv,
                                 v[4 * e + 3] * inv);
    } else {
        uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(p.o) + ob);
#pragma unroll
        for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pack_bf16x2(v[8 * e] * inv, v[8 * e + 1] * inv),
                                pack_bf16x2(v[8 * e + 2] * inv, v[8 * e + 3] * inv),
                                pack_bf16x2(v[8 * e + 4] * inv, v[8 * e + 5] * inv),
                                pack_bf16x2(v[8 * e + 6] * inv, v[8 * e + 7] * inv));
    }
}

// The row's log-sum-exp (natural log) into the partial buffer or the output.
template <bool kKvSplit>
__device__ __forceinline__ void store_lse(const AttnParams &p, const Unit &U, int slot, int h,
                                          int i, float lse) {
    if constexpr (kKvSplit)
        p.part_lse[(((long long)slot * p.B + U.b) * p.Hq + h) * p.L + i] = lse;
    else if (p.lse)
        p.lse[(U.b * (long long)p.Hq + h) * p.L + i] = lse;
}

// Query row `row` of tile t: its head, its query index and whether it holds a
// query.  Head-packed tiles: the tile's k-th head starts at row
// k stride + t off (stride >= Lp rows per head; tile 1 shifted by a warp when
// the room allows, so the few busy softmax warps of the two tiles sit on
// different SMSPs).
struct RowMap {
    int h, i;
    bool valid;
};
__device__ __forceinline__ RowMap map_row(const AttnParams &p, const Unit &U, int t, int row,
                                          bool packed) {
    RowMap m;
    if (packed) {
        const int rel = row - t * p.pack_off;
        const int k = rel >= 0 ? rel / p.pack_stride : U.hpt;
        m.i = rel - k * p.pack_stride;
        m.h = U.hq0 + (p.pack_ilv ? 0 : t * U.hpt) + k;
        m.valid = rel >= 0 && k < U.hpt && m.i < p.L;
    } else {
        m.h = U.th(t);
        m.i = U.tq0(t) + row;
        m.valid = m.i < p.L;
    }
    return m;
}

// Key tiles of a head-packed split-KV launch rotated by 256 threads: the
// rotation warpgroup (tw 0..127) and four softmax warps that hold no query
// (tw 128..255), each thread taking every 32nd row of its pairs.  The same
// stage protocol as the rotation warpgroup alone: wait for the TMA, rotate in
// place (split mode: into the fp16 and 8-bit cross parts), arrive on ready_k.
template <int D, int RD, bool kHalf, bool kSplit, int NSK, int BN, int kParts, int kTileK,
          typename Bar>
__device__ __forceinline__ void rotate_keys_helped(int tw, const Tiles &T, uint8_t *sK, Bar &bar,
                                                   const AttnParams &p, volatile int *abort,
                                                   uint64_t tmo) {
    Phasor<RD, kHalf, 256> ph;
    ph.init(tw, p);
    PhasorCarry<Rot<RD, kHalf>::PPJ> carry;
    for (int j = 0; j < T.n; ++j) {
        const int jt = T.tile(j), s = j % NSK;
        uint8_t *tk = sK + s * kParts * kTileK;
        if (!__all_sync(0xffffffffu, mbar_wait(&bar.full_k[s], (j / NSK) & 1, abort, tmo)))
            break;
        rotate_tile_bf16<D, RD, kHalf, kSplit, true, BN, 256>(tk, tk + kTileK, (long long)jt * BN,
                                                              ph, p, true, &carry);
        fence_proxy_async_smem();
        mbar_arrive(&bar.ready_k[s]);
    }
}

// ---------------------------------------------------------------- kernel
// D: query/key head dim, DV: value/output head dim, RD: rotated (last) dims;
// kKvSplit: this launch is one pass of split-KV (partial results per split).
template <int D, int DV, int RD, bool kF32, bool kHalf, bool kSplit, bool kKvSplit,
          bool kPersist = false>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmq,
                    const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv,
                    const __grid_constant__ CUtensorMap tmkr, const __grid_constant__ AttnParams p) {
    // fp32 operands at D = 64 stay 32-bit (rounded to tf32) for kind::tf32
    // products; at D = 128 two query tiles of them would not fit beside the
    // K/V stages, so they are rounded to bf16 like the split mode's values.
    constexpr bool kTF = kF32 && !kSplit && D == 64;
    // split mode: P and V in fp16 for PV (bf16 V tiles from the TMA are
    // converted in shared memory by the rotation warpgroup)
    constexpr bool kPF16 = kSplit && LCX_SPLIT_P_F16;
    constexpr bool kConvV = kPF16 && !kF32;
    using C = Cfg<D, DV, kSplit, kTF, kKvSplit>;
    static_assert(!kF32 || (RD == D && DV == D), "fp32 operands: full rotary, DV = D");
    static_assert(!kSplit || (RD == D && DV == D), "split QK^T: full rotary, DV = D");
    constexpr int NSK = C::kStagesK;
    constexpr int NSV = C::kStagesV;
    constexpr int BN = C::BN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // Q part x of tile t at sQ + (t * kParts + x) * kTileQ (split mode: staging
    // in the last K stage); K part x of stage s at
    // sK + (s * kParts + x) * kTileK; V stage s at sV + s * kTileK.
    uint8_t *sQ = smem + C::kOffQ;
    uint8_t *sK = smem + C::kOffK;
    uint8_t *sV = smem + C::kOffV;
    Bars<NSK, NSV> &bar = *reinterpret_cast<Bars<NSK, NSV> *>(smem + C::kOffBar);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const Unit U = decode_unit<kKvSplit>(p);
    const Tiles T = make_tiles<BN, kKvSplit>(U.q0, U.split, p);   // this CTA's key tiles
    const bool packed = kKvSplit && !kF32 && p.pack_lp > 0;       // head-packed query tiles
    volatile int *abort = &bar.abort;
    const uint64_t tmo = p.timeout_ns;

    if (threadIdx.x == 0) {
        mbar_init(&bar.full_q, 1);
        mbar_init(&bar.ready_q, 128);
        for (int s = 0; s < NSK; ++s) {
            mbar_init(&bar.full_k[s], 1);
            mbar_init(&bar.ready_k[s], 128 + 32 * __popc(p.rot_help));
            mbar_init(&bar.empty_k[s], 1);
        }
        for (int s = 0; s < NSV; ++s) {
            mbar_init(&bar.full_v[s], kF32 ? 128 : 1);
            mbar_init(&bar.fp16_v[s], 128);
            mbar_init(&bar.empty_v[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            for (int b = 0; b < 2; ++b) {
                mbar_init(&bar.s_ready[t][b], 1);
                // the tile's four softmax warps hand over P, except the ones
                // that help rotate keys; all eight in the split mode with fp16 V
                mbar_init(&bar.p_ready[t][b], (kSplit && !kKvSplit && p.v_f16)
                                                  ? 256
                                                  : 32 * (4 - __popc((p.rot_help >> (4 * t)) & 0xF)));
            }
            mbar_init(&bar.o_ready[t], 1);
        }
        mbar_init(&bar.drain, 1);
        mbar_init(&bar.o_free, 256);
        bar.abort = 0;
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(&bar.tmem_base, 512);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_base;
    // A CTA that starts after another one's watchdog fired gives up at its
    // first wait that does not complete at once: thread 0 reads the status
    // word here, after the barrier, so no role waits for that load to start.
    bool pre = false;   // thread 0: the word was already set
    if (threadIdx.x == 0 && p.status && *reinterpret_cast<volatile int *>(p.status) != 0) {
        pre = true;
        *abort = 1;
    }
    // key splits: the merge may be scheduled now (it waits for this grid to
    // finish before it reads the partial results)
    if constexpr (kKvSplit) pdl_launch_dependents();

    if (kKvSplit && T.n == 0) {
        // A key split that received no tile (more splits than tiles): the
        // empty partial result, o = 0 and lse = -inf.
        if (warp < 8 && (warp >> 2) < U.nt) {
            const int t = warp >> 2;
            const RowMap rm = map_row(p, U, t, (warp & 3) * 32 + lane, packed);
            if (rm.valid) {
                float z[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) z[e] = 0.f;
                const int slot = p.pack_ilv ? 2 * U.split + t : U.split;
                for (int c = 0; c < DV / 32; ++c)
                    store_o32<DV, kF32, kKvSplit>(p, U, slot, rm.h, rm.i, c, z, 0.f);
                store_lse<kKvSplit>(p, U, slot, rm.h, rm.i, -INFINITY);
            }
        }
    } else if ((warp >> 2) == 3) {
        // warpgroup 3: warps 12 and 14 issue the TMA copies (Q and K; V), warp 13
        // the MMAs
        setmaxnreg_dec<kRegsIssue>();
        if (warp == kWarpTma) {
            // ------------------------------------------------ TMA producer
            constexpr bool persistent = kPersist;
            if constexpr (kPersist) {
                static_assert(kSplit && !kKvSplit && C::kKFreeOnS, "persistent split mode");
                // Persistent split mode: per unit, the query tile into its staging
                // area (the last K stage) once the last key tile there has been
                // multiplied, then the unit's key tiles, stages counted across
                // units; the first key tile into the staging stage waits until the
                // query's parts have moved to TMEM.
                if (lane == 0) {
                    tma_prefetch_desc(&tmq);
                    tma_prefetch_desc(&tmk);
                    if (p.k_x8_tma) tma_prefetch_desc(&tmkr);
                    int issued_k[NSK] = {};
                    int nq = 0, g = 0;
                    bool ok = true;
                    for (int ku = 0; ok; ++ku) {
                        const int uu = int(blockIdx.x) + ku * int(gridDim.x);
                        if (uu >= p.n_units) break;
                        const Unit Uu = decode_unit<kKvSplit>(p, uu);
                        const Tiles Tu = make_tiles<BN, kKvSplit>(Uu.q0, Uu.split, p);
                        if (ku > 0) {
                            // the previous query tile has left the staging area (a
                            // unit whose key tiles all went to other stages never
                            // waited for that below) ...
                            ok = mbar_wait(&bar.ready_q, (ku - 1) & 1, abort, tmo);
                            // ... and the last key tile (index < g) in that stage
                            // has been multiplied
                            const int gl = (g - 1) - (((g - 1) - (NSK - 1)) % NSK + NSK) % NSK;
                            if (ok && gl >= 0)
                                ok = mbar_wait(&bar.s_ready[0][gl % C::kNB], (gl / C::kNB) & 1,
                                               abort, tmo);
                        }
                        if (!ok) break;
                        mbar_arrive_expect_tx(&bar.full_q, C::kTileQ);
                        for (int bx = 0; bx < D / 64; ++bx)
                            tma_load_4d(sQ + bx * C::kBoxQ, &tmq, &bar.full_q, bx * 64, Uu.tq0(0),
                                        Uu.th(0), Uu.b);
                        ++nq;
                        bool staged = true;
                        for (int j = 0; ok && j < Tu.n; ++j, ++g) {
                            const int jt = Tu.tile(j), sk = g % NSK, uk = g / NSK;
                            if (uk > 0) ok = mbar_wait(&bar.s_ready[0][sk], (uk - 1) & 1, abort, tmo);
                            if (ok && sk == NSK - 1 && staged) {
                                ok = mbar_wait(&bar.ready_q, ku & 1, abort, tmo);
                                staged = false;
                            }
                            if (!ok) break;
                            const bool x8 = p.k_x8_tma != 0;
                            uint8_t *st = sK + sk * C::kParts * C::kTileK;
                            mbar_arrive_expect_tx(&bar.full_k[sk], x8 ? 2 * C::kTileK : C::kTileK);
                            if (x8)
                                for (int bx = 0; bx < D / 64; ++bx)
                                    tma_load_4d(st + C::kTileK + bx * C::kBoxK, &tmkr, &bar.full_k[sk],
                                                bx * 128, jt * BN, Uu.g, Uu.b);
                            for (int bx = 0; bx < D / 64; ++bx)
                                tma_load_4d(st + bx * C::kBoxK, &tmk, &bar.full_k[sk], bx * 64,
                                            jt * BN, Uu.g, Uu.b);
                            ++issued_k[sk];
                        }
                    }
                    // never leave the CTA with copies in flight (bounded)
                    if (nq) mbar_wait(&bar.full_q, (nq - 1) & 1, nullptr, tmo);
                    for (int s = 0; s < NSK; ++s)
                        if (issued_k[s]) mbar_wait(&bar.full_k[s], (issued_k[s] - 1) & 1, nullptr, tmo);
                }
            }
            if (!persistent && !kF32 && lane == 0 && !p.test_stall) {
                tma_prefetch_desc(&tmq);
                tma_prefetch_desc(&tmk);
                tma_prefetch_desc(&tmv);
                if ((RD < D && p.k_rope_shared) || p.k_x8_tma) tma_prefetch_desc(&tmkr);
                // With a shared rotary key, the K boxes from column D - RD on
                // come from that tensor's single head.
                constexpr int kNopeBoxes = (D - RD) / 64;
                int issued_k[NSK] = {};
                if (packed) {
                    // each head's pack_lp rows at row k pack_lp of its tile (the Q
                    // map's box is pack_lp rows high; 8-row multiples keep the
                    // 128-byte swizzle phase of the full tile)
                    mbar_arrive_expect_tx(&bar.full_q,
                                          U.nt * U.hpt * (D / 64) * p.pack_lp * 128);
                    for (int t = 0; t < U.nt; ++t)
                        for (int k = 0; k < U.hpt; ++k)
                            for (int bx = 0; bx < D / 64; ++bx)
                                tma_load_4d(sQ + t * C::kParts * C::kTileQ + bx * C::kBoxQ +
                                                (k * p.pack_stride + t * p.pack_off) * 128,
                                            &tmq, &bar.full_q, bx * 64, 0,
                                            U.hq0 + (p.pack_ilv ? 0 : t * U.hpt) + k, U.b);
                } else {
                    mbar_arrive_expect_tx(&bar.full_q, U.nt * C::kTileQ);
                    for (int t = 0; t < U.nt; ++t)
                        for (int bx = 0; bx < D / 64; ++bx)
                            tma_load_4d(sQ + t * C::kParts * C::kTileQ + bx * C::kBoxQ, &tmq,
                                        &bar.full_q, bx * 64, U.tq0(t), U.th(t), U.b);
                }
                bool ok = true;
                for (int j = 0; ok && j < T.n; ++j) {
                    const int jt = T.tile(j);
                    const int sk = j % NSK, uk = j / NSK;
                    if (uk > 0)
                        ok = mbar_wait(C::kKFreeOnS ? &bar.s_ready[0][sk] : &bar.empty_k[sk],
                                       (uk - 1) & 1, abort, tmo);
                    // the last K stage is the query tile's staging area until its
                    // parts are in TMEM
                    if (C::kQT && j == NSK - 1) ok = ok && mbar_wait(&bar.ready_q, 0, abort, tmo);
                    if (!ok) break;
                    // split mode with keys split by the rotate pass: the fp16 parts
                    // come through tmk, the 8-bit cross parts (fourth tensor map,
                    // 2 D bytes per key, 128-byte boxes) into the stage's second part
                    const bool x8 = kSplit && p.k_x8_tma;
                    mbar_arrive_expect_tx(&bar.full_k[sk], x8 ? 2 * C::kTileK : C::kTileK);
                    if (x8)
                        for (int bx = 0; bx < D / 64; ++bx)
                            tma_load_4d(sK + sk * C::kParts * C::kTileK + C::kTileK +
                                            bx * C::kBoxK,
                                        &tmkr, &bar.full_k[sk], bx * 128, jt * BN, U.g, U.b);
                    for (int bx = 0; bx < D / 64; ++bx) {
                        uint8_t *dst = sK + sk * C::kParts * C::kTileK + bx * C::kBoxK;
                        if constexpr (RD < D) {
                            if (p.k_rope_shared && bx >= kNopeBoxes) {
                                tma_load_4d(dst, &tmkr, &bar.full_k[sk], (bx - kNopeBoxes) * 64,
                                            jt * BN, 0, U.b);
                                continue;
                            }
                        }
                        tma_load_4d(dst, &tmk, &bar.full_k[sk], bx * 64, jt * BN, U.g, U.b);
                    }
                    ++issued_k[sk];
                }
                // Never leave the CTA with copies in flight: wait (bounded, even
                // after an abort) for the last load issued to every buffer.
                mbar_wait(&bar.full_q, 0, nullptr, tmo);
                for (int s = 0; s < NSK; ++s)
                    if (issued_k[s]) mbar_wait(&bar.full_k[s], (issued_k[s] - 1) & 1, nullptr, tmo);
            }
        } else if (warp == kWarpTmaV) {
            // ------------------------------------------------ TMA producer of V
            // V tiles come from their own warp, so a V stage that frees late (one
            // V stage: after the last PV of the previous tile) never holds back the
            // next K tile behind it.
            constexpr bool persistent = kPersist;
            if constexpr (kPersist) {
                // persistent split mode: the units' V tiles, stages counted across units
                if (lane == 0) {
                    int issued_v[NSV] = {};
                    int g = 0;
                    bool ok = true;
                    for (int ku = 0; ok; ++ku) {
                        const int uu = int(blockIdx.x) + ku * int(gridDim.x);
                        if (uu >= p.n_units) break;
                        const Unit Uu = decode_unit<kKvSplit>(p, uu);
                        const Tiles Tu = make_tiles<BN, kKvSplit>(Uu.q0, Uu.split, p);
                        for (int j = 0; ok && j < Tu.n; ++j, ++g) {
                            const int jt = Tu.tile(j), sv = g % NSV, uv = g / NSV;
                            if (uv > 0) ok = mbar_wait(&bar.empty_v[sv], (uv - 1) & 1, abort, tmo);
                            if (!ok) break;
                            mbar_arrive_expect_tx(&bar.full_v[sv], C::kTileV);
                            for (int bx = 0; bx < DV / 64; ++bx)
                                tma_load_4d(sV + sv * C::kTileV + bx * C::kBoxK, &tmv, &bar.full_v[sv],
                                            bx * 64, jt * BN, Uu.g, Uu.b);
                            ++issued_v[sv];
                        }
                    }
                    for (int s = 0; s < NSV; ++s)
                        if (issued_v[s]) mbar_wait(&bar.full_v[s], (issued_v[s] - 1) & 1, nullptr, tmo);
                }
            }
            if (!persistent && !kF32 && lane == 0 && !p.test_stall) {
                int issued_v[NSV] = {};
                bool ok = true;
                for (int j = 0; ok && j < T.n; ++j) {
                    const int jt = T.tile(j);
                    const int sv = j % NSV, uv = j / NSV;
                    if (uv > 0) ok = mbar_wait(&bar.empty_v[sv], (uv - 1) & 1, abort, tmo);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&bar.full_v[sv], C::kTileV);
                    for (int bx = 0; bx < DV / 64; ++bx)
                        tma_load_4d(sV + sv * C::kTileV + bx * C::kBoxK, &tmv, &bar.full_v[sv],
                                    bx * 64, jt * BN, U.g, U.b);
                    ++issued_v[sv];
                }
                for (int s = 0; s < NSV; ++s)
                    if (issued_v[s]) mbar_wait(&bar.full_v[s], (issued_v[s] - 1) & 1, nullptr, tmo);
            }
        } else if (warp == kWarpMma) {
            // ------------------------------------------------ MMA issuer
            if (lane == 0) {
                // S: bf16 (plain) or fp16 (split: the Qh Kh^T product) operands;
                // the split mode's cross product takes e5m2 operands.
                constexpr uint32_t kIdS = kSplit ? idesc_f32acc(128, BN, kFmtF16, kFmtF16, 0, 0)
                                          : kTF ? idesc_f32acc(128, BN, kFmtTF32, kFmtTF32, 0, 0)
                                                : idesc_bf16_f32(128, BN, 0, 0);
                constexpr uint32_t kIdX8 = idesc_f32acc(128, BN, kFmtE5M2, kFmtE5M2, 0, 0);
                // PV: V MN-major (bf16 tiles as the TMA lands them), or K-major
                // (the tf32 tile, which the loader writes transposed)
                constexpr uint32_t kIdPV = kTF ? idesc_f32acc(128, DV, kFmtTF32, kFmtTF32, 0, 0)
                                          : kPF16 ? idesc_f32acc(128, DV, kFmtF16, kFmtF16, 0, 1)
                                                  : idesc_bf16_f32(128, DV, 0, 1);
                // V ready for PV: landed (TMA, or written by the fp32 loader), or
                // converted to fp16 by the rotation warpgroup
                uint64_t *vready = (kConvV && !p.v_f16) ? bar.fp16_v : bar.full_v;
                const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
                // S_t = Q_t K^T over D in steps of 16 (32 bytes inside a 128-byte
                // swizzle row, then the next 64-column box).  Descriptors of the
                // first K step; later steps only move the start address (in
                // 16-byte units, well inside the 14-bit field).
                // All descriptors share their upper word (1024-byte stride), so
                // the loops below carry only the lower words.
                const uint64_t dq0 = sdesc_sw128(q_addr, 16, 1024);
                const uint32_t dhi = uint32_t(dq0 >> 32);
                const uint32_t q_lo = uint32_t(dq0);
                const uint32_t k_lo = uint32_t(sdesc_sw128(k_addr, 16, 1024));
                const uint32_t v_lo = uint32_t(kTF ? sdesc_sw128(v_addr, 16, 1024)
                                                   : sdesc_sw128(v_addr, C::kBoxK, 1024));
                constexpr int NB = C::kNB;
                auto issue_s = [&](int t, int s, int b) {
                    const uint32_t ka = k_lo + ((s * C::kParts * C::kTileK) >> 4);
                    const uint32_t dst = tmem + (t * NB + b) * BN;
                    if constexpr (C::kQT) {
                        // Split mode, query parts in TMEM (8 columns = 32 bytes of
                        // K per instruction): the e5m2 cross product first, into a
                        // fresh accumulator, [h8 | r8]_q [r8 | h8]_k^T over K = 2 D,
                        // then the fp16 product on top of it.
                        const uint32_t qh = tmem + C::kColQ, qx = qh + D / 2;
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t ok_ = ((kk >> 2) * C::kBoxK + (kk & 3) * 32) >> 4;
                            mma_ts_w<1>(dst, qx + kk * 8, ka + (C::kTileK >> 4) + ok_, dhi, kIdX8,
                                        kk > 0);
                        }
#pragma unroll
                        for (int kk = 0; kk < C::kKSteps; ++kk) {
                            const uint32_t ok_ = ((kk >> 2) * C::kBoxK + (kk & 3) * 32) >> 4;
                            mma_ts_w<0>(dst, qh + kk * 8, ka + ok_, dhi, kIdS, 1);
                        }
                    } else {
                        const uint32_t qa = q_lo + ((t * C::kParts * C::kTileQ) >> 4);
#pragma unroll
                        for (int kk = 0; kk < C::kKSteps; ++kk) {
                            const uint32_t oq = ((kk >> 2) * C::kBoxQ + (kk & 3) * 32) >> 4;
                            const uint32_t ok_ = ((kk >> 2) * C::kBoxK + (kk & 3) * 32) >> 4;
                            mma_ss_w<kTF ? 2 : 0>(dst, qa + oq, ka + ok_, dhi, kIdS, kk > 0);
                        }
                    }
                };
                // O_t += P_t V: P from TMEM (BN/2 columns of bf16 pairs, or BN of
                // tf32); each instruction takes 32 bytes of keys per row of P (8
                // TMEM columns).  bf16 V is MN-major (as many 128-byte rows of V
                // per step); the tf32 tile is V^T, K-major (32 bytes of each row).
                auto issue_pv = [&](int t, int s, int b, bool acc) {
                    const uint32_t va = v_lo + ((s * C::kTileV) >> 4);
                    const uint32_t dst = tmem + C::kColO + t * DV;
                    const uint32_t pa = tmem + (t * NB + b) * BN;
                    constexpr int KS = 32 / C::ES;   // keys per instruction
#pragma unroll
                    for (int kk = 0; kk < BN / KS; ++kk) {
                        // K-major V^T (tf32): 32 keys per box row, four 8-key steps
                        // per box; MN-major V: KS rows of 128 bytes per step
                        const uint32_t ov = kTF ? ((((kk >> 2) * DV * 128) + (kk & 3) * 32) >> 4)
                                                : ((kk * KS * 128) >> 4);
                        mma_ts_w<kTF ? 2 : 0>(dst, pa + kk * 8, va + ov, dhi, kIdPV,
                                              (acc || kk > 0));
                    }
                };
                // S_t(j + 1) is issued after PV_t(j), into the buffer P_t(j)
                // occupied (MMAs of one thread execute in order): the order is
                // PV0(j), S0(j+1), PV1(j), S1(j+1), so one query tile's softmax
                // overlaps the other tile's products.
                // Keys already rotated (and, in the split mode, already in parts)
                // need no pass through the rotation warpgroup: the MMA waits for
                // the TMA itself.
                uint64_t *kready = (kF32 || (kSplit && !p.k_x8_tma) || p.rotate_k) ? bar.ready_k
                                                                                    : bar.full_k;
                bool ok = mbar_wait(&bar.ready_q, 0, abort, tmo);
                if (kKvSplit && p.pack_ilv) {
                    // Both query tiles hold the same queries and tile t takes the
                    // key tiles j = t mod 2, so two K/V tiles are in flight per
                    // CTA: S_t(j + 2) follows PV_t(j) into the buffer P_t(j) held.
                    for (int j = 0; ok && j < 2 && j < T.n; ++j) {
                        ok = mbar_wait(&kready[j % NSK], (j / NSK) & 1, abort, tmo);
                        tc_fence_after();
                        if (!ok) break;
                        issue_s(j, j % NSK, 0);
                        mma_commit(&bar.s_ready[j][0]);
                        mma_commit(&bar.empty_k[j % NSK]);
                    }
                    for (int j = 0; ok && j < T.n; ++j) {
                        const int t = j & 1, sv = j % NSV, jn = j + 2;
                        ok = mbar_wait(&vready[sv], (j / NSV) & 1, abort, tmo);
                        if (ok) ok = mbar_wait(&bar.p_ready[t][0], (j >> 1) & 1, abort, tmo);
                        tc_fence_after();
                        if (!ok) break;
                        issue_pv(t, sv, 0, j >= 2);
                        mma_commit(&bar.empty_v[sv]);
                        if (jn < T.n) {
                            const int sk = jn % NSK;
                            ok = mbar_wait(&kready[sk], (jn / NSK) & 1, abort, tmo);
                            tc_fence_after();
                            if (!ok) break;
                            issue_s(t, sk, 0);
                            mma_commit(&bar.s_ready[t][0]);
                            mma_commit(&bar.empty_k[sk]);
                        }
                    }
                } else if constexpr (NB == 1) {
                    if (T.n > 0) {
                        ok = ok && mbar_wait(&kready[0], 0, abort, tmo);
                        tc_fence_after();
                        if (ok) {
                            for (int t = 0; t < U.nt; ++t) {
                                issue_s(t, 0, 0);
                                mma_commit(&bar.s_ready[t][0]);
                            }
                            mma_commit(&bar.empty_k[0]);
                        }
                    }
                    for (int j = 0; ok && j < T.n; ++j) {
                        const int sv = j % NSV, jn = j + 1;
                        ok = mbar_wait(&vready[sv], (j / NSV) & 1, abort, tmo);
                        for (int t = 0; ok && t < U.nt; ++t) {
                            ok = mbar_wait(&bar.p_ready[t][0], j & 1, abort, tmo);
                            tc_fence_after();
                            if (!ok) break;
                            issue_pv(t, sv, 0, j > 0);
                            if (jn < T.n) {
                                const int sk = jn % NSK;
                                if (t == 0) {
                                    ok = mbar_wait(&kready[sk], (jn / NSK) & 1, abort, tmo);
                                    tc_fence_after();
                                    if (!ok) break;
                                }
                                issue_s(t, sk, 0);
                                mma_commit(&bar.s_ready[t][0]);
                            }
                        }
                        if (ok) {
                            mma_commit(&bar.empty_v[sv]);
                            if (jn < T.n) mma_commit(&bar.empty_k[jn % NSK]);
                        }
                    }
                } else {
                    // Two S buffers (the split mode's single query tile): S(j + 2)
                    // goes into the buffer P(j) held, right after PV(j), so the
                    // softmax of key tile j + 1 runs while PV(j) and S(j + 2) do.
                    // Every wait of iteration j comes before PV(j), so PV(j) and
                    // S(j + 2) reach the tensor core back to back.  PV(j)'s
                    // completion is signalled once, on its V stage's barrier (a
                    // softmax that rescales O waits there); with as many K stages
                    // as S buffers, S(j)'s completion also frees its K stage.
                    static_assert(C::kNTQ == 1, "one query tile with two S buffers");
                    // Persistent launches: the units of this CTA one after the
                    // other, S buffers, K and V stages counted across them (g);
                    // a later unit's first PV waits until the previous unit's
                    // epilogue has read O.
                    int g = 0;
                    for (int ku = 0; ok; ++ku) {
                        const int uu = int(blockIdx.x) + ku * int(gridDim.x);
                        if (kPersist ? uu >= p.n_units : ku > 0) break;
                        const Tiles Tu =
                            kPersist ? make_tiles<BN, kKvSplit>(decode_unit<kKvSplit>(p, uu).q0, 0, p)
                                     : T;
                        if (ku > 0) {
                            ok = mbar_wait(&bar.ready_q, ku & 1, abort, tmo);
                            tc_fence_after();
                            if (!ok) break;
                        }
                        for (int jj = 0; ok && jj < NB && jj < Tu.n; ++jj) {
                            const int gj = g + jj;
                            ok = mbar_wait(&kready[gj % NSK], (gj / NSK) & 1, abort, tmo);
                            tc_fence_after();
                            if (!ok) break;
                            issue_s(0, gj % NSK, gj % NB);
                            mma_commit(&bar.s_ready[0][gj % NB]);
                            if (!C::kKFreeOnS) mma_commit(&bar.empty_k[gj % NSK]);
                        }
                        for (int j = 0; ok && j < Tu.n; ++j) {
                            const int gj = g + j;
                            const int sv = gj % NSV, jn = gj + NB, b = gj % NB, sk = jn % NSK;
                            const bool more = j + NB < Tu.n;
                            // The three phases are polled together first: each test's
                            // result takes ~100 cycles to come back, so polling them
                            // one after the other would keep the tensor core waiting.
                            const bool kr = !more || mbar_try_wait(&kready[sk], (jn / NSK) & 1);
                            const bool all = kr & mbar_try_wait(&vready[sv], (gj / NSV) & 1) &
                                             mbar_try_wait(&bar.p_ready[0][b], (gj / NB) & 1);
                            if (!all) {
                                if (more) ok = mbar_wait(&kready[sk], (jn / NSK) & 1, abort, tmo);
                                if (ok) ok = mbar_wait(&vready[sv], (gj / NSV) & 1, abort, tmo);
                                if (ok) ok = mbar_wait(&bar.p_ready[0][b], (gj / NB) & 1, abort, tmo);
                            }
                            if (kPersist && ok && j == 0 && ku > 0)
                                ok = mbar_wait(&bar.o_free, (ku - 1) & 1, abort, tmo);
                            tc_fence_after();
                            if (!ok) break;
                            issue_pv(0, sv, b, j > 0);
                            mma_commit(&bar.empty_v[sv]);
                            if (more) {
                                issue_s(0, sk, b);
                                mma_commit(&bar.s_ready[0][b]);
                                if (!C::kKFreeOnS) mma_commit(&bar.empty_k[sk]);
                            }
                        }
                        if (ok) mma_commit(&bar.o_ready[0]);
                        g += Tu.n;
                    }
                }
                // (two S buffers: O ready is signalled per unit inside the loop)
                if (ok && NB == 1)
                    for (int t = 0; t < U.nt; ++t) mma_commit(&bar.o_ready[t]);
                // Drain: all issued MMAs complete before TMEM is released.
                mma_commit(&bar.drain);
                mbar_wait(&bar.drain, 0, nullptr, tmo);
            }
        }
    } else if ((warp >> 2) == 2) {
        setmaxnreg_dec<kRegsRotate>();
        // ------------------------------------------------ rotation warpgroup
        const int tw = threadIdx.x - kWarpRot0 * 32;
        const bool rotq = p.rotate_q != 0, rotk = p.rotate_k != 0;
        Phasor<RD, kHalf> ph;
        ph.init(tw, p);
        PhasorCarry<Rot<RD, kHalf>::PPJ> kcarry;
        bool ok = true;
        if constexpr (!kF32) {
            ok = __all_sync(0xffffffffu, mbar_wait(&bar.full_q, 0, abort, tmo));
            if (ok && (rotq || kSplit))
                for (int t = 0; t < U.nt; ++t) {
                    uint8_t *qt = sQ + t * C::kParts * C::kTileQ;
                    if (packed)
                        rotate_packed_q<D, RD, kHalf, kSplit>(qt, qt + C::kTileQ, p.qoff,
                                                              p.pack_lp, p.pack_stride,
                                                              t * p.pack_off, U.hpt, ph, p, rotq);
                    else
                        rotate_tile_bf16<D, RD, kHalf, kSplit, false, kBM>(
                            qt, qt + C::kTileQ, (long long)U.tq0(t) + p.qoff, ph, p, rotq);
                }
        } else {
            for (int t = 0; t < U.nt; ++t) {
                const float *base = reinterpret_cast<const float *>(p.q) + U.b * p.qs[0] +
                                    (long long)U.th(t) * p.qs[1];
                uint8_t *qt = sQ + t * C::kParts * C::kTileQ;
                load_tile_f32<D, kHalf, kSplit, false, kBM, kTF>(qt, qt + C::kTileQ, base,
                                                                 p.qs[2], U.tq0(t), p.L,
                                                                 (long long)U.tq0(t) + p.qoff,
                                                                 rotq, ph, p);
            }
        }
        if constexpr (C::kQT) {
            // the query tile's parts move to TMEM (A operands of QK^T); the
            // staging area then serves as the last K stage.  Each thread copies
            // one row, which other threads of the warpgroup rotated.
            named_bar_sync(1, 128);
            if (ok) {
                const uint8_t *qt = sQ;
                q_parts_to_tmem<D, C::kBoxQ>(qt, qt + C::kTileQ, tw,
                                             tmem + (uint32_t((warp & 3) * 32) << 16) + C::kColQ);
                tc_fence_before();
            }
            named_bar_sync(1, 128);   // every row copied before keys overwrite the area
        }
        if (ok) {
            fence_proxy_async_smem();
            mbar_arrive(&bar.ready_q);
        }
        if constexpr (kPersist) {
            // Persistent split mode: the query tile of every later unit of this
            // CTA, rotated into its parts in the staging area as soon as it lands,
            // and copied to TMEM once the previous unit's last S product is done.
            // Both named barriers run in every iteration, whatever the waits
            // returned, so the four warps always meet.
            {
                int g = T.n;   // key tiles of the units before
                for (int ku = 1;; ++ku) {
                    const int uu = int(blockIdx.x) + ku * int(gridDim.x);
                    if (uu >= p.n_units) break;
                    const Unit Uu = decode_unit<kKvSplit>(p, uu);
                    const Tiles Tu = make_tiles<BN, kKvSplit>(Uu.q0, Uu.split, p);
                    bool okq = __all_sync(0xffffffffu, mbar_wait(&bar.full_q, ku & 1, abort, tmo));
                    if (okq)
                        rotate_tile_bf16<D, RD, kHalf, kSplit, false, kBM>(
                            sQ, sQ + C::kTileQ, (long long)Uu.tq0(0) + p.qoff, ph, p, rotq);
                    named_bar_sync(1, 128);
                    if (okq)
                        okq = __all_sync(0xffffffffu,
                                         mbar_wait(&bar.s_ready[0][(g - 1) % C::kNB],
                                                   ((g - 1) / C::kNB) & 1, abort, tmo));
                    if (okq) {
                        tc_fence_after();
                        q_parts_to_tmem<D, C::kBoxQ>(sQ, sQ + C::kTileQ, tw,
                                                     tmem + (uint32_t((warp & 3) * 32) << 16) +
                                                         C::kColQ);
                        tc_fence_before();
                    }
                    named_bar_sync(1, 128);
                    if (okq) {
                        fence_proxy_async_smem();
                        mbar_arrive(&bar.ready_q);
                    }
                    g += Tu.n;
                }
            }
        }
        // bf16 keys that are already rotated (and, split, already in parts) go
        // straight from the TMA to the MMA
        bool relay_k = kF32 || (kSplit && !p.k_x8_tma) || rotk;
        if constexpr (kKvSplit && !kF32) {
            if (ok && p.rot_help) {
                rotate_keys_helped<D, RD, kHalf, kSplit, NSK, BN, C::kParts, C::kTileK>(
                    tw, T, sK, bar, p, abort, tmo);
                relay_k = false;
            }
        }
        for (int j = 0; ok && relay_k && j < T.n; ++j) {
            const int jt = T.tile(j);
            const int s = j % NSK, use = j / NSK, sv = j % NSV, usev = j / NSV;
            uint8_t *tk = sK + s * C::kParts * C::kTileK;
            if constexpr (!kF32) {
                ok = __all_sync(0xffffffffu, mbar_wait(&bar.full_k[s], use & 1, abort, tmo));
                if (!ok) break;
                if (rotk || kSplit)
                    rotate_tile_bf16<D, RD, kHalf, kSplit, true, BN>(
                        tk, tk + C::kTileK, (long long)jt * BN, ph, p, rotk, &kcarry);
            } else {
                if (use > 0)
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait(C::kKFreeOnS ? &bar.s_ready[0][s] : &bar.empty_k[s],
                                              (use - 1) & 1, abort, tmo));
                if (!ok) break;
                const float *base = reinterpret_cast<const float *>(p.k) + U.b * p.ks[0] +
                                    (long long)U.g * p.ks[1];
                load_tile_f32<D, kHalf, kSplit, true, BN, kTF>(tk, tk + C::kTileK, base,
                                                               p.ks[2], jt * BN, p.Lk,
                                                               (long long)jt * BN, rotk, ph, p);
            }
            fence_proxy_async_smem();
            mbar_arrive(&bar.ready_k[s]);
            if constexpr (kF32) {
                if (usev > 0)
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait(&bar.empty_v[sv], (usev - 1) & 1, abort, tmo));
                if (!ok) break;
                const float *base = reinterpret_cast<const float *>(p.v) + U.b * p.vs[0] +
                                    (long long)U.g * p.vs[1];
                load_v_f32<D, BN, kTF, kPF16>(sV + sv * C::kTileV, base, p.vs[2], jt * BN, p.Lk,
                                              tw);
                fence_proxy_async_smem();
                mbar_arrive(&bar.full_v[sv]);
            }
        }
    } else {
        setmaxnreg_inc<kRegsSoftmax>();
        if (kKvSplit && !kF32 && ((p.rot_help >> warp) & 1)) {
            // a softmax warp whose rows hold no query: it helps rotate key tiles
            const int ord = __popc(p.rot_help & ((1u << warp) - 1u));
            rotate_keys_helped<D, RD, kHalf, kSplit, NSK, BN, C::kParts, C::kTileK>(
                128 + 32 * ord + lane, T, sK, bar, p, abort, tmo);
        } else if (kSplit && !kKvSplit && p.v_f16) {
            // ------------------------------------------------ softmax, split mode
            // With V already in fp16 the one query tile takes all eight softmax
            // warps, two threads per row: warp w holds rows 32 (w % 4) + 16 (w / 4)
            // .. + 15 (TMEM lanes of its quadrant), its lanes 0-15 keys 0-63 of
            // those rows (output dims 0-63) and lanes 16-31 keys 64-127 (dims
            // 64-127).  Row max and sum combine with one shuffle; the two warps
            // of an SMSP overlap one's exponentials with the other's other work.
            constexpr int NB = C::kNB;
            constexpr int HB = BN / 2;                        // keys per thread
            static_assert(kPF16 || !kSplit, "the split mode's P is fp16");
            const int hf = lane >> 4;                         // column half
            const int row = (warp & 3) * 32 + (warp >> 2) * 16 + (lane & 15);
            const uint32_t tl = tmem + (uint32_t((warp & 3) * 32 + (warp >> 2) * 16) << 16);
            const float cl2 = p.c_log2;
            bool ok = true;
            // Persistent launches take their units one after the other; S
            // buffers and V stages keep counting across them (g: the key tiles
            // of the units before).
            int g = 0;
            for (int ku = 0; ok; ++ku) {
            const int uu = int(blockIdx.x) + ku * int(gridDim.x);
            if (kPersist ? uu >= p.n_units : ku > 0) break;
            const Unit Uu = kPersist ? decode_unit<kKvSplit>(p, uu) : U;
            const Tiles Tu = kPersist ? make_tiles<BN, kKvSplit>(Uu.q0, Uu.split, p) : T;
            const RowMap rm = map_row(p, Uu, 0, row, false);
            const int pi = rm.i + p.qoff;                     // this row's query position
            const int tq0 = Uu.tq0(0);
            float m = -INFINITY, l = 0.f;                     // l: this thread's half
            for (int it = 0; it < Tu.n; ++it) {
                const int gi = g + it;
                const int b = gi % NB;
                const uint32_t s_col = b * BN;
                ok = __all_sync(0xffffffffu,
                                mbar_wait(&bar.s_ready[0][b], (gi / NB) & 1, abort, tmo));
                if (!ok) break;
                tc_fence_after();
                const int jt = Tu.tile(it), k0 = jt * BN + hf * HB;   // this thread's first key
                const bool partial = !tile_full<BN>(tq0, jt, p);
                // visible columns: col <= hi and (no window or col >= lo or col < sk)
                const int hi = p.causal ? min(pi - k0, p.Lk - 1 - k0) : p.Lk - 1 - k0;
                const int lo = pi - p.window + 1 - k0;
                const int sk = p.sinks - k0;
                const bool win = p.causal && p.window > 0;
                float v[HB];
                tmem_ld16x2_64(tl + s_col, v);
                if (partial) {
#pragma unroll
                    for (int e = 0; e < HB; ++e) {
                        const bool keep = (e <= hi) & (!win | (e >= lo) | (e < sk));
                        v[e] = keep ? v[e] : -INFINITY;
                    }
                }
                const float mh = row_max(v);
                const float mx = fmaxf(mh, __shfl_xor_sync(0xffffffffu, mh, 16));
                const float m_new = fmaxf(m, mx * cl2);
                // Keep the old reference unless the max grew by more than 2^15.
                const bool need = (m != -INFINITY) && (m_new > m + kRescaleLog2);
                if (__any_sync(0xffffffffu, need)) {
                    // O must not be in flight: PV(j - 1), signalled on its V
                    // stage's barrier.  Each thread rescales its half of the row's
                    // output dims.
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait(&bar.empty_v[(gi - 1) % NSV], ((gi - 1) / NSV) & 1,
                                              abort, tmo));
                    if (!ok) break;
                    tc_fence_after();
                    const float alpha = need ? ex2_approx(m - m_new) : 1.f;
#pragma unroll 1
                    for (int c = 0; c < DV / 64; ++c) {
                        float o[32];
                        tmem_ld16x2_32(tl + C::kColO + c * 64, o);
                        uint32_t u[32];
#pragma unroll
                        for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(o[e] * alpha);
                        tmem_st16x2_32(tl + C::kColO + c * 64, u);
                    }
                    if (need) {
                        l *= alpha;
                        m = m_new;
                    }
                }
                if (m == -INFINITY) m = m_new;
                const float mref = (m == -INFINITY) ? 0.f : m;
                // P = 2^(s c - m) as fp16 pairs over the first half of S (this
                // thread's keys: P columns 32 hf .. 32 hf + 31), summed in fp32
                const float2 c2 = make_float2(cl2, cl2), nm2 = make_float2(-mref, -mref);
                float2 lsum = make_float2(0.f, 0.f);
                uint32_t pk[HB / 2];
#pragma unroll
                for (int e = 0; e < HB / 2; ++e) {
                    const float2 x = fma2(make_float2(v[2 * e], v[2 * e + 1]), c2, nm2);
                    const float2 pe = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                    pk[e] = pack_f16x2(pe.x, pe.y);
                    lsum = add2(lsum, pe);
                }
                tmem_st16x2_32(tl + s_col, pk);
                l += lsum.x + lsum.y;
                tc_fence_before();
                mbar_arrive(&bar.p_ready[0][b]);
            }
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar.o_ready[0], ku & 1, abort, tmo));
            if (ok) {
                tc_fence_after();
                const float lt = l + __shfl_xor_sync(0xffffffffu, l, 16);   // the row's sum
                const float inv = lt > 0.f ? 1.f / lt : 0.f;
#pragma unroll 1
                for (int c = 0; c < DV / 64; ++c) {
                    float o[32];
                    tmem_ld16x2_32(tl + C::kColO + c * 64, o);
                    if constexpr (kPersist) {
                        // O read: a persistent launch's next unit may start its
                        // first PV into the same columns
                        if (c == DV / 64 - 1) {
                            tc_fence_before();
                            mbar_arrive(&bar.o_free);
                        }
                    }
                    if (rm.valid)
                        store_o32<DV, kF32, kKvSplit>(p, Uu, Uu.split, rm.h, rm.i, 2 * c + hf, o, inv);
                }
                if (rm.valid && hf == 0) {
                    const float ln2 = 0.69314718055994531f;
                    store_lse<kKvSplit>(p, Uu, Uu.split, rm.h, rm.i,
                                        lt > 0.f ? (m + __log2f(lt)) * ln2 : -INFINITY);
                }
            }
            g += Tu.n;
            }
        } else if (kConvV && warp >= 4) {
            // split mode: its one query tile leaves softmax warps 4-7 free; unless
            // V arrives in fp16 already, they convert every V tile to fp16 for the
            // PV product, in key-tile order
            const int tw = threadIdx.x - 128;
            bool ok = !p.v_f16;
            for (int j = 0; ok && j < T.n; ++j) {
                const int sv = j % NSV;
                ok = __all_sync(0xffffffffu, mbar_wait(&bar.full_v[sv], (j / NSV) & 1, abort, tmo));
                if (!ok) break;
                bf16_tile_to_f16<C::kTileV>(sV + sv * C::kTileV, tw);
                fence_proxy_async_smem();
                mbar_arrive(&bar.fp16_v[sv]);
            }
        } else if ((warp >> 2) < U.nt) {
            // ------------------------------------------------ softmax, tile t
            // Warps 0-3 serve query tile 0 and warps 4-7 tile 1, one thread per
            // row (TMEM lane), the whole S row in registers.  (All eight warps
            // on one tile at a time, two threads per row, was measured 5%
            // slower: twice the per-row overhead for the same MUFU work.)
            const int t = warp >> 2;
            const int wq = warp & 3;
            const int row = wq * 32 + lane;
            const uint32_t trow = tmem + (uint32_t(wq * 32) << 16);
            const uint32_t o_col = C::kColO + t * DV;
            const RowMap rm = map_row(p, U, t, row, packed);
            const int pi = rm.i + p.qoff;  // this row's query position
            const int tq0 = U.tq0(t);      // the tile's first query row
            const float cl2 = p.c_log2;
            float m = -INFINITY, l = 0.f;
            bool ok = true;
            // Split-KV (decode) tiles hold few queries: a warp whose 32 rows hold
            // none only keeps step with the barriers, which leaves its SMSP to the
            // rotation warp (its P rows are never used: their O rows are not stored).
            const bool idle = kKvSplit && !__any_sync(0xffffffffu, rm.valid);
            // Interleaved key tiles (head-packed split-KV): this tile takes the
            // key tiles j = t mod 2 of the split and writes partial 2 split + t.
            const bool ilv = kKvSplit && p.pack_ilv;
            const int n_it = ilv ? (T.n - t + 1) / 2 : T.n;
            constexpr int NB = C::kNB;
            for (int it = 0; it < n_it; ++it) {
                const int j = ilv ? 2 * it + t : it;
                const int b = it % NB;
                const uint32_t s_col = (t * NB + b) * BN;
                ok = __all_sync(0xffffffffu,
                                mbar_wait(&bar.s_ready[t][b], (it / NB) & 1, abort, tmo));
                if (!ok) break;
                if (idle) {
                    mbar_arrive(&bar.p_ready[t][b]);
                    continue;
                }
                tc_fence_after();
                const int jt = T.tile(j), k0 = jt * BN;
                const bool partial = !tile_full<BN>(tq0, jt, p);
                // visible columns: col <= hi and (no window or col >= lo or col < sk)
                const int hi = p.causal ? min(pi - k0, p.Lk - 1 - k0) : p.Lk - 1 - k0;
                const int lo = pi - p.window + 1 - k0;
                const int sk = p.sinks - k0;
                const bool win = p.causal && p.window > 0;

                // The whole S row of this thread in one TMEM load.
                float v[BN];
                tmem_ld128(trow + s_col, v);
                if (partial) {
                    // A select per column, no branch: the rows of a warp see
                    // different columns, and a branch per column (divergent across
                    // the warp) cost ~13k cycles per partial tile.
#pragma unroll
                    for (int e = 0; e < BN; ++e) {
                        const bool keep = (e <= hi) & (!win | (e >= lo) | (e < sk));
                        v[e] = keep ? v[e] : -INFINITY;
                    }
                }
                const float mx = row_max(v);
                const float m_new = fmaxf(m, mx * cl2);
                // Keep the old reference unless the max grew by more than 2^15: the
                // result is exact either way, only O's rescale is saved.
                const bool need = (m != -INFINITY) && (m_new > m + kRescaleLog2);
                if (__any_sync(0xffffffffu, need)) {
                    if (NB > 1) {
                        // O must not be in flight: wait for PV(j - 1), whose
                        // completion is signalled on its V stage's barrier (S(j)
                        // done implies PV(j - 2) was, and PV(j) needs this tile's
                        // P, so no other phase of that barrier can be pending).
                        // With one S buffer, S_t(j) is issued after PV_t(j - 1), so
                        // its completion implies it.
                        ok = __all_sync(0xffffffffu,
                                        mbar_wait(&bar.empty_v[(it - 1) % NSV],
                                                  ((it - 1) / NSV) & 1, abort, tmo));
                        if (!ok) break;
                        tc_fence_after();
                    }
                    const float alpha = need ? ex2_approx(m - m_new) : 1.f;
                    // chunk by chunk; the stores are not waited for one by one,
                    // only once before P is handed over
#pragma unroll 1
                    for (int c = 0; c < DV / 32; ++c) {
                        float o[32];
                        tmem_ld32(trow + o_col + c * 32, o);
                        uint32_t u[32];
#pragma unroll
                        for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(o[e] * alpha);
                        tmem_st32_nowait(trow + o_col + c * 32, u);
                    }
                    tmem_wait_st();
                    if (need) {
                        l *= alpha;
                        m = m_new;
                    }
                }
                if (m == -INFINITY) m = m_new;
                const float mref = (m == -INFINITY) ? 0.f : m;
                // P = 2^(s c - m): as bf16 pairs (fp16 pairs in the split mode)
                // over the first half of S, or, tf32 operands, as tf32 values over
                // all of S.  One column pair in kEmuEvery takes 2^x on the FMA pipe.
                const float2 c2 = make_float2(cl2, cl2), nm2 = make_float2(-mref, -mref);
                float2 lsum = make_float2(0.f, 0.f);
                if constexpr (kTF) {
#pragma unroll
                    for (int e = 0; e < BN / 2; ++e) {
                        const float2 x = fma2(make_float2(v[2 * e], v[2 * e + 1]), c2, nm2);
                        // the weights the tensor core multiplies V with (tf32), and
                        // the normalisation by their sum
                        const float2 pe = make_float2(round_tf32(ex2_approx(x.x)),
                                                      round_tf32(ex2_approx(x.y)));
                        v[2 * e] = pe.x;
                        v[2 * e + 1] = pe.y;
                        lsum = add2(lsum, pe);
                    }
                    uint32_t pw[64];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
#pragma unroll
                        for (int e = 0; e < 64; ++e) pw[e] = __float_as_uint(v[64 * h + e]);
                        tmem_st64(trow + s_col + 64 * h, pw);
                    }
                } else {
                    uint32_t pk[BN / 2];
#pragma unroll
                    for (int e = 0; e < BN / 2; ++e) {
                        const float2 x = fma2(make_float2(v[2 * e], v[2 * e + 1]), c2, nm2);
                        float2 pe;
                        if (kEmuEvery > 0 && (e % (kEmuEvery > 0 ? kEmuEvery : 1)) == kEmuEvery - 1)
                            pe = exp2_fma2(x);
                        else
                            pe = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                        if (kPF16) {
                            // fp16 weights (11 significant bits; at most 2^15 with
                            // the stale reference, inside fp16's range).  Summed
                            // before rounding: an fp16 weight is within 2^-12 of
                            // its fp32 value, and unpacking every pair would put
                            // two more conversions per pair on the pipe the
                            // exponentials use.
                            pk[e] = pack_f16x2(pe.x, pe.y);
                            lsum = add2(lsum, pe);
                        } else if (kSplit) {
                            pk[e] = pack_bf16x2(pe.x, pe.y);
                            // Normalise by the weights the tensor core actually
                            // multiplies V with (bf16), not their fp32 values: with
                            // the stale max reference the dominant weight is 2^d,
                            // d in [0, 15], and its rounding must cancel in o.
                            lsum = add2(lsum,
                                        make_float2(bf16lo_to_f32(pk[e]), bf16hi_to_f32(pk[e])));
                        } else {
                            pk[e] = pack_bf16x2(pe.x, pe.y);
                            lsum = add2(lsum, pe);
                        }
                    }
                    tmem_st64(trow + s_col, pk);
                }
                l += lsum.x + lsum.y;
                tc_fence_before();
                mbar_arrive(&bar.p_ready[t][b]);
            }
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar.o_ready[t], 0, abort, tmo));
            if (ok) {
                tc_fence_after();
                const float inv = l > 0.f ? 1.f / l : 0.f;
                const int slot = ilv ? 2 * U.split + t : U.split;
#pragma unroll 1
                for (int c = 0; c < DV / 32; ++c) {
                    float v[32];
                    if (n_it > 0) {
                        tmem_ld32(trow + o_col + c * 32, v);
                    } else {
                        // no key tile reached this tile: O_t was never written
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = 0.f;
                    }
                    if (rm.valid)
                        store_o32<DV, kF32, kKvSplit>(p, U, slot, rm.h, rm.i, c, v, inv);
                }
                if (rm.valid) {
                    const float ln2 = 0.69314718055994531f;
                    store_lse<kKvSplit>(p, U, slot, rm.h, rm.i,
                                        l > 0.f ? (m + __log2f(l)) * ln2 : -INFINITY);
                }
            }
        }
    }

    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (threadIdx.x == 0 && !pre && bar.abort && p.status)
        atomicExch(p.status, int(LCX_ERR_TIMEOUT));
}

// ---------------------------------------------------------------- decode kernel
// Split-KV decode with the scores transposed: S^T = K Q^T puts one key per TMEM
// lane and one query per column, the queries being the kv group's G heads times
// the L rows of the call (G L <= NQ).  The query-tile kernel above gives each
// query row a thread that evaluates all 128 keys of a tile, so a decode tile
// of 4 heads keeps 4 of a warp's 32 rows busy and computes 8 times the
// exponentials it needs.  Here the thread of key r evaluates only that key's
// G L weights.  A column's maximum is reduced over the 128 key threads
// (shuffles, then four warps through shared memory) only when a vote finds a
// logit past the column's lazy reference; its sum once, at the end.  The weights go to shared
// memory as the K-major B operand of O^T = V^T P^T, whose A operand is the V
// tile read MN-major exactly as the TMA lands it, and O^T keeps one output
// column per TMEM lane.  The query block takes 4 KB of shared memory instead of
// two 32 KB query tiles, which leaves room for three K and three V stages.
namespace dec {
constexpr int kThreads = 480;  // warps 0-3 softmax, 4-11 rotation, 12 K, 13 MMA, 14 V
constexpr int D = 128, BN = 128, NQ = 16;
constexpr int NBS = 4, NBP = 2;    // S^T buffers, P buffers
constexpr int kTile = BN * D * 2;  // a K (or K part) or V tile of 16-bit values
constexpr int kBox = BN * 128;     // its 128-byte-wide boxes
constexpr int kQBox = NQ * 128;    // a 128-byte-wide box of the query or P block
constexpr int kColO = NBS * NQ;    // TMEM: NBS S^T buffers of NQ columns, then O^T
// Shared-memory plan.  bf16 QK^T: three K and three V stages.  Split QK^T
// (keys as the fp16 part plus the 8-bit cross part, 64 KB a stage; V in fp16):
// two of each.  Then the query block (its parts), two P buffers, the column
// exchange area and the barriers.
template <bool kSplitQK>
struct Cfg {
    static constexpr int kParts = kSplitQK ? 2 : 1;
    static constexpr int NSK = kSplitQK ? 2 : 3, NSV = kSplitQK ? 2 : 3;
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kOffK + NSK * kParts * kTile;
    static constexpr int kOffQ = kOffV + NSV * kTile;
    static constexpr int kOffP = kOffQ + kParts * (D / 64) * kQBox;
    static constexpr int kOffX = kOffP + NBP * (BN / 64) * kQBox;
    static constexpr int kOffBar = kOffX + 1024;
    static constexpr int kSmemBytes = kOffBar + 256 + 1024;  // barriers + alignment slack
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};
template <int NSK, int NSV>
struct Bars {
    uint64_t ready_q;
    uint64_t full_k[NSK], ready_k[NSK], empty_k[NSK];
    uint64_t full_v[NSV], empty_v[NSV];
    uint64_t s_ready[NBS], p_ready[NBP], p_free[NBP];
    uint64_t o_ready, drain;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Bars<3, 3>) <= 256, "barrier block");
}  // namespace dec

// The group's query block: row n = k L + i holds query i of head hq0 + k
// (n < nq; the other rows are zero), rotated at position qoff + i unless the
// queries arrive rotated, stored as the K-major B operand of S^T (two 64-column
// boxes of NQ 128-byte rows, 128-byte swizzle; split QK^T: the fp16 part, then
// the 8-bit cross part in as many boxes).  Thread tw (of 128) takes row tw / 8
// and its pairs 8 (tw % 8) .. + 7: two 16-byte loads; each angle from the
// accurate sine and cosine.
template <bool kHalf, bool kSplitQK>
__device__ __forceinline__ void load_q_decode(uint8_t *sQ, const AttnParams &p, const Unit &U,
                                              int nq, int tw) {
    using namespace dec;
    static_assert(NQ * 8 == 128, "one row segment per thread");
    const int n = tw >> 3, g = tw & 7;
    // the 16-byte chunks (8 columns each) that hold the thread's pairs
    const int c1 = kHalf ? g : 2 * g, c2 = kHalf ? g + D / 16 : 2 * g + 1;
    float x[8], y[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = y[e] = 0.f;
    if (n < nq) {
        const int i = n % p.L;
        const uint4 *row = reinterpret_cast<const uint4 *>(
            reinterpret_cast<const __nv_bfloat16 *>(p.q) + U.b * p.qs[0] +
            (long long)(U.hq0 + n / p.L) * p.qs[1] + (long long)i * p.qs[2]);
        unpack8(row[c1], x);
        unpack8(row[c2], y);
        if (p.rotate_q) {
            float c[8], s[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                rope_sincos((long long)p.qoff + i, p.theta[8 * g + e], &c[e], &s[e]);
            // half pairing: pair 8 g + e is (x[e], y[e]); interleaved: pairs
            // 8 g + e and 8 g + 4 + e are (x[2e], x[2e+1]) and (y[2e], y[2e+1])
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float &u = kHalf ? x[e] : (e < 4 ? x[2 * e] : y[2 * (e - 4)]);
                float &v = kHalf ? y[e] : (e < 4 ? x[2 * e + 1] : y[2 * (e - 4) + 1]);
                const float u0 = u, v0 = v;
                u = u0 * c[e] - v0 * s[e];
                v = v0 * c[e] + u0 * s[e];
            }
        }
    }
    if constexpr (kSplitQK) {
        // the fp16 part, and the 8-bit cross part [h8 | r8], of the rotated values
        store8<true, false, D, kQBox>(sQ, sQ + (D / 64) * kQBox, n, c1, x);
        store8<true, false, D, kQBox>(sQ, sQ + (D / 64) * kQBox, n, c2, y);
    } else {
        *reinterpret_cast<uint4 *>(sQ + chunk_off(n, c1, kQBox)) = pack8(x);
        *reinterpret_cast<uint4 *>(sQ + chunk_off(n, c2, kQBox)) = pack8(y);
    }
}

// One CTA per (batch, kv group, key split): bf16 operands, D = DV = 128, full
// rotary, partial results (o normalised, lse) into the split workspace.  kNQ:
// the query columns the softmax reads (4, 8 or 16 >= G L).  kSplitQK: the
// split mode's S = Qh Kh^T + [Qh8 | Qr8] [Kr8 | Kh8]^T, transposed, with the
// keys' parts and V in fp16 as the rotate pass wrote them (tmk: the fp16 parts,
// tmkr: the 8-bit cross parts), and fp16 weights for PV.
template <bool kHalf, int kNQ, bool kSplitQK>
__global__ void __launch_bounds__(dec::kThreads, 1)
    attn_decode_kernel(const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv,
                       const __grid_constant__ CUtensorMap tmkr,
                       const __grid_constant__ AttnParams p) {
    using namespace dec;
    using C = dec::Cfg<kSplitQK>;
    constexpr int NSK = C::NSK, NSV = C::NSV;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sK = smem + C::kOffK;  // stage s at sK + s kParts kTile (split: fp16 part, 8-bit part)
    uint8_t *sV = smem + C::kOffV;
    uint8_t *sQ = smem + C::kOffQ;
    uint8_t *sP = smem + C::kOffP;
    float *xmax = reinterpret_cast<float *>(smem + C::kOffX);  // [2][4][kNQ] column maxima per warp
    float *xsum = xmax + 2 * 4 * kNQ;                           // [4][kNQ] column sums per warp
    dec::Bars<NSK, NSV> &bar = *reinterpret_cast<dec::Bars<NSK, NSV> *>(smem + C::kOffBar);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const Unit U = decode_unit<true>(p);
    const Tiles T = make_tiles<BN, true>(U.q0, U.split, p);
    const int nq = p.G * p.L;  // query columns in use
    volatile int *abort = &bar.abort;
    const uint64_t tmo = p.timeout_ns;

    if (threadIdx.x == 0) {
        mbar_init(&bar.ready_q, 128);
        for (int s = 0; s < NSK; ++s) {
            mbar_init(&bar.full_k[s], 1);
            mbar_init(&bar.ready_k[s], 256);
            mbar_init(&bar.empty_k[s], 1);
        }
        for (int s = 0; s < NSV; ++s) {
            mbar_init(&bar.full_v[s], 1);
            mbar_init(&bar.empty_v[s], 1);
        }
        for (int b = 0; b < NBS; ++b) mbar_init(&bar.s_ready[b], 1);
        for (int b = 0; b < NBP; ++b) {
            mbar_init(&bar.p_ready[b], 128);
            mbar_init(&bar.p_free[b], 1);
        }
        mbar_init(&bar.o_ready, 1);
        mbar_init(&bar.drain, 1);
        bar.abort = 0;
        fence_mbar_init();
    }
    if (warp == 13) {
        tmem_alloc(&bar.tmem_base, 128);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_base;
    // A CTA that starts after another one's watchdog fired gives up at its
    // first wait that does not complete at once (the status word is read by
    // thread 0 after the barrier, off the roles' path).
    bool pre = false;   // thread 0: the word was already set
    if (threadIdx.x == 0 && p.status && *reinterpret_cast<volatile int *>(p.status) != 0) {
        pre = true;
        *abort = 1;
    }
    // the merge of the partial results may be scheduled now (it waits for this
    // grid to finish before it reads them)
    pdl_launch_dependents();

    if (T.n == 0) {
        // a split that received no key tile: the empty partial result
        if (warp < 4) {
            for (int n = 0; n < nq; ++n) {
                const long long prow =
                    (((long long)U.split * p.B + U.b) * p.Hq + U.hq0 + n / p.L) * p.L + n % p.L;
                p.part_o[prow * D + threadIdx.x] = 0.f;
                if (threadIdx.x == 0) p.part_lse[prow] = -INFINITY;
            }
        }
    } else if (warp == 12 || warp == 14) {
        // ------------------------------------------------ TMA producers: K (12), V (14)
        if (lane == 0 && !p.test_stall) {
            const bool isk = warp == 12;
            constexpr int NS = NSK > NSV ? NSK : NSV;
            const int ns = isk ? NSK : NSV;
            uint64_t *full = isk ? bar.full_k : bar.full_v;
            uint64_t *empty = isk ? bar.empty_k : bar.empty_v;
            uint8_t *base = isk ? sK : sV;
            const CUtensorMap *map = isk ? &tmk : &tmv;
            tma_prefetch_desc(map);
            if (kSplitQK && isk) tma_prefetch_desc(&tmkr);
            // split mode: a K stage is the fp16 part then the 8-bit cross part
            const int parts = (kSplitQK && isk) ? 2 : 1;
            int issued[NS] = {};
            bool ok = true;
            for (int j = 0; ok && j < T.n; ++j) {
                const int jt = T.tile(j), s = j % ns, u = j / ns;
                if (u > 0) ok = mbar_wait(&empty[s], (u - 1) & 1, abort, tmo);
                if (!ok) break;
                uint8_t *dst = base + s * parts * kTile;
                mbar_arrive_expect_tx(&full[s], parts * kTile);
                for (int bx = 0; bx < D / 64; ++bx)
                    tma_load_4d(dst + bx * kBox, map, &full[s], bx * 64, jt * BN, U.g, U.b);
                if (parts == 2)   // 2 D bytes per key: D / 64 boxes of 128 bytes
                    for (int bx = 0; bx < D / 64; ++bx)
                        tma_load_4d(dst + kTile + bx * kBox, &tmkr, &full[s], bx * 128, jt * BN,
                                    U.g, U.b);
                ++issued[s];
            }
            // never leave the CTA with copies in flight (bounded, even after an abort)
            for (int s = 0; s < ns; ++s)
                if (issued[s]) mbar_wait(&full[s], (issued[s] - 1) & 1, nullptr, tmo);
        }
    } else if (warp == 13) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            // S^T: A = the K tile, B = the query block, both K-major.  O^T: A = the
            // V tile, MN-major; B = the weights, K-major.  M = 128, N = NQ.
            constexpr uint32_t kIdS = kSplitQK ? idesc_f32acc(128, NQ, kFmtF16, kFmtF16, 0, 0)
                                               : idesc_bf16_f32(128, NQ, 0, 0);
            constexpr uint32_t kIdX8 = idesc_f32acc(128, NQ, kFmtE5M2, kFmtE5M2, 0, 0);
            constexpr uint32_t kIdO = kSplitQK ? idesc_f32acc(128, NQ, kFmtF16, kFmtF16, 1, 0)
                                               : idesc_bf16_f32(128, NQ, 1, 0);
            const uint64_t dv0 = sdesc_sw128(smem_u32(sV), kBox, 1024);
            const uint32_t dhi = uint32_t(dv0 >> 32);  // the same for every descriptor here
            const uint32_t v_lo = uint32_t(dv0);
            const uint32_t k_lo = uint32_t(sdesc_sw128(smem_u32(sK), 16, 1024));
            const uint32_t q_lo = uint32_t(sdesc_sw128(smem_u32(sQ), 16, 1024));
            const uint32_t p_lo = uint32_t(sdesc_sw128(smem_u32(sP), 16, 1024));
            uint64_t *kready = p.rotate_k ? bar.ready_k : bar.full_k;
            auto issue_s = [&](int j) {
                const uint32_t ka = k_lo + (((j % NSK) * C::kParts * kTile) >> 4);
                const uint32_t dst = tmem + (j % NBS) * NQ;
                if constexpr (kSplitQK) {
                    // the e5m2 cross product over K = 2 D bytes (32 per
                    // instruction, the same box geometry as the 16-bit parts)
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t ok_ = ((kk >> 2) * kBox + (kk & 3) * 32) >> 4;
                        const uint32_t oq = ((kk >> 2) * kQBox + (kk & 3) * 32) >> 4;
                        mma_ss_w<1>(dst, ka + (kTile >> 4) + ok_,
                                    q_lo + (((D / 64) * kQBox) >> 4) + oq, dhi, kIdX8, kk > 0);
                    }
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t ok_ = ((kk >> 2) * kBox + (kk & 3) * 32) >> 4;
                    const uint32_t oq = ((kk >> 2) * kQBox + (kk & 3) * 32) >> 4;
                    mma_ss_w<0>(dst, ka + ok_, q_lo + oq, dhi, kIdS, kSplitQK || kk > 0);
                }
            };
            auto issue_pv = [&](int j) {
                const uint32_t va = v_lo + (((j % NSV) * kTile) >> 4);
                const uint32_t pa = p_lo + (((j % NBP) * (BN / 64) * kQBox) >> 4);
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint32_t ov = (kk * 16 * 128) >> 4;  // 16 keys: 16 rows of the V tile
                    const uint32_t op = ((kk >> 2) * kQBox + (kk & 3) * 32) >> 4;
                    mma_ss_w<0>(tmem + kColO, va + ov, pa + op, dhi, kIdO, (j > 0 || kk > 0));
                }
            };
            bool ok = mbar_wait(&bar.ready_q, 0, abort, tmo);
            // S^T runs up to NBS key tiles ahead of the softmax
            for (int j = 0; ok && j < NBS && j < T.n; ++j) {
                ok = mbar_wait(&kready[j % NSK], (j / NSK) & 1, abort, tmo);
                tc_fence_after();
                if (!ok) break;
                issue_s(j);
                mma_commit(&bar.s_ready[j % NBS]);
                mma_commit(&bar.empty_k[j % NSK]);
            }
            for (int j = 0; ok && j < T.n; ++j) {
                ok = mbar_wait(&bar.full_v[j % NSV], (j / NSV) & 1, abort, tmo);
                if (ok) ok = mbar_wait(&bar.p_ready[j % NBP], (j / NBP) & 1, abort, tmo);
                tc_fence_after();
                if (!ok) break;
                issue_pv(j);
                mma_commit(&bar.empty_v[j % NSV]);
                mma_commit(&bar.p_free[j % NBP]);
                // S^T(j + NBS) into the buffer the softmax of j has read
                const int jn = j + NBS;
                if (jn < T.n) {
                    ok = mbar_wait(&kready[jn % NSK], (jn / NSK) & 1, abort, tmo);
                    tc_fence_after();
                    if (!ok) break;
                    issue_s(jn);
                    mma_commit(&bar.s_ready[jn % NBS]);
                    mma_commit(&bar.empty_k[jn % NSK]);
                }
            }
            if (ok) mma_commit(&bar.o_ready);
            // every product done before the CTA frees its TMEM (bounded)
            mma_commit(&bar.drain);
            mbar_wait(&bar.drain, 0, nullptr, tmo);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------ queries, then key rotation
        const int tw = threadIdx.x - 128;  // 0..255
        if (tw < 128) {
            load_q_decode<kHalf, kSplitQK>(sQ, p, U, nq, tw);
            fence_proxy_async_smem();
            mbar_arrive(&bar.ready_q);
        }
        // (split mode: the keys always arrive in their parts from the rotate pass)
        if (!kSplitQK && p.rotate_k)
            rotate_keys_helped<D, D, kHalf, false, NSK, BN, 1, kTile>(tw, T, sK, bar, p, abort,
                                                                      tmo);
    } else {
        // ------------------------------------------------ softmax, warps 0-3
        // Thread r holds key r of every key tile (TMEM lane r of S^T) and output
        // column r (lane r of O^T).  Every iteration passes named barrier 2 once,
        // whatever happened, so the four warps always meet.
        const int r = threadIdx.x;
        const uint32_t tl = tmem + (uint32_t(warp * 32) << 16);
        const float cl2 = p.c_log2;
        // the weight buffers' rows n >= nq stay zero
        for (int i = r; i < NBP * (BN / 64) * kQBox / 16; i += 128)
            reinterpret_cast<uint4 *>(sP)[i] = make_uint4(0u, 0u, 0u, 0u);
        // column n sees the keys [lo, hi] and the sinks (none when n >= nq)
        int hi[kNQ], lo[kNQ];
        float m[kNQ], l[kNQ];
#pragma unroll
        for (int n = 0; n < kNQ; ++n) {
            const int pi = p.qoff + n % p.L;  // the query's position
            hi[n] = n >= nq ? -1 : p.causal ? min(pi, p.Lk - 1) : p.Lk - 1;
            lo[n] = (p.causal && p.window > 0) ? pi - p.window + 1 : INT_MIN;
            m[n] = -INFINITY;
            l[n] = 0.f;
        }
        bool ok = true;
        for (int j = 0; j < T.n; ++j) {
            const int pb = j % NBP;
            const uint32_t ps = (j / NBS) & 1, pp = ((j - NBP) / NBP) & 1;
            if (ok) {
                // S^T(j) computed and the weight buffer free (PV(j - NBP) done):
                // both tested at once first, the full waits only if one is pending
                const bool rdy = mbar_try_wait(&bar.s_ready[j % NBS], ps) &&
                                 (j < NBP || mbar_try_wait(&bar.p_free[pb], pp));
                if (!__all_sync(0xffffffffu, rdy)) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&bar.s_ready[j % NBS], ps, abort, tmo));
                    if (ok && j >= NBP)
                        ok = __all_sync(0xffffffffu, mbar_wait(&bar.p_free[pb], pp, abort, tmo));
                }
            }
            float x[kNQ];
            if (ok) {
                tc_fence_after();
                tmem_ldn<kNQ>(tl + (j % NBS) * NQ, x);
            }
            const int key = T.tile(j) * BN + r;
            // logits in log2 units, masked.  The reference m of a column moves
            // only when a logit passes m + 2^15 (exact either way; O^T's
            // rescale is saved): a vote per column, and the warp's maximum only
            // for the columns where the vote says so.
            bool grow[kNQ];
#pragma unroll
            for (int n = 0; n < kNQ; ++n) {
                const bool vis = ok && key <= hi[n] && (key >= lo[n] || key < p.sinks);
                x[n] = vis ? x[n] * cl2 : -INFINITY;
                grow[n] = __any_sync(0xffffffffu, x[n] > m[n] + kRescaleLog2);
            }
#pragma unroll
            for (int n = 0; n < kNQ; ++n) {
                float mx = -INFINITY;
                if (grow[n]) {
                    mx = x[n];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1)
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                }
                if (lane == 0) xmax[((j & 1) * 4 + warp) * kNQ + n] = mx;
            }
            named_bar_sync(2, 128);
            bool rescale = false;
            float alpha[NQ];
#pragma unroll
            for (int n = 0; n < NQ; ++n) alpha[n] = 1.f;
#pragma unroll
            for (int n = 0; n < kNQ; ++n) {
                const float *xm = xmax + (j & 1) * 4 * kNQ + n;
                const float mt = fmaxf(fmaxf(xm[0], xm[kNQ]), fmaxf(xm[2 * kNQ], xm[3 * kNQ]));
                if (mt > m[n] + kRescaleLog2) {
                    if (m[n] != -INFINITY) {
                        alpha[n] = ex2_approx(m[n] - mt);
                        l[n] *= alpha[n];
                        rescale = true;
                    }
                    m[n] = mt;
                }
            }
            if (ok && rescale) {
                // O^T must not be in flight: PV(j - 1) done
                ok = __all_sync(0xffffffffu, mbar_wait(&bar.p_free[(j - 1) % NBP],
                                                       ((j - 1) / NBP) & 1, abort, tmo));
                if (ok) {
                    tc_fence_after();
                    float o[NQ];
                    tmem_ld16(tl + kColO, o);
#pragma unroll
                    for (int n = 0; n < NQ; ++n) o[n] *= alpha[n];
                    tmem_st16(tl + kColO, o);
                }
            }
            if (ok) {
                // the weights 2^(s c - m), bf16 (split mode: fp16, for the fp16
                // V), into row n of the K-major P block
                uint8_t *pbuf = sP + pb * (BN / 64) * kQBox;
#pragma unroll
                for (int n = 0; n < kNQ; ++n) {
                    const float w = ex2_approx(x[n] - (m[n] == -INFINITY ? 0.f : m[n]));
                    l[n] += w;
                    uint8_t *dst = pbuf + chunk_off(n, r >> 3, kQBox) + (r & 7) * 2;
                    if constexpr (kSplitQK)
                        *reinterpret_cast<uint16_t *>(dst) = uint16_t(pack_f16x2(w, 0.f) & 0xFFFFu);
                    else
                        *reinterpret_cast<__nv_bfloat16 *>(dst) = __float2bfloat16_rn(w);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bar.p_ready[pb]);
            }
        }
        // each column's sum over the 128 keys
#pragma unroll
        for (int n = 0; n < kNQ; ++n) {
            float sum = l[n];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            if (lane == 0) xsum[warp * kNQ + n] = sum;
        }
        named_bar_sync(2, 128);
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar.o_ready, 0, abort, tmo));
        if (ok) {
            tc_fence_after();
            float o[kNQ];
            tmem_ldn<kNQ>(tl + kColO, o);
            const float ln2 = 0.69314718055994531f;
#pragma unroll
            for (int n = 0; n < kNQ; ++n) {
                if (n >= nq) break;
                const float lt = xsum[n] + xsum[kNQ + n] + xsum[2 * kNQ + n] + xsum[3 * kNQ + n];
                const long long prow =
                    (((long long)U.split * p.B + U.b) * p.Hq + U.hq0 + n / p.L) * p.L + n % p.L;
                p.part_o[prow * D + r] = lt > 0.f ? o[n] * (1.f / lt) : 0.f;
                if (r == 0) p.part_lse[prow] = lt > 0.f ? (m[n] + __log2f(lt)) * ln2 : -INFINITY;
            }
        }
    }

    __syncthreads();
    if (warp == 13) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
    if (threadIdx.x == 0 && !pre && bar.abort && p.status)
        atomicExch(p.status, int(LCX_ERR_TIMEOUT));
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(ptr);
    }();
    return fn;
}

// [B, H, L, D] tensor of es-byte elements (2: bf16 or fp16 bits, 1: bytes) ->
// 4-D tensor map whose boxes are 128 bytes (64 or 128 elements) x box_rows,
// 128-byte swizzle.  TMA copies the bits; it never converts them.
lcx_status make_map(CUtensorMap *map, const void *ptr, int64_t B, int64_t H, int64_t L, int64_t D,
                    const int64_t *st, uint32_t box_rows, const char *name, int es = 2) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(LCX_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(L), cuuint64_t(H), cuuint64_t(B)};
    cuuint64_t strides[3] = {cuuint64_t(st[2] * es), cuuint64_t(st[1] * es),
                             cuuint64_t(st[0] * es)};
    cuuint32_t box[4] = {cuuint32_t(128 / es), box_rows, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, es == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                    4, const_cast<void *>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(LCX_ERR_UNSUPPORTED, "tensor map for %s rejected (CUresult %d)", name, int(r));
    return LCX_OK;
}

// The four tensor maps of a launch: q, k (its non-shared columns), v, and the
// shared rotary key (unused unless AttnParams::k_rope_shared).
struct Maps {
    CUtensorMap q, k, v, kr;
};

// Which kernel instance a launch needs.
struct AttnLaunchShape {
    bool f32, half, split_qk;
    int D, DV, RD;    // query/key head dim, value head dim, rotated dims
};

template <int D, int DV, int RD, bool kF32, bool kHalf, bool kSplit, bool kKvSplit,
          bool kPersist>
lcx_status launch_instance(const Maps &m, const AttnParams &p, unsigned grid, cudaStream_t s) {
    auto kern = attn_fwd_kernel<D, DV, RD, kF32, kHalf, kSplit, kKvSplit, kPersist>;
    const int smem = Cfg<D, DV, kSplit, kF32 && !kSplit && D == 64, kKvSplit>::kSmemBytes;
    // The warpgroups re-balance registers with setmaxnreg, which waits until the
    // registers it asks for are free: the launch must hold the whole split.
    static const int regs = []() {
        cudaFuncAttributes fa;
        return cudaFuncGetAttributes(&fa, attn_fwd_kernel<D, DV, RD, kF32, kHalf, kSplit,
                                                         kKvSplit, kPersist>) == cudaSuccess
                   ? fa.numRegs
                   : -1;
    }();
    if (regs * kThreads < (2 * kRegsSoftmax + kRegsRotate + kRegsIssue) * 128)
        return fail(LCX_ERR_CUDA, "attn_fwd kernel built with %d registers per thread; the "
                    "warpgroup register split needs 128", regs);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return fail(LCX_ERR_CUDA, "cudaFuncSetAttribute failed: %s", cudaGetErrorString(e));
    kern<<<grid, kThreads, smem, s>>>(m.q, m.k, m.v, m.kr, p);
    e = cudaGetLastError();
    if (e != cudaSuccess)
        return fail(LCX_ERR_CUDA, "attn_fwd launch failed: %s", cudaGetErrorString(e));
    return LCX_OK;
}

// The persistent instance for the split mode's CTA-per-SM launches (see
// AttnParams::persist), the plain instance otherwise.
template <int D, int DV, int RD, bool kF32, bool kHalf, bool kSplit, bool kKvSplit>
lcx_status launch(const Maps &m, const AttnParams &p, unsigned grid, cudaStream_t s) {
    if constexpr (kSplit && !kKvSplit && !kF32 && D == 128)
        if (p.persist)
            return launch_instance<D, DV, RD, kF32, kHalf, kSplit, kKvSplit, true>(m, p, grid, s);
    return launch_instance<D, DV, RD, kF32, kHalf, kSplit, kKvSplit, false>(m, p, grid, s);
}

// Full rotary (RD = D = DV): bf16 or fp32 operands, plain or split QK^T.
template <int D, bool kSplit, bool kKv>
lcx_status launch_full(bool f32, bool half, const Maps &m, const AttnParams &p, unsigned grid,
                       cudaStream_t s) {
    if (f32)
        return half ? launch<D, D, D, true, true, kSplit, kKv>(m, p, grid, s)
                    : launch<D, D, D, true, false, kSplit, kKv>(m, p, grid, s);
    return half ? launch<D, D, D, false, true, kSplit, kKv>(m, p, grid, s)
                : launch<D, D, D, false, false, kSplit, kKv>(m, p, grid, s);
}

// Partial rotary (the last RD of D dims): bf16 operands, plain QK^T.
template <int D, int DV, int RD, bool kKv>
lcx_status launch_partial(bool half, const Maps &m, const AttnParams &p, unsigned grid,
                          cudaStream_t s) {
    return half ? launch<D, DV, RD, false, true, false, kKv>(m, p, grid, s)
                : launch<D, DV, RD, false, false, false, kKv>(m, p, grid, s);
}

template <bool kKv>
lcx_status launch_shape(const AttnLaunchShape &x, const Maps &m, const AttnParams &p,
                        unsigned g, cudaStream_t s) {
    if (x.D == 192) return launch_partial<192, 128, 64, kKv>(x.half, m, p, g, s);
    if (x.D == 128 && x.RD == 64) return launch_partial<128, 128, 64, kKv>(x.half, m, p, g, s);
    if (x.D == 128)
        return x.split_qk ? launch_full<128, true, kKv>(x.f32, x.half, m, p, g, s)
                          : launch_full<128, false, kKv>(x.f32, x.half, m, p, g, s);
    return x.split_qk ? launch_full<64, true, kKv>(x.f32, x.half, m, p, g, s)
                      : launch_full<64, false, kKv>(x.f32, x.half, m, p, g, s);
}

// The transposed decode kernel (bf16, D = DV = 128, full rotary, G L <= 16).
template <bool kHalf, int kNQ, bool kSplitQK>
lcx_status launch_decode(const Maps &m, const AttnParams &p, unsigned grid, cudaStream_t s) {
    auto kern = attn_decode_kernel<kHalf, kNQ, kSplitQK>;
    constexpr int smem = dec::Cfg<kSplitQK>::kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
        return fail(LCX_ERR_CUDA, "cudaFuncSetAttribute failed: %s", cudaGetErrorString(e));
    kern<<<grid, dec::kThreads, smem, s>>>(m.k, m.v, m.kr, p);
    e = cudaGetLastError();
    if (e != cudaSuccess)
        return fail(LCX_ERR_CUDA, "attn_decode launch failed: %s", cudaGetErrorString(e));
    return LCX_OK;
}

template <bool kHalf, bool kSplitQK>
lcx_status launch_decode_nq(int nq, const Maps &m, const AttnParams &p, unsigned grid,
                            cudaStream_t s) {
    return nq <= 4 ? launch_decode<kHalf, 4, kSplitQK>(m, p, grid, s)
                   : nq <= 8 ? launch_decode<kHalf, 8, kSplitQK>(m, p, grid, s)
                             : launch_decode<kHalf, 16, kSplitQK>(m, p, grid, s);
}

lcx_status check_tensor(const void *ptr, const int64_t *st, int es, const char *name) {
    if (!ptr) return fail(LCX_ERR_INVALID_ARG, "%s is NULL", name);
    if (!aligned16(ptr)) return fail(LCX_ERR_UNSUPPORTED, "%s must be 16-byte aligned", name);
    if (st[3] != 1) return fail(LCX_ERR_UNSUPPORTED, "%s: head_dim stride must be 1", name);
    for (int d = 0; d < 3; ++d) {
        if (st[d] < 0) return fail(LCX_ERR_UNSUPPORTED, "%s: negative stride", name);
        if ((st[d] * es) % 16 != 0)
            return fail(LCX_ERR_UNSUPPORTED, "%s: strides must be multiples of 16 bytes", name);
    }
    return LCX_OK;
}

}  // namespace
}  // namespace lcx

namespace lcx {
namespace {

// Everything one attn_fwd launch needs, derived from validated arguments.
struct AttnLaunch : AttnLaunchShape {
    AttnParams p;
    Maps m;
    long long units;  // CTAs without key splits
    // Keys rotated once before the attention kernel (args.k_rot): the rotate
    // pass reads k_src and writes the contiguous buffer the kernel then reads.
    bool rotate_k_once;
    lcx_rope_params rope;
    const void *k_src;
    int64_t k_src_strides[4];
    void *k_x8;       // split mode: where the pass writes the keys' 8-bit cross parts, or NULL
    void *v16;        // split mode: where a pass writes V in fp16 (contiguous), or NULL
    const void *v_src;
    int64_t v_src_strides[4];
    int rot_h, rot_d; // heads and columns the pass rotates (Hkv, D; or 1, d_R)
    void *k_rot;      // where the pass writes
    bool decode;      // split-KV launch of the transposed decode kernel
    int sms;          // the device's SM count
};

// Validate `a` and fill `x`.  *noop is set for empty problems (B or L zero),
// which succeed without device work.
lcx_status attn_prepare(const lcx_attn_args *a, AttnLaunch &x, bool *noop) {
    *noop = false;
    if (!a) return fail(LCX_ERR_INVALID_ARG, "args is NULL");
    lcx_status st = check_rope_params(&a->rope);
    if (st != LCX_OK) return st;
    if (a->dtype != LCX_BF16 && a->dtype != LCX_F32)
        return fail(LCX_ERR_INVALID_ARG, "unknown dtype %d", a->dtype);
    if (a->B < 0 || a->Hq <= 0 || a->Hkv <= 0 || a->L < 0 || a->D <= 0)
        return fail(LCX_ERR_INVALID_ARG, "bad sizes");
    if (a->Hq % a->Hkv != 0)
        return fail(LCX_ERR_INVALID_ARG, "Hq (%lld) must be a multiple of Hkv (%lld)",
                    (long long)a->Hq, (long long)a->Hkv);
    const int64_t Dv = a->Dv > 0 ? a->Dv : a->D;
    const int64_t RD = a->rope.head_dim;
    if (a->Dv < 0) return fail(LCX_ERR_INVALID_ARG, "Dv must be >= 0");
    if (RD > a->D) return fail(LCX_ERR_INVALID_ARG, "rope.head_dim > D");
    const bool partial = RD < a->D;
    if (a->causal != 0 && a->causal != 1) return fail(LCX_ERR_INVALID_ARG, "causal must be 0 or 1");
    if (a->window < 0 || a->sinks < 0)
        return fail(LCX_ERR_INVALID_ARG, "window and sinks must be >= 0");
    if (!a->causal && (a->window != 0 || a->sinks != 0))
        return fail(LCX_ERR_UNSUPPORTED, "window / sinks need causal attention");
    if (a->flags & ~uint32_t(LCX_ATTN_PREROTATED | LCX_ATTN_PREROTATED_K | LCX_ATTN_SPLIT_QK |
                             LCX_ATTN_TEST_STALL))
        return fail(LCX_ERR_INVALID_ARG, "unknown flags");
    if (a->reserved0 != 0) return fail(LCX_ERR_INVALID_ARG, "reserved0 must be 0");
    const int64_t Lk = a->Lk > 0 ? a->Lk : a->L;
    if (a->Lk < 0 || a->q_offset < 0)
        return fail(LCX_ERR_INVALID_ARG, "Lk and q_offset must be >= 0");
    if (a->causal && a->L > 0 && a->q_offset + a->L > Lk)
        return fail(LCX_ERR_INVALID_ARG,
                    "causal attention needs q_offset + L <= Lk (got %lld + %lld > %lld)",
                    (long long)a->q_offset, (long long)a->L, (long long)Lk);
    if (a->watchdog_ms < 0 || a->watchdog_ms > 60000)
        return fail(LCX_ERR_INVALID_ARG, "watchdog_ms must be in [0, 60000]");
    if ((a->flags & LCX_ATTN_TEST_STALL) && a->dtype != LCX_BF16)
        return fail(LCX_ERR_UNSUPPORTED, "the stall test hook needs bf16 operands");
    if (!(a->softmax_scale >= 0.f) || !std::isfinite(a->softmax_scale))
        return fail(LCX_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
    const bool shape_ok = (a->D == 64 && Dv == 64 && RD == 64) ||
                          (a->D == 128 && Dv == 128 && (RD == 128 || RD == 64)) ||
                          (a->D == 192 && Dv == 128 && RD == 64);
    if (!shape_ok)
        return fail(LCX_ERR_UNSUPPORTED,
                    "(D, Dv, rotated dims) = (%lld, %lld, %lld): supported are (64, 64, 64), "
                    "(128, 128, 128), (128, 128, 64), (192, 128, 64)",
                    (long long)a->D, (long long)Dv, (long long)RD);
    if (partial && (a->dtype != LCX_BF16 || (a->flags & LCX_ATTN_SPLIT_QK)))
        return fail(LCX_ERR_UNSUPPORTED, "partial rotary needs bf16 operands and plain QK^T");
    if (a->k_rope && !partial)
        return fail(LCX_ERR_INVALID_ARG, "k_rope needs rope.head_dim < D");
    if (a->B == 0 || a->L == 0) {
        *noop = true;
        return LCX_OK;
    }
    if (a->L > (int64_t(1) << 30) || Lk > (int64_t(1) << 30) ||
        a->q_offset + a->L > (int64_t(1) << 30) || a->B > (int64_t(1) << 20) || a->Hq > 65536)
        return fail(LCX_ERR_UNSUPPORTED, "sizes too large");
    const int es = a->dtype == LCX_BF16 ? 2 : 4;
    if ((st = check_tensor(a->q, a->q_strides, es, "q")) != LCX_OK) return st;
    if ((st = check_tensor(a->k, a->k_strides, es, "k")) != LCX_OK) return st;
    if ((st = check_tensor(a->v, a->v_strides, es, "v")) != LCX_OK) return st;
    if ((st = check_tensor(a->o, a->o_strides, es, "o")) != LCX_OK) return st;
    if (a->k_rope && (st = check_tensor(a->k_rope, a->k_rope_strides, es, "k_rope")) != LCX_OK)
        return st;
    // Keys rotated once into args.k_rot (by the rotate pass, mscale included)
    // instead of once per key tile per CTA, where the kernel would otherwise
    // rotate them on chip: full-rotary keys ([B, Hkv, Lk, D]), or the shared
    // rotary key of decoupled RoPE ([B, 1, Lk, d_R]; k keeps its un-rotated
    // columns).  In the split-QK^T mode with bf16 keys the pass writes the
    // keys' fp16 parts there, followed by their 8-bit cross parts ([r8 | h8],
    // 2 D bytes per key: as many bytes again), and a second pass the values in
    // fp16 (as many bytes again), so the kernel loads every PV operand as it
    // multiplies it.
    const bool rot_shared = partial && a->k_rope != nullptr;
    const bool rotate_k_once =
        a->k_rot != nullptr && !(a->flags & (LCX_ATTN_PREROTATED | LCX_ATTN_PREROTATED_K |
                                             LCX_ATTN_TEST_STALL)) &&
        ((!partial && !a->k_rope && a->D % 16 == 0) || rot_shared);
    const bool k_x8 = rotate_k_once && (a->flags & LCX_ATTN_SPLIT_QK) && a->dtype == LCX_BF16;
    const int64_t rot_h = rot_shared ? 1 : a->Hkv, rot_d = rot_shared ? RD : a->D;
    const int64_t kst_rot[4] = {rot_h * Lk * rot_d, Lk * rot_d, rot_d, 1};
    const int64_t k_part_bytes = a->B * rot_h * Lk * rot_d * es;
    if (rotate_k_once) {
        if (!aligned16(a->k_rot)) return fail(LCX_ERR_UNSUPPORTED, "k_rot must be 16-byte aligned");
        if (a->k_rot_bytes < k_part_bytes * (k_x8 ? 3 : 1))
            return fail(LCX_ERR_INVALID_ARG, "k_rot holds %lld bytes; %lld needed",
                        (long long)a->k_rot_bytes, (long long)(k_part_bytes * (k_x8 ? 3 : 1)));
    }
    void *k_x8_ptr = k_x8 ? static_cast<char *>(a->k_rot) + k_part_bytes : nullptr;
    void *v16_ptr = k_x8 ? static_cast<char *>(a->k_rot) + 2 * k_part_bytes : nullptr;
    const bool k_from_rot = rotate_k_once && !rot_shared;   // k itself read from k_rot
    const void *kptr = k_from_rot ? a->k_rot : a->k;
    const int64_t *kst = k_from_rot ? kst_rot : a->k_strides;

    memset(&x, 0, sizeof(x));
    x.rotate_k_once = rotate_k_once;
    x.k_x8 = k_x8_ptr;
    x.v16 = v16_ptr;
    x.v_src = a->v;
    for (int d = 0; d < 4; ++d) x.v_src_strides[d] = a->v_strides[d];
    x.rope = a->rope;
    x.k_src = rot_shared ? a->k_rope : a->k;
    for (int d = 0; d < 4; ++d)
        x.k_src_strides[d] = rot_shared ? a->k_rope_strides[d] : a->k_strides[d];
    x.rot_h = int(rot_h);
    x.rot_d = int(rot_d);
    x.k_rot = rotate_k_once ? a->k_rot : nullptr;
    AttnParams &p = x.p;
    p.q = static_cast<const char *>(a->q);
    p.k = static_cast<const char *>(kptr);
    p.v = static_cast<const char *>(a->v);
    p.o = static_cast<char *>(a->o);
    p.lse = a->lse;
    p.status = a->dev_status;
    for (int d = 0; d < 3; ++d) {
        p.qs[d] = a->q_strides[d];
        p.ks[d] = kst[d];
        p.vs[d] = a->v_strides[d];
        p.os[d] = a->o_strides[d];
    }
    p.B = int(a->B);
    p.Hq = int(a->Hq);
    p.Hkv = int(a->Hkv);
    p.L = int(a->L);
    p.Lk = int(Lk);
    p.qoff = int(a->q_offset);
    p.G = int(a->Hq / a->Hkv);
    p.causal = a->causal;
    // A window of Lk or more keys, or Lk sinks, no longer restricts anything.
    p.window = int(a->window > Lk ? Lk : a->window);
    p.sinks = int(a->sinks > Lk ? Lk : a->sinks);
    // Two query heads share a CTA's K/V tiles when the group allows it and the
    // CTA holds two query tiles (at D = 192 only with LCX_D192_TWO_TILES; never
    // in the split mode, whose CTA holds one tile with two S buffers); with an
    // odd group the two tiles are consecutive query blocks of one head.
    const bool two_tiles =
        (a->D <= 128 || LCX_D192_TWO_TILES) && !(a->flags & LCX_ATTN_SPLIT_QK);
    // Pairs only when the paired units still fill the GPU: a problem of few
    // query blocks (the tiny workload is one pair) runs faster spread over
    // twice the CTAs, one query tile each.
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sms = 148;
    const int64_t paired_units =
        p.G % 2 == 0 ? (a->L + kBM - 1) / kBM * (a->B * a->Hq / 2)
                     : (a->L + 2 * kBM - 1) / (2 * kBM) * (a->B * a->Hq);
    const bool pair = two_tiles && paired_units >= sms;
    p.heads_per_unit = (p.G % 2 == 0 && pair) ? 2 : 1;
    p.qpair = (p.G % 2 == 1 && pair) ? 1 : 0;
    p.n_qb = int((a->L + (p.qpair ? 2 * kBM : kBM) - 1) / (p.qpair ? 2 * kBM : kBM));
    p.units_per_qb = p.B * p.Hq / p.heads_per_unit;
    p.n_split = 1;
    x.units = (long long)p.n_qb * p.units_per_qb;
    if (x.units > 0x7fffffffLL) return fail(LCX_ERR_UNSUPPORTED, "too many work units");
    x.sms = sms;
    p.rotate_q = (a->flags & LCX_ATTN_PREROTATED) ? 0 : 1;
    p.rotate_k = (rotate_k_once || (a->flags & (LCX_ATTN_PREROTATED | LCX_ATTN_PREROTATED_K)))
                     ? 0 : 1;
    float ms = 1.f;
    // The length-dependent modes see the whole context: the Lk keys.
    rope_table_unchecked(&a->rope, effective_seq_len(&a->rope, Lk), p.theta, &ms);
    const double scale = a->softmax_scale > 0.f ? double(a->softmax_scale) : 1.0 / std::sqrt(double(a->D));
    double msq = 1.0;
    p.rot_ms = 1.f;
    if (!partial) {
        // Each operand rotated on chip contributes its mscale factor to the
        // logits (pre-rotated operands already carry theirs): folded into the
        // logit scale.
        msq = (p.rotate_q ? double(ms) : 1.0) * (p.rotate_k ? double(ms) : 1.0);
    } else {
        // Only the rotated dims carry mscale: applied to the rotated values.
        p.rot_ms = ms;
    }
    p.c_log2 = float(scale * msq * 1.4426950408889634);
    p.k_rope_shared = a->k_rope ? 1 : 0;
    p.k_x8_tma = k_x8 ? 1 : 0;
    p.v_f16 = v16_ptr ? 1 : 0;
    // Split QK^T with the key parts and V from the rotate pass at D = 128: a
    // CTA per SM takes its units one after the other, the next unit's query
    // tile loaded, rotated and copied to TMEM while the current one finishes
    // (cleared again for key-split launches).
    p.n_units = int(x.units);
    p.persist = ((a->flags & LCX_ATTN_SPLIT_QK) && a->dtype == LCX_BF16 && a->D == 128 &&
                 v16_ptr && !(a->flags & LCX_ATTN_TEST_STALL) && x.units > sms) ? 1 : 0;
    // Legitimate waits last microseconds; the default limit is 2 s.
    p.timeout_ns = 1000000ull * (unsigned long long)(a->watchdog_ms > 0 ? a->watchdog_ms : 2000);
    p.test_stall = (a->flags & LCX_ATTN_TEST_STALL) ? 1 : 0;

    x.split_qk = (a->flags & LCX_ATTN_SPLIT_QK) != 0;
    x.f32 = a->dtype == LCX_F32;
    x.half = a->rope.pairing == LCX_PAIR_HALF;
    x.D = int(a->D);
    x.DV = int(Dv);
    x.RD = int(RD);
    // K/V boxes are one key tile high: the kernel's expect-tx byte counts and
    // stage layout assume exactly Cfg::BN rows per box.
    const uint32_t bn = uint32_t(Cfg<64, 64, false>::BN);
    static_assert(Cfg<64, 64, true>::BN == Cfg<64, 64, false>::BN &&
                      Cfg<128, 128, true>::BN == Cfg<64, 64, false>::BN &&
                      Cfg<128, 128, false>::BN == Cfg<64, 64, false>::BN &&
                      Cfg<192, 128, false>::BN == Cfg<64, 64, false>::BN,
                  "one key-tile height for every kernel instance");
    if (!x.f32) {
        const int64_t dk = a->k_rope ? a->D - RD : a->D;   // columns k itself holds
        if ((st = make_map(&x.m.q, a->q, a->B, a->Hq, a->L, a->D, a->q_strides, 128, "q")) != LCX_OK)
            return st;
        if ((st = make_map(&x.m.k, kptr, a->B, a->Hkv, Lk, dk, kst, bn, "k")) != LCX_OK)
            return st;
        // V, or (split mode with the key buffer) its contiguous fp16 copy
        const int64_t v16_st[4] = {a->Hkv * Lk * Dv, Lk * Dv, Dv, 1};
        if ((st = make_map(&x.m.v, v16_ptr ? v16_ptr : a->v, a->B, a->Hkv, Lk, Dv,
                           v16_ptr ? v16_st : a->v_strides, bn, "v")) != LCX_OK)
            return st;
        if (k_x8) {
            // the keys' 8-bit cross parts: [B, Hkv, Lk, 2 D] bytes, boxes of
            // 128 bytes x one key tile
            const int64_t bst[4] = {kst_rot[0] * 2, kst_rot[1] * 2, kst_rot[2] * 2, 1};
            if ((st = make_map(&x.m.kr, k_x8_ptr, a->B, a->Hkv, Lk, 2 * a->D, bst, bn, "k_x8",
                               1)) != LCX_OK)
                return st;
        }
        if (a->k_rope) {
            // one head: the head stride never matters, any valid value will do;
            // rotated once, the shared key is read from k_rot
            const void *kr = rot_shared && rotate_k_once ? a->k_rot : a->k_rope;
            int64_t krs[4] = {a->k_rope_strides[0], Lk * RD, a->k_rope_strides[2], 1};
            if (rot_shared && rotate_k_once) {
                krs[0] = kst_rot[0];
                krs[2] = kst_rot[2];
            }
            if ((st = make_map(&x.m.kr, kr, a->B, 1, Lk, RD, krs, bn, "k_rope")) != LCX_OK)
                return st;
        }
    }
    return LCX_OK;
}

// Launch the attention kernel described by x (x.p.n_split CTAs per unit).
lcx_status attn_enqueue(const AttnLaunch &x, cudaStream_t s) {
    const long long grid =
        x.p.persist ? std::min<long long>(x.units, x.sms) : x.units * x.p.n_split;
    if (grid > 0x7fffffffLL) return fail(LCX_ERR_UNSUPPORTED, "too many work units");
    if (x.rotate_k_once) {
        // the rotate pass over all keys (positions 0..Lk-1), same stream first
        lcx_rope_params rp = x.rope;
        if (rp.seq_len <= 0) rp.seq_len = x.p.Lk;   // the context of the call, as the kernel's
        const int64_t kst[4] = {(int64_t)x.rot_h * x.p.Lk * x.rot_d, (int64_t)x.p.Lk * x.rot_d,
                                x.rot_d, 1};
        lcx_status st =
            apply_rope_impl(&rp, x.k_src, x.k_rot, x.k_x8, x.f32 ? LCX_F32 : LCX_BF16, x.p.B,
                            x.rot_h, x.p.Lk, x.k_src_strides, kst, 0, s);
        if (st != LCX_OK) return st;
        if (x.v16) {
            st = bf16_to_f16_impl(x.v_src, x.v_src_strides, x.v16, x.p.B, x.p.Hkv, x.p.Lk, x.DV, s);
            if (st != LCX_OK) return st;
        }
    }
    const unsigned g = unsigned(grid);
    if (x.decode) {
        const int nq = x.p.G * x.p.L;
        if (x.split_qk)
            return x.half ? launch_decode_nq<true, true>(nq, x.m, x.p, g, s)
                          : launch_decode_nq<false, true>(nq, x.m, x.p, g, s);
        return x.half ? launch_decode_nq<true, false>(nq, x.m, x.p, g, s)
                      : launch_decode_nq<false, false>(nq, x.m, x.p, g, s);
    }
    return x.p.n_split > 1 ? launch_shape<true>(x, x.m, x.p, g, s)
                           : launch_shape<false>(x, x.m, x.p, g, s);
}

constexpr int kMaxKvSplits = 256;
constexpr int64_t kMaxSplitRows = int64_t(1) << 40;  // keeps workspace sizes far from overflow

// Workspace of the split path: the partial o block then the partial lse block,
// each starting on a 256-byte boundary.
int64_t split_o_bytes(int64_t rows, int64_t D, int64_t n) {
    return ((n * rows * D * 4) + 255) / 256 * 256;
}
int64_t split_ws_bytes(int64_t rows, int64_t D, int64_t n) {
    return split_o_bytes(rows, D, n) + ((n * rows * 4) + 255) / 256 * 256;
}

}  // namespace
}  // namespace lcx

extern "C" lcx_status lcx_attn_fwd(const lcx_attn_args *a, void *stream) {
    using namespace lcx;
    clear_error();
    AttnLaunch x;
    bool noop = false;
    lcx_status st = attn_prepare(a, x, &noop);
    if (st != LCX_OK || noop) return st;
    return attn_enqueue(x, static_cast<cudaStream_t>(stream));
}

extern "C" int64_t lcx_attn_split_workspace_bytes(int64_t B, int64_t Hq, int64_t L, int64_t D,
                                                  int32_t num_splits) {
    if (B < 0 || Hq < 0 || L < 0 || (D != 64 && D != 128) || num_splits < 1 ||
        num_splits > lcx::kMaxKvSplits || B > (int64_t(1) << 20) || Hq > 65536 ||
        L > (int64_t(1) << 30) || B * Hq > (int64_t(1) << 30) ||
        B * Hq * L > lcx::kMaxSplitRows)
        return -1;
    if (num_splits == 1) return 0;
    // room for two partial results per split (head-packed launches write one
    // per query tile)
    return lcx::split_ws_bytes(B * Hq * L, D, 2 * int64_t(num_splits));
}

extern "C" lcx_status lcx_attn_fwd_split(const lcx_attn_args *a, int32_t num_splits,
                                         void *workspace, int64_t workspace_bytes, void *stream) {
    using namespace lcx;
    clear_error();
    if (num_splits < 1 || num_splits > kMaxKvSplits)
        return fail(LCX_ERR_INVALID_ARG, "num_splits must be in [1, %d]", kMaxKvSplits);
    AttnLaunch x;
    bool noop = false;
    lcx_status st = attn_prepare(a, x, &noop);
    if (st != LCX_OK || noop) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (num_splits == 1) return attn_enqueue(x, s);
    const int64_t rows = a->B * a->Hq * a->L;
    if (rows > kMaxSplitRows) return fail(LCX_ERR_UNSUPPORTED, "too many query rows to split");
    const int64_t need = split_ws_bytes(rows, x.DV, 2 * int64_t(num_splits));
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(LCX_ERR_INVALID_ARG, "workspace must be a 256-byte aligned device pointer");
    if (workspace_bytes < need)
        return fail(LCX_ERR_INVALID_ARG, "workspace holds %lld bytes; %lld needed",
                    (long long)workspace_bytes, (long long)need);
    float *part_o = static_cast<float *>(workspace);
    float *part_lse = reinterpret_cast<float *>(
        static_cast<char *>(workspace) + split_o_bytes(rows, x.DV, 2 * int64_t(num_splits)));
    x.p.n_split = num_splits;
    x.p.split_recip = std::nextafter(1.0f / float(num_splits), 2.0f);
    x.p.persist = 0;
    // Head-packed query tiles: with few queries per head (decode, short chunks)
    // the G heads of a kv group share the CTA's query tiles (pack_lp rows per
    // head: L rounded up to 8 rows), so every K/V tile is read and rotated once
    // per kv group instead of once per head pair.
    //  - bf16, G pack_lp <= 128: both tiles hold all G heads (rows
    //    [0, G pack_lp), tile 1 shifted by whole warps when that fits, so the
    //    busy softmax warps of the two tiles use different SMSPs) and tile t
    //    takes the key tiles j = t mod 2: two K/V tiles in flight per CTA, two
    //    partial results per split.
    //  - otherwise (fp32, or G pack_lp > 128), G even and
    //    G/2 pack_lp <= 128: G/2 heads per tile, both tiles multiply every key
    //    tile.
    //  - split QK^T (one query tile per CTA): all G heads in that tile when
    //    G pack_lp <= 128, its two S buffers walking the key tiles in turn.
    const int64_t lp = (a->L + 7) / 8 * 8;
    int n_parts = num_splits;
    // A kv group's G L queries fit in the columns of one transposed score
    // block (bf16, D = DV = 128, full rotary): the decode kernel, one CTA per
    // (batch, kv group, split), one partial result per split.
    // Split QK^T: with the keys' parts and V in fp16 from the rotate pass.
    x.decode = !x.f32 && x.D == 128 && x.DV == 128 && x.RD == 128 && !x.p.k_rope_shared &&
               int64_t(x.p.G) * a->L <= dec::NQ &&
               (!x.split_qk || (x.p.k_x8_tma && x.p.v_f16));
    if (x.decode) {
        x.p.qpair = 0;
        x.p.heads_per_unit = x.p.G;
        x.p.n_qb = 1;
        x.p.units_per_qb = x.p.B * x.p.Hkv;
        x.units = (long long)x.p.B * x.p.Hkv;
    } else if (x.split_qk) {
        // one query tile per CTA: all G heads in it when they fit
        if (!x.f32 && lp * x.p.G <= kBM) {
            x.p.pack_lp = int(lp);
            x.p.pack_hpt = x.p.G;
            x.p.pack_stride = int(lp);
            x.p.pack_off = 0;
        }
    } else if (!x.f32 && x.D <= 128 && lp * x.p.G <= kBM) {
        const int used = int(lp) * x.p.G;
        x.p.pack_lp = int(lp);
        x.p.pack_hpt = x.p.G;
        x.p.pack_stride = int(lp);
        x.p.pack_off = (used + 31) / 32 * 32;
        if (x.p.pack_off + used > kBM) x.p.pack_off = 0;
        x.p.pack_ilv = 1;
        n_parts = 2 * num_splits;
        // Keys rotated on chip: softmax warps whose 32 rows of their tile (warp
        // w: rows 32 (w % 4) .. + 31 of tile w / 4) hold no query rotate key
        // tiles beside warps 8-11 (four of them, which halves each thread's
        // rows; with fewer idle warps nobody helps).  Not in the split mode,
        // whose rotation warpgroup also converts every V tile to fp16.
        if (x.p.rotate_k && !x.split_qk) {
            int mask = 0, n = 0;
            for (int w = 0; w < 8 && n < 4; ++w) {
                bool any = false;
                for (int r = 32 * (w % 4); r < 32 * (w % 4) + 32 && !any; ++r) {
                    const int rel = r - (w / 4) * x.p.pack_off;
                    any = rel >= 0 && rel < used && rel % x.p.pack_stride < a->L;
                }
                if (!any) {
                    mask |= 1 << w;
                    ++n;
                }
            }
            x.p.rot_help = n == 4 ? mask : 0;
        }
    } else if (!x.f32 && x.p.G % 2 == 0 && x.D <= 128 && lp * (x.p.G / 2) <= kBM) {
        x.p.pack_lp = int(lp);
        x.p.pack_hpt = x.p.G / 2;
        // Heads spread over the tile (multiples of 8 rows keep the 128-byte
        // swizzle phase), and tile 1 shifted by one warp's 32 rows when that
        // still fits, so the busy softmax warps of both tiles use different SMSPs.
        x.p.pack_stride = (kBM / x.p.pack_hpt) / 8 * 8;
        x.p.pack_off = (x.p.pack_stride - x.p.pack_lp >= 32) ? 32 : 0;
    }
    if (x.p.pack_lp) {
        x.p.qpair = 0;
        x.p.heads_per_unit = x.p.G;
        x.p.n_qb = 1;
        x.p.units_per_qb = x.p.B * x.p.Hkv;
        x.units = (long long)x.p.B * x.p.Hkv;
        if ((st = make_map(&x.m.q, a->q, a->B, a->Hq, a->L, a->D, a->q_strides, uint32_t(lp),
                           "q")) != LCX_OK)
            return st;
    }
    x.p.part_o = part_o;
    x.p.part_lse = part_lse;
    if ((st = attn_enqueue(x, s)) != LCX_OK) return st;
    return launch_merge(part_o, part_lse, n_parts, a->B, a->Hq, a->L, x.DV, a->o, a->dtype,
                        a->o_strides, a->lse, s);
}
