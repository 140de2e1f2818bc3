// hv_attn.cu - joint full self-attention with 3D RoPE for B200 (sm_100a).
//
// One persistent, warp-specialised kernel computes, per (batch b, head h),
//   out = softmax(scale * R(Q) R(K)^T, keys < N + valid_b) V
// over the joint sequence [video ; text] ("HunyuanVideo 模型结构与数学原理"
// §5.2 joint attention, §5.5 3D RoPE with the (16, 56, 56) split and
// theta = 256 on video rows only; §9.1: exact attention computed tile by tile
// without materialising the score matrix).
//
// Work unit: (b, h, 256 query rows) = two 128-row Q tiles sharing every K/V
// tile. Per CTA (one per SM, 512 threads = 4 warpgroups):
//   warps 0-3   softmax for Q tile 0 (thread = TMEM lane = query row)
//   warps 4-7   softmax for Q tile 1
//   warps 8-11, 14-15  RoPE: rotate the video rows of each Q/K tile in shared
//               memory right after TMA lands it, then hand it to the tensor
//               core (Q only when the keys arrive rotated)
//   warp  12    TMA producer (Q once per unit, then K/V tiles into a ring)
//   warp  13    TMEM owner and tcgen05.mma issuer
// setmaxnreg moves registers to the softmax warpgroups, which hold a full
// 128-column score row per thread.
// Tensor memory (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each; the
// bf16 probabilities P_i overwrite the first 64 columns of S_i and feed the
// PV MMA straight from TMEM.
//
// Every mbarrier wait is bounded by a %globaltimer budget; when one runs out
// the CTA records the role in a device error word and in a host-visible status
// word, tells the other roles to stop, waits (bounded) for its own copies and
// MMAs in flight, frees its TMEM and returns.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "hv_attn.h"
#include "sm100_ptx.cuh"

namespace hv {

constexpr int D = HV_HEAD_DIM;      // head dim
constexpr int BM = 128;             // query rows per Q tile
constexpr int BN = 128;             // keys per K/V tile
constexpr int QTILES = 2;           // Q tiles per work unit
constexpr int UNIT_ROWS = BM * QTILES;
// K and V tiles share a pool of KV_SLOTS shared-memory tiles: K takes the
// first KST slots and V the next VST (fixed per kernel instantiation). When
// the RoPE warps rotate K, three K stages and one V stage let them work on K
// tiles up to two tiles ahead of the tensor core; pre-rotated keys need no
// lead and keep two of each.
constexpr int KV_SLOTS = 4;
constexpr int KSTAGES_MAX = 3;
constexpr int VSTAGES_MAX = 2;
constexpr int KSTAGES_ROPE = 3, VSTAGES_ROPE = 1;
constexpr int KSTAGES_ROTATED = 2, VSTAGES_ROTATED = 2;
static_assert(KSTAGES_ROPE + VSTAGES_ROPE <= KV_SLOTS && KSTAGES_ROTATED + VSTAGES_ROTATED <= KV_SLOTS, "KV pool");
static_assert(KSTAGES_ROPE <= KSTAGES_MAX && KSTAGES_ROTATED <= KSTAGES_MAX, "K stages");
static_assert(VSTAGES_ROPE <= VSTAGES_MAX && VSTAGES_ROTATED <= VSTAGES_MAX, "V stages");
constexpr int BOX_BYTES = 128 * 64 * 2;   // 128 rows x 64 channels bf16, 128B-swizzled
constexpr int TILE_BYTES = 2 * BOX_BYTES; // 128 rows x 128 channels

constexpr int NUM_WARPS = 16;
constexpr int NUM_THREADS = NUM_WARPS * 32;
constexpr int WARP_ROPE = 8;
constexpr int WARP_TMA = 12;
constexpr int WARP_MMA = 13;
// RoPE runs on warpgroup 2 (warps 8-11) and on the two control-warpgroup
// warps that neither load nor issue MMAs (warps 14-15).
constexpr int ROPE_THREADS = 192;
constexpr int ROPE_WARPS = ROPE_THREADS / 32;
constexpr int ROPE_GROUPS = ROPE_THREADS / 16;   // rows rb, rb + 12, rb + 24, ... per thread
// per-thread registers after setmaxnreg: 2 x 128 x 176 + 128 x 64 + 128 x 96
// = 65536 = 512 threads x 128 registers at launch. With the QK RMSNorm
// prologue the RoPE warps carry the normalisation too and take 80, the
// control warpgroup 80.
constexpr uint32_t REGS_SOFTMAX = 176;
__host__ __device__ constexpr uint32_t regs_rope(bool qkn) { return qkn ? 80u : 64u; }
__host__ __device__ constexpr uint32_t regs_control(bool qkn) { return qkn ? 80u : 96u; }
__host__ __device__ constexpr uint32_t regs_split(bool qkn) { return 2 * 128 * REGS_SOFTMAX + 128 * regs_rope(qkn) + 128 * regs_control(qkn); }
static_assert(regs_split(false) <= NUM_WARPS * 32 * 128 && regs_split(true) <= NUM_WARPS * 32 * 128,
              "register split exceeds the launch allocation");

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int OFF_Q = 0;
constexpr int OFF_KV = OFF_Q + QTILES * TILE_BYTES;
// cos/sin table of the rotation angles: a cos and a sin per (axis, position,
// pair) = 8*T + 28*(Hp + Wp) entries of 8 bytes, built once per CTA.
constexpr int OFF_TABLE = OFF_KV + KV_SLOTS * TILE_BYTES;
// 3840 entries cover every size of the pages' supported-size table (720p
// needs 3764); larger grids compute (cos, sin) per pair instead.
constexpr int TABLE_MAX_ENTRIES = 3840;
// QK RMSNorm gammas (fp32 [4][128]: Q video, K video, Q text, K text), copied
// in at kernel start when the prologue is on.
constexpr int OFF_GAMMA = OFF_TABLE + TABLE_MAX_ENTRIES * 8;
constexpr int GAMMA_BYTES = 4 * D * 4;
constexpr int OFF_BAR = OFF_GAMMA + GAMMA_BYTES;
// barrier indices
constexpr int B_Q_FULL = 0, B_Q_READY = 1, B_Q_EMPTY = 2;
constexpr int B_K_FULL = 3;
constexpr int B_K_READY = B_K_FULL + KSTAGES_MAX;
constexpr int B_K_EMPTY = B_K_READY + KSTAGES_MAX;
constexpr int B_V_FULL = B_K_EMPTY + KSTAGES_MAX;
constexpr int B_V_EMPTY = B_V_FULL + VSTAGES_MAX;
constexpr int B_S_FULL = B_V_EMPTY + VSTAGES_MAX;
constexpr int B_P_READY = B_S_FULL + QTILES;
constexpr int B_O_DONE = B_P_READY + QTILES;
constexpr int B_DRAIN = B_O_DONE + QTILES;
constexpr int NUM_BARS = B_DRAIN + 1;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
// 1/rms of the 128 rows of each K stage (QK RMSNorm with per-row statistics)
constexpr int KR_BYTES = BN * 4;
constexpr int OFF_KR = (OFF_MISC + 16 + 127) & ~127;
constexpr int SMEM_USED = OFF_KR + KSTAGES_MAX * KR_BYTES;
constexpr int SMEM_BYTES = SMEM_USED + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory over the sm_100 per-block limit");

constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_S = 0;     // + 128*i
constexpr uint32_t TM_O = 256;   // + 128*i

constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, false);  // Q (K-major) x K (K-major)
constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, true);    // P (TMEM)    x V (MN-major)

// rescale O only when a row max grows by more than this (log2 units)
constexpr float RESCALE_THRESHOLD = 8.0f;

enum Role : uint32_t { ROLE_TMA = 1, ROLE_MMA = 2, ROLE_SOFTMAX = 3, ROLE_ROPE = 4, ROLE_SELFTEST = 5 };

struct __align__(64) Params {
    CUtensorMap tm_q;
    CUtensorMap tm_k;
    CUtensorMap tm_v;
    void* out;          // bf16 [B, S, H, 128], or fp32 when out_f32
    int B, H, S, N, T, Hp, Wp, HpWp;
    int use_table;      // 1: cos/sin from the shared-memory table, 0: sincospif per pair
    float qk_eps;       // RMSNorm epsilon
    const float* qk_gamma;   // device, fp32 [4][128]: Q video, K video, Q text, K text
    // Optional, with the QK RMSNorm: 1/rms of every K row, fp32 [B, H, k_rinv_ld]
    // (k_rinv_ld a multiple of 128, entries past the rows 0), computed once
    // per call by hv_k_rinv_kernel; the producer copies each K tile's 128
    // values beside it and the RoPE warps scale by them instead of reducing
    // every row again for every unit.
    const float* k_rinv;
    int k_rinv_ld;
    int n_qunits;       // ceil(S / 256)
    int units;          // B * H * n_qunits
    float theta_log2;   // log2(rope_theta)
    float scale_log2;   // scale * log2(e)
    unsigned long long timeout_ns;
    unsigned int* status;   // host-visible status word (mapped pinned memory) or nullptr
    int withhold_k;     // test hook: CTA 0 skips its K load number withhold_k (-1: off)
    // place of this launch's heads in the whole call (a call split into head
    // groups launches heads h_offset .. h_offset + H - 1 of h_total), and the
    // round width of the traversal-direction rule (the device's SM count)
    int h_total, h_offset, round_width;
    // Geometry of the row blocks. The standard call: Q and K/V are the whole
    // joint sequence (Sk = S, q_vid = k_vid = N, offsets 0). A ring-attention
    // block: Q rows and K/V rows are runs of the joint sequence whose first
    // q_vid / k_vid rows are video tokens with global token indices starting
    // at q_pos0 / k_pos0; the other rows are text.
    int Sk;             // rows of the K and V tensors (S: rows of Q and out)
    int q_vid, q_pos0, k_vid, k_pos0;
    int out_f32;        // 1: out rows are fp32 (ring-attention partial results)
    float* lse;         // optional [B, S, H] fp32: natural-log log-sum-exp of each row's scaled scores
    int kv_len[HV_MAX_BATCH];   // keys taking part, per batch sample (the rest are masked)
};

__device__ unsigned int g_dev_error = 0;

struct Waiter {
    volatile int* abort_flag;
    unsigned long long timeout_ns;
    unsigned int* status;
    bool record = true;   // false for the bounded drains of an abort already recorded

    // Record a wait that ran out in the error words, and stop every role of
    // the CTA at its next wait.
    __device__ __forceinline__ void fail(uint32_t role) const {
        *abort_flag = 1;
        if (!record) return;
        const uint32_t word = 1u | (role << 8);
        atomicOr(&g_dev_error, word);
        if (status != nullptr) st_sys_u32(status, word);
        __threadfence_block();
    }

    // Spin until the phase of `bar` with `parity` has completed. Returns false
    // when the CTA is aborting (this wait ran out, or another role's did).
    __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity, uint32_t role) const {
        if (mbar_try_wait(bar, parity)) return true;
        const uint64_t t0 = global_timer_ns();
        while (true) {
            if (mbar_try_wait(bar, parity)) return true;
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > timeout_ns) {
                fail(role);
                return false;
            }
        }
    }
    // Warp-wide version: lane 0 waits, the result is broadcast and the
    // warp synchronises, so the other lanes are ordered after the wait
    // without each polling the barrier.
    __device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, uint32_t role) const {
        int ok = 1;
        if ((threadIdx.x & 31) == 0) ok = wait(bar, parity, role) ? 1 : 0;
        return __shfl_sync(0xffffffffu, ok, 0) != 0;
    }
};

// Position in a ring of n stages: the stage in use and the parity of its
// current fill (flips each time the ring wraps).
// Cursor over a ring of N stages: stage s, and the mbarrier phase parity of
// the current pass over the ring.
template <uint32_t N>
struct Ring {
    uint32_t s = 0, ph = 0;
    __device__ __forceinline__ void next() {
        if constexpr (N == 1) {
            ph ^= 1u;
        } else if (++s == N) {
            s = 0;
            ph ^= 1u;
        }
    }
};

struct UnitCoord {
    int b, h, qu, nt, last_lim;
    int rev;   // 1: this unit walks the K/V tiles from the last to the first
    // K/V tile visited at step j of the unit's loop
    __device__ __forceinline__ int tile(int j) const { return rev ? nt - 1 - j : j; }
};

// Units are dealt to the CTAs round-robin, head-major, so the CTAs of one
// round share a head's K/V through L2. Consecutive rounds walk the K/V tiles
// in opposite directions: a CTA starting its next unit begins on the tiles it
// (and the rest of the round) read last, which are still in L2. The
// direction is a function of the unit's place in the whole call (its global
// unit number over a fixed round width), so a call split into launches over
// head groups sums in the same order and gives the same bits.
__device__ __forceinline__ UnitCoord decode_unit(const Params& p, int u) {
    UnitCoord c;
    c.qu = u % p.n_qunits;
    const int bh = u / p.n_qunits;
    c.h = bh % p.H;
    c.b = bh / p.H;
    const int kv_len = p.kv_len[c.b];
    c.nt = (kv_len + BN - 1) / BN;
    c.last_lim = kv_len - (c.nt - 1) * BN;
    // < B * heads * ceil(S / 256) <= 2^24 (S * heads * 128 < 2^31, B <= 512): fits an int
    const int ug = (c.b * p.h_total + p.h_offset + c.h) * p.n_qunits + c.qu;
    c.rev = (ug / p.round_width) & 1;
    return c;
}

// Rotate the video rows (sequence index < N) of one tile of ROWS rows (two
// boxes of 64 channels) in place.
// Thread `rt` (0..191) owns 16-byte chunk cc = rt % 16 of rows rt/16 + 12k.
// A chunk holds channels [8cc, 8cc+8): four adjacent pairs, all inside one
// axis segment because the segment borders 16 and 72 are multiples of 8.
// Axis t: channels [0,16), 8 pairs; h: [16,72), 28 pairs; w: [72,128), 28 pairs.
struct RopeLane {
    int box, cin, axis;
    int ch0;           // first of the chunk's 8 channels
    int i0;            // first pair index of the chunk inside its axis segment
    int half_dim;      // pairs in the axis segment (8 or 28)
    int table_base;    // first table float of the axis segment
};

// Angles are passed to sincospif in units of pi: sin(pi*x) needs no
// argument reduction beyond taking x modulo 2.
constexpr float kInvPi = 0.318309886183790672f;

__device__ __forceinline__ float axis_freq(int i, int dax, float theta_log2) {
    // theta^(-2i/d) = 2^(-(2i/d) * log2(theta))
    return exp2f(__fdiv_rn(__fmul_rn(-static_cast<float>(2 * i), theta_log2), static_cast<float>(dax)));
}

// The angle pos * theta^(-2i/d) in units of pi, for sincospif.
__device__ __forceinline__ float angle_over_pi(int pos, int i, int dax, float theta_log2) {
    return __fmul_rn(__fmul_rn(static_cast<float>(pos), axis_freq(i, dax, theta_log2)), kInvPi);
}

__device__ __forceinline__ RopeLane make_rope_lane(int rt, const Params& p) {
    RopeLane L;
    const int cc = rt & 15;
    L.box = cc >> 3;
    L.cin = cc & 7;
    const int ch0 = cc * 8;
    L.ch0 = ch0;
    int dax;
    if (ch0 < 16) {
        L.axis = 0; L.i0 = ch0 / 2; dax = 16; L.table_base = 0;
    } else if (ch0 < 72) {
        L.axis = 1; L.i0 = (ch0 - 16) / 2; dax = 56; L.table_base = 16 * p.T;
    } else {
        L.axis = 2; L.i0 = (ch0 - 72) / 2; dax = 56; L.table_base = 16 * p.T + 56 * p.Hp;
    }
    L.half_dim = dax / 2;
    return L;
}

// Fill the rotation table. Per axis segment (pairs P = 8, 28, 28) and per
// position pos it holds P cosines then P sines: float f = base + pos*2P + k
// is cos (k < P) or sin (k >= P) of pos * theta^(-2i/d_a), i = k mod P.
// Cosines and sines in separate runs let a chunk's four of each be read
// with one 16-byte load, and neighbouring chunks hit neighbouring banks.
__device__ __forceinline__ void build_rope_table(float* table, const Params& p) {
    const int n_t = 16 * p.T, n_h = 56 * p.Hp, n_w = 56 * p.Wp;
    for (int f = threadIdx.x; f < n_t + n_h + n_w; f += blockDim.x) {
        int pos, k, half, dax;
        if (f < n_t) {
            pos = f / 16; k = f % 16; half = 8; dax = 16;
        } else if (f < n_t + n_h) {
            pos = (f - n_t) / 56; k = (f - n_t) % 56; half = 28; dax = 56;
        } else {
            pos = (f - n_t - n_h) / 56; k = (f - n_t - n_h) % 56; half = 28; dax = 56;
        }
        const int i = k < half ? k : k - half;
        float sn, cs;
        sincospif(angle_over_pi(pos, i, dax, p.theta_log2), &sn, &cs);
        table[f] = k < half ? cs : sn;
    }
}

// Explicitly rounded operations (no contraction choices left to the
// compiler), so that every kernel rotating a pair gets the same bits.
__device__ __forceinline__ uint32_t rotate_f(float x0, float x1, float cs, float sn) {
    const float y0 = __fmaf_rn(x0, cs, -__fmul_rn(x1, sn));
    const float y1 = __fmaf_rn(x0, sn, __fmul_rn(x1, cs));
    return pack_bf16x2(y0, y1);
}

__device__ __forceinline__ uint32_t rotate_pair(uint32_t w, float cs, float sn) {
    // channel 2i in the low half, 2i+1 in the high half
    return rotate_f(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u), cs, sn);
}

// QK RMSNorm of one row ("HunyuanVideo 模型结构与数学原理" §5.4):
// y = gamma * x / sqrt(mean_j x_j^2 + eps) over the 128 channels. The row's 16
// chunks of 8 channels sit in the 16 lanes of one half-warp (lane & 15 =
// chunk). The sum of squares is taken in a fixed order (channel order inside
// a chunk, then a butterfly over the half-warp), so every kernel that
// normalises a row this way gets the same bits.
__device__ __forceinline__ void unpack_bf16x8(uint4 d, float (&x)[8]) {
    const uint32_t w[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        x[2 * q] = __uint_as_float(w[q] << 16);
        x[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
    }
}

// 1/rms of the row: every lane of the warp must call this together.
__device__ __forceinline__ float row_rms_inv(uint4 d, float eps) {
    float x[8];
    unpack_bf16x8(d, x);
    float ss = __fmul_rn(x[0], x[0]);
#pragma unroll
    for (int c = 1; c < 8; ++c) ss = __fmaf_rn(x[c], x[c], ss);
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
    return rsqrtf(__fmaf_rn(ss, 1.f / D, eps));
}

// y = (x * r) * gamma for the chunk's eight channels, two at a time.
__device__ __forceinline__ void rms_scale_chunk(uint4 d, float r, uint4 g0, uint4 g1, float (&y)[8]) {
    float x[8];
    unpack_bf16x8(d, x);
    const uint32_t g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
    for (int c = 0; c < 8; c += 2) {
        float t0, t1;
        fmul2(t0, t1, x[c], x[c + 1], r, r);
        fmul2(y[c], y[c + 1], t0, t1, __uint_as_float(g[c]), __uint_as_float(g[c + 1]));
    }
}

__device__ __forceinline__ void rms_norm_chunk(uint4 d, uint4 g0, uint4 g1, float eps, float (&y)[8]) {
    rms_scale_chunk(d, row_rms_inv(d, eps), g0, g1, y);
}

__device__ __forceinline__ uint4 rotate_chunk(uint4 d, uint4 c, uint4 sn) {
    d.x = rotate_pair(d.x, __uint_as_float(c.x), __uint_as_float(sn.x));
    d.y = rotate_pair(d.y, __uint_as_float(c.y), __uint_as_float(sn.y));
    d.z = rotate_pair(d.z, __uint_as_float(c.z), __uint_as_float(sn.z));
    d.w = rotate_pair(d.w, __uint_as_float(c.w), __uint_as_float(sn.w));
    return d;
}

struct GridPos {
    int t, h, w;
};

// Move a token ROPE_GROUPS positions further along the flattened (t, h, w) grid.
__device__ __forceinline__ void advance8(GridPos& g, const Params& p) {
    g.w += ROPE_GROUPS;
    while (g.w >= p.Wp) {
        g.w -= p.Wp;
        if (++g.h == p.Hp) {
            g.h = 0;
            ++g.t;
        }
    }
}

// Rows n0 + rb, n0 + rb + 12, ... of a tile of ROWS rows; sequence rows
// below `vid` are video tokens whose global token index is pos0 + row (the
// rest are text, left as they are).
template <int ROWS, bool TABLE>
__device__ __forceinline__ void rope_tile(uint32_t tile, uint32_t table, int n0, int vid, int pos0, int rt,
                                          const RopeLane& L, const Params& p) {
    const int rb = rt >> 4;
    int n = n0 + rb;
    if (n >= vid || rb >= ROWS) return;
    GridPos g;
    g.w = (pos0 + n) % p.Wp;
    const int th = (pos0 + n) / p.Wp;
    g.h = th % p.Hp;
    g.t = th / p.Hp;
    const uint32_t box_base = tile + L.box * (ROWS * 128);
    auto row_addr = [&](int r) { return box_base + r * 128 + ((L.cin ^ (r & 7)) << 4); };
    const uint32_t sin_off = 4u * static_cast<uint32_t>(L.half_dim);
    const uint32_t tab = table + 4u * static_cast<uint32_t>(L.table_base + L.i0);
    const int stride = 2 * L.half_dim;
    if constexpr (TABLE) {
        // two rows (r, r + ROPE_GROUPS) per iteration so that their loads overlap;
        // the t and h lanes keep the (cos, sin) of their last position and read
        // the table only when it changes (every Hp*Wp or Wp tokens)
        const bool keep = L.axis != 2;
        int kpos = -1;
        uint4 kc = make_uint4(0u, 0u, 0u, 0u), ks = kc;
#pragma unroll 1
        for (int r = rb; r < ROWS; r += 2 * ROPE_GROUPS) {
            const int pos0 = L.axis == 0 ? g.t : (L.axis == 1 ? g.h : g.w);
            const bool has1 = n + ROPE_GROUPS < vid && r + ROPE_GROUPS < ROWS;
            advance8(g, p);
            const int pos1 = L.axis == 0 ? g.t : (L.axis == 1 ? g.h : g.w);
            const uint32_t a0 = row_addr(r);
            const uint32_t a1 = row_addr(r + ROPE_GROUPS);
            const uint32_t t0 = tab + 4u * static_cast<uint32_t>(pos0 * stride);
            const uint32_t t1 = tab + 4u * static_cast<uint32_t>(pos1 * stride);
            const uint4 d0 = lds128(a0);
            uint4 c0 = kc, s0 = ks;
            if (!keep || pos0 != kpos) {
                c0 = lds128(t0);
                s0 = lds128(t0 + sin_off);
            }
            uint4 d1 = d0, c1 = c0, s1 = s0;
            if (has1) {
                d1 = lds128(a1);
                if (!keep || pos1 != pos0) {
                    c1 = lds128(t1);
                    s1 = lds128(t1 + sin_off);
                }
            }
            kpos = has1 ? pos1 : pos0;
            kc = has1 ? c1 : c0;
            ks = has1 ? s1 : s0;
            sts128(a0, rotate_chunk(d0, c0, s0));
            if (!has1) break;
            sts128(a1, rotate_chunk(d1, c1, s1));
            n += 2 * ROPE_GROUPS;
            if (n >= vid) break;   // rows only grow: the rest are text or past the end
            advance8(g, p);
        }
    } else {
#pragma unroll 1
        for (int r = rb; r < ROWS; r += ROPE_GROUPS) {
            const int pos = L.axis == 0 ? g.t : (L.axis == 1 ? g.h : g.w);
            const uint32_t a = row_addr(r);
            uint4 d = lds128(a);
            uint32_t wv[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float sn, cs;
                sincospif(angle_over_pi(pos, L.i0 + q, 2 * L.half_dim, p.theta_log2), &sn, &cs);
                wv[q] = rotate_pair(wv[q], cs, sn);
            }
            sts128(a, make_uint4(wv[0], wv[1], wv[2], wv[3]));
            n += ROPE_GROUPS;
            if (n >= vid) break;
            advance8(g, p);
        }
    }
}

// RMSNorm prologue, then the rotation of the video rows, for every row of a
// tile of ROWS rows (rows rb, rb + 12, ...); text rows and rows past the
// sequence are only normalised (rows past the sequence hold TMA's zero fill
// and stay zero). gamma_v / gamma_t: shared-memory addresses of the video /
// text gamma of this tensor (Q or K). RINV: the tile's 128 row factors 1/rms
// were computed beforehand and sit at shared-memory address k_rinv (K tiles);
// otherwise each row's sum is reduced here, a half-warp shuffle, and every
// lane of a warp runs the same number of iterations (rb and rb + 1 share a
// warp, and as ROWS is even they share a trip count). Separate
// instantiations keep each call site's code to the one it uses.
template <int ROWS, bool TABLE, bool RINV>
__device__ __forceinline__ void rope_norm_tile(uint32_t tile, uint32_t table, uint32_t gamma_v, uint32_t gamma_t,
                                               uint32_t k_rinv, int n0, int vid, int pos0, int rt,
                                               const RopeLane& L, const Params& p) {
    static_assert(ROWS % 2 == 0, "half-warp row pairs");
    const int rb = rt >> 4;
    int n = n0 + rb;
    GridPos g;
    g.w = (pos0 + n) % p.Wp;
    const int th = (pos0 + n) / p.Wp;
    g.h = th % p.Hp;
    g.t = th / p.Hp;
    const uint32_t box_base = tile + L.box * (ROWS * 128);
    const uint32_t sin_off = 4u * static_cast<uint32_t>(L.half_dim);
    const uint32_t tab = table + 4u * static_cast<uint32_t>(L.table_base + L.i0);
    const int stride = 2 * L.half_dim;
    const uint32_t gofs = 4u * static_cast<uint32_t>(L.ch0);
    const uint4 gv0 = lds128(gamma_v + gofs), gv1 = lds128(gamma_v + gofs + 16);
#pragma unroll 1
    for (int r = rb; r < ROWS; r += ROPE_GROUPS) {
        const bool video = n < vid;
        const int pos = L.axis == 0 ? g.t : (L.axis == 1 ? g.h : g.w);
        const uint32_t a = box_base + r * 128 + ((L.cin ^ (r & 7)) << 4);
        const uint4 d = lds128(a);
        uint4 g0 = gv0, g1 = gv1;
        if (!video) {
            g0 = lds128(gamma_t + gofs);
            g1 = lds128(gamma_t + gofs + 16);
        }
        uint4 c = make_uint4(0u, 0u, 0u, 0u), sn = c;
        if (TABLE && video) {
            const uint32_t t = tab + 4u * static_cast<uint32_t>(pos * stride);
            c = lds128(t);
            sn = lds128(t + sin_off);
        }
        float y[8];
        float rr;
        if constexpr (RINV)
            rr = lds_f32(k_rinv + 4u * static_cast<uint32_t>(r));
        else
            rr = row_rms_inv(d, p.qk_eps);
        rms_scale_chunk(d, rr, g0, g1, y);
        uint32_t w[4];
        if (video) {
            if constexpr (TABLE) {
                const float cs[4] = {__uint_as_float(c.x), __uint_as_float(c.y), __uint_as_float(c.z),
                                     __uint_as_float(c.w)};
                const float ss[4] = {__uint_as_float(sn.x), __uint_as_float(sn.y), __uint_as_float(sn.z),
                                     __uint_as_float(sn.w)};
#pragma unroll
                for (int q = 0; q < 4; ++q) w[q] = rotate_f(y[2 * q], y[2 * q + 1], cs[q], ss[q]);
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float s1, c1;
                    sincospif(angle_over_pi(pos, L.i0 + q, 2 * L.half_dim, p.theta_log2), &s1, &c1);
                    w[q] = rotate_f(y[2 * q], y[2 * q + 1], c1, s1);
                }
            }
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) w[q] = pack_bf16x2(y[2 * q], y[2 * q + 1]);
        }
        sts128(a, make_uint4(w[0], w[1], w[2], w[3]));
        n += ROPE_GROUPS;
        advance8(g, p);
    }
}

// The RoPE role: rotate the Q tiles of every unit and every K tile, then hand
// each to the MMA warp.
template <bool BLOCK, bool QKN, bool KROT, bool TABLE>
__device__ __forceinline__ void rope_role(int rt, const Params& p, const Waiter& waiter, uint32_t bars, uint32_t sQ,
                                          uint32_t sK, uint32_t sTable, uint32_t sGamma, uint32_t sKR) {
    const int q_vid = BLOCK ? p.q_vid : p.N, q_pos0 = BLOCK ? p.q_pos0 : 0;
    const int k_vid = BLOCK ? p.k_vid : p.N, k_pos0 = BLOCK ? p.k_pos0 : 0;
    const RopeLane L = make_rope_lane(rt, p);
    const int lane = threadIdx.x & 31;
    auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
    Ring<KSTAGES_ROPE> kr;
    uint32_t lu = 0;
    for (int u = blockIdx.x; u < p.units; u += gridDim.x, ++lu) {
        const UnitCoord c = decode_unit(p, u);
        // every lane tests the barriers itself (a lane-0 wait and a broadcast cost more)
        if (!waiter.wait(bar(B_Q_FULL), lu & 1, ROLE_ROPE)) break;
        for (int qi = 0; qi < QTILES; ++qi) {
            const int n0 = c.qu * UNIT_ROWS + qi * BM;
            if constexpr (QKN)
                rope_norm_tile<BM, TABLE, false>(sQ + qi * TILE_BYTES, sTable, sGamma, sGamma + 2 * D * 4, 0u, n0, q_vid, q_pos0,
                                   rt, L, p);
            else
                rope_tile<BM, TABLE>(sQ + qi * TILE_BYTES, sTable, n0, q_vid, q_pos0, rt, L, p);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_Q_READY));
        // with KROT the keys arrive rotated: the MMA warp takes them straight from TMA
        if constexpr (!KROT) {
            bool ok = true;
            for (int j = 0; j < c.nt; ++j, kr.next()) {
                if (!(ok = waiter.wait(bar(B_K_FULL + kr.s), kr.ph, ROLE_ROPE))) break;
                const int k0 = c.tile(j) * BN;
                if constexpr (QKN)   // keys normalised on load always come with their row factors
                    rope_norm_tile<BN, TABLE, true>(sK + kr.s * TILE_BYTES, sTable, sGamma + D * 4,
                                                    sGamma + 3 * D * 4, sKR + kr.s * KR_BYTES, k0, k_vid, k_pos0,
                                                    rt, L, p);
                else if (k0 < k_vid)
                    rope_tile<BN, TABLE>(sK + kr.s * TILE_BYTES, sTable, k0, k_vid, k_pos0, rt, L, p);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_K_READY + kr.s));
            }
            if (!ok) break;
        }
    }
}

// S_i = Q_i K^T: 8 MMAs of K=16 channels; both operands K-major, 128B swizzle.
// q_desc, k_desc: shared-memory descriptors of the tiles' first 16 channels.
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint64_t q_desc, uint64_t k_desc) {
    mma_ss_k128<BOX_BYTES / 16>(d_tmem, q_desc, k_desc, IDESC_QK, 0u);
}

// O_i (+)= P_i V: 8 MMAs of K=16 keys; P from TMEM (2 bf16 per column),
// V MN-major (channels contiguous): LBO = distance between the two 64-channel
// boxes, SBO = 8 key rows. v_desc: descriptor of the tile's first 16 keys.
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint64_t v_desc, bool accumulate) {
    mma_ts_k128(d_tmem, p_tmem, v_desc, IDESC_PV, accumulate ? 1u : 0u);
}

// Descriptor of a K-major operand tile (Q or K) and of an MN-major V tile.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile) { return smem_desc_sw128(tile, 16, 1024); }
__device__ __forceinline__ uint64_t v_desc_of(uint32_t tile) { return smem_desc_sw128(tile, BOX_BYTES, 1024); }

// BLOCK: a ring-attention block (Q and K/V rows at their own global offsets,
// log-sum-exp and optionally fp32 output); the standard call is compiled
// without that generality (video rows = the first N rows of both, no offsets).
// QKN: the QK RMSNorm prologue (qk_gamma, qk_eps, optionally k_rinv); a
// kernel of its own, so that the plain call carries none of its code.
// KROT: K holds rotated keys (workspace paths): the RoPE warps rotate Q only
// and the K/V ring is split 2 + 2 instead of 3 + 1. TABLE: (cos, sin) from
// the shared-memory table (p.use_table = 1), else sincospif per pair. Each a
// kernel of its own, for the same reason.
template <bool BLOCK, bool QKN, bool KROT, bool TABLE>
__global__ void __launch_bounds__(NUM_THREADS, 1) hv_attn_fwd_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* base_ptr = smem_raw + (base - raw);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const uint32_t bars = base + OFF_BAR;
    auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + OFF_MISC + 4);

    if (threadIdx.x == 0) {
        mbar_init(bar(B_Q_FULL), 1);
        mbar_init(bar(B_Q_READY), ROPE_WARPS);
        mbar_init(bar(B_Q_EMPTY), 1);
        for (int s = 0; s < KSTAGES_MAX; ++s) {
            mbar_init(bar(B_K_FULL + s), 1);
            mbar_init(bar(B_K_READY + s), ROPE_WARPS);
            mbar_init(bar(B_K_EMPTY + s), 1);
        }
        for (int s = 0; s < VSTAGES_MAX; ++s) {
            mbar_init(bar(B_V_FULL + s), 1);
            mbar_init(bar(B_V_EMPTY + s), 1);
        }
        for (int i = 0; i < QTILES; ++i) {
            mbar_init(bar(B_S_FULL + i), 1);
            mbar_init(bar(B_P_READY + i), 4);
            mbar_init(bar(B_O_DONE + i), 1);
        }
        mbar_init(bar(B_DRAIN), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == WARP_MMA) {
        tmem_alloc(smem_addr(tmem_slot), TMEM_COLS);
        tmem_relinquish();
    }
    if constexpr (TABLE) build_rope_table(reinterpret_cast<float*>(base_ptr + OFF_TABLE), p);
    if constexpr (QKN) {
        float* gdst = reinterpret_cast<float*>(base_ptr + OFF_GAMMA);
        for (int i = threadIdx.x; i < 4 * D; i += blockDim.x) gdst[i] = __ldg(p.qk_gamma + i);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const Waiter waiter{abort_flag, p.timeout_ns, p.status};
    const uint32_t sQ = base + OFF_Q;
    const uint32_t sK = base + OFF_KV;
    constexpr int KST = KROT ? KSTAGES_ROTATED : KSTAGES_ROPE;
    constexpr int VST = KROT ? VSTAGES_ROTATED : VSTAGES_ROPE;
    const uint32_t sV = sK + static_cast<uint32_t>(KST) * TILE_BYTES;
    const uint32_t sTable = base + OFF_TABLE;
    const uint32_t sGamma = base + OFF_GAMMA;
    const uint32_t sKR = base + OFF_KR;

    if (warp >= WARP_TMA) {
      regs_decrease<regs_control(QKN)>();
      if (warp == WARP_TMA) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&p.tm_q);
            tma_prefetch_desc(&p.tm_k);
            tma_prefetch_desc(&p.tm_v);
            // Q tiles are read once per call: evicted from L2 first, so that
            // the K/V tiles every unit re-reads stay there longer
            const uint64_t once = l2_evict_first_policy();
            // Two cursors over this CTA's (unit, tile) sequence: keys (each
            // unit's Q ahead of its first key) run up to KST tiles ahead
            // of the values.
            Ring<KST> kr;
            Ring<VST> vr;
            uint32_t kt = 0, vt = 0, klu = 0;   // K and V tiles issued, units whose Q is issued
            int ku = blockIdx.x, kj = 0, vu = blockIdx.x, vj = 0;
            UnitCoord kc{}, vc{};
            if (ku < p.units) kc = vc = decode_unit(p, ku);
            // stages with a load in flight and the parity it completes (bit per stage)
            uint32_t armed_q = 0, armed_k = 0, armed_v = 0;
            uint32_t par_q = 0, par_k = 0, par_v = 0;
            bool ok = true;
            while (ok && vu < p.units) {
                while (ku < p.units && kt < vt + KST) {
                    if (kj == 0) {
                        // The Q buffer frees when the previous unit's last QK
                        // MMA completes, which needs that unit's values up to
                        // its second-last tile: issue those before waiting.
                        if (kt >= vt + 2) break;
                        if (!(ok = waiter.wait(bar(B_Q_EMPTY), (klu & 1) ^ 1, ROLE_TMA))) break;
                        mbar_arrive_expect_tx(bar(B_Q_FULL), QTILES * TILE_BYTES);
                        armed_q = 1; par_q = klu & 1;
                        for (int qi = 0; qi < QTILES; ++qi)
                            for (int bx = 0; bx < 2; ++bx)
                                tma_load_4d_hint(sQ + qi * TILE_BYTES + bx * BOX_BYTES, &p.tm_q, bar(B_Q_FULL),
                                                 bx * 64, kc.h, kc.qu * UNIT_ROWS + qi * BM, kc.b, once);
                    }
                    if (!(ok = waiter.wait(bar(B_K_EMPTY + kr.s), kr.ph ^ 1, ROLE_TMA))) break;
                    // test hook: CTA 0 leaves one K tile unloaded, so that the
                    // next wait for it runs out
                    if (!(p.withhold_k >= 0 && blockIdx.x == 0 && kt == static_cast<uint32_t>(p.withhold_k))) {
                        mbar_arrive_expect_tx(bar(B_K_FULL + kr.s), p.k_rinv ? TILE_BYTES + KR_BYTES : TILE_BYTES);
                        armed_k |= 1u << kr.s;
                        par_k = (par_k & ~(1u << kr.s)) | (kr.ph << kr.s);
                        for (int bx = 0; bx < 2; ++bx)
                            tma_load_4d(sK + kr.s * TILE_BYTES + bx * BOX_BYTES, &p.tm_k, bar(B_K_FULL + kr.s),
                                        bx * 64, kc.h, kc.tile(kj) * BN, kc.b);
                        if (p.k_rinv) {
                            // the tile's 128 row factors: 512 contiguous bytes, 512-byte aligned
                            const long long row0 = (static_cast<long long>(kc.b) * p.H + kc.h) * p.k_rinv_ld +
                                                   static_cast<long long>(kc.tile(kj)) * BN;
                            bulk_load(sKR + kr.s * KR_BYTES, p.k_rinv + row0, KR_BYTES, bar(B_K_FULL + kr.s));
                        }
                    }
                    kr.next();
                    ++kt;
                    if (++kj == kc.nt) {
                        kj = 0;
                        ++klu;
                        ku += gridDim.x;
                        if (ku < p.units) kc = decode_unit(p, ku);
                    }
                }
                if (!ok) break;
                if (!(ok = waiter.wait(bar(B_V_EMPTY + vr.s), vr.ph ^ 1, ROLE_TMA))) break;
                mbar_arrive_expect_tx(bar(B_V_FULL + vr.s), TILE_BYTES);
                armed_v |= 1u << vr.s;
                par_v = (par_v & ~(1u << vr.s)) | (vr.ph << vr.s);
                for (int bx = 0; bx < 2; ++bx)
                    tma_load_4d(sV + vr.s * TILE_BYTES + bx * BOX_BYTES, &p.tm_v, bar(B_V_FULL + vr.s), bx * 64,
                                vc.h, vc.tile(vj) * BN, vc.b);
                vr.next();
                ++vt;
                if (++vj == vc.nt) {
                    vj = 0;
                    vu += gridDim.x;
                    if (vu < p.units) vc = decode_unit(p, vu);
                }
            }
            if (!ok) {
                // Abort: let every copy this warp started land before the CTA
                // (and its shared memory) goes away.
                volatile int never = 0;
                Waiter tail{&never, 20000000ull, nullptr, false};
                if (armed_q) tail.wait(bar(B_Q_FULL), par_q, ROLE_TMA);
                for (int s = 0; s < KST; ++s)
                    if ((armed_k >> s) & 1u) tail.wait(bar(B_K_FULL + s), (par_k >> s) & 1u, ROLE_TMA);
                for (int s = 0; s < VST; ++s)
                    if ((armed_v >> s) & 1u) tail.wait(bar(B_V_FULL + s), (par_v >> s) & 1u, ROLE_TMA);
            }
        }
      } else if (warp > WARP_MMA) {
        // RoPE helpers: threads 128..191 of the RoPE role
        rope_role<BLOCK, QKN, KROT, TABLE>(128 + threadIdx.x - (WARP_MMA + 1) * 32, p, waiter, bars, sQ, sK, sTable, sGamma, sKR);
      } else if (warp == WARP_MMA) {
        // ------------------------------------------------------------- MMA
        if (lane == 0) {
            // K tiles are ready for the tensor core once the RoPE warps have
            // rotated them, or, when they arrive rotated, once TMA lands them.
            constexpr int k_ready = KROT ? B_K_FULL : B_K_READY;
            // operand descriptors, computed once: the MMAs only add offsets
            // (a stage's tile lies TILE_BYTES / 16 address units after the previous one)
            const uint64_t dq0 = kmajor_desc(sQ), dq1 = kmajor_desc(sQ + TILE_BYTES);
            const uint64_t dk0 = kmajor_desc(sK), dv0 = v_desc_of(sV);
            auto dk = [&](uint32_t st) { return dk0 + static_cast<uint64_t>(st * (TILE_BYTES / 16)); };
            auto dv = [&](uint32_t st) { return dv0 + static_cast<uint64_t>(st * (TILE_BYTES / 16)); };
            Ring<KST> kr;
            Ring<VST> vr;
            uint32_t lu = 0;
            uint32_t pr[QTILES] = {0, 0};
            bool ok = true;
            for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x, ++lu) {
                const UnitCoord c = decode_unit(p, u);
                if (!(ok = waiter.wait(bar(B_Q_READY), lu & 1, ROLE_MMA))) break;
                if (!(ok = waiter.wait(bar(k_ready + kr.s), kr.ph, ROLE_MMA))) break;
                tc_fence_after();
                issue_qk(tmem_base + TM_S + 0, dq0, dk(kr.s));
                mma_commit(bar(B_S_FULL + 0));
                issue_qk(tmem_base + TM_S + 128, dq1, dk(kr.s));
                mma_commit(bar(B_S_FULL + 1));
                mma_commit(bar(B_K_EMPTY + kr.s));
                kr.next();
                if (c.nt == 1) mma_commit(bar(B_Q_EMPTY));
                for (int j = 0; j < c.nt; ++j) {
                    if (!(ok = waiter.wait(bar(B_V_FULL + vr.s), vr.ph, ROLE_MMA))) break;
                    const uint64_t v_d = dv(vr.s);
                    // Q tile 0: PV for tile j, then QK for tile j+1
                    if (!(ok = waiter.wait(bar(B_P_READY + 0), pr[0] & 1, ROLE_MMA))) break;
                    ++pr[0];
                    tc_fence_after();
                    issue_pv(tmem_base + TM_O + 0, tmem_base + TM_S + 0, v_d, j > 0);
                    if (j == c.nt - 1) mma_commit(bar(B_O_DONE + 0));
                    const bool more = j + 1 < c.nt;
                    const uint64_t k_d = dk(kr.s);
                    if (more) {
                        if (!(ok = waiter.wait(bar(k_ready + kr.s), kr.ph, ROLE_MMA))) break;
                        tc_fence_after();
                        issue_qk(tmem_base + TM_S + 0, dq0, k_d);
                        mma_commit(bar(B_S_FULL + 0));
                    }
                    // Q tile 1
                    if (!(ok = waiter.wait(bar(B_P_READY + 1), pr[1] & 1, ROLE_MMA))) break;
                    ++pr[1];
                    tc_fence_after();
                    issue_pv(tmem_base + TM_O + 128, tmem_base + TM_S + 128, v_d, j > 0);
                    mma_commit(bar(B_V_EMPTY + vr.s));
                    vr.next();
                    if (j == c.nt - 1) mma_commit(bar(B_O_DONE + 1));
                    if (more) {
                        issue_qk(tmem_base + TM_S + 128, dq1, k_d);
                        mma_commit(bar(B_S_FULL + 1));
                        mma_commit(bar(B_K_EMPTY + kr.s));
                        kr.next();
                        if (j + 1 == c.nt - 1) mma_commit(bar(B_Q_EMPTY));
                    }
                }
            }
            if (!ok) {
                // Abort: wait for the MMAs already issued before TMEM is freed.
                mma_commit(bar(B_DRAIN));
                volatile int never = 0;
                Waiter tail{&never, 20000000ull, nullptr, false};
                tail.wait(bar(B_DRAIN), 0, ROLE_MMA);
            }
        }
      }
    } else if (warp >= WARP_ROPE) {
        regs_decrease<regs_rope(QKN)>();
        // ------------------------------------------------------------ RoPE
        rope_role<BLOCK, QKN, KROT, TABLE>(threadIdx.x - WARP_ROPE * 32, p, waiter, bars, sQ, sK, sTable, sGamma, sKR);
    } else {
        regs_increase<REGS_SOFTMAX>();
        // --------------------------------------------------------- softmax
        const int qi = warp >> 2;                       // Q tile of this warpgroup
        const int row = ((warp & 3) << 5) + lane;       // = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) << 5) << 16;
        const uint32_t tS = tmem_base + lane_off + TM_S + 128 * qi;
        const uint32_t tO = tmem_base + lane_off + TM_O + 128 * qi;
        const float sl2 = p.scale_log2;
        uint32_t sp = 0, lu = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x, ++lu) {
            const UnitCoord c = decode_unit(p, u);
            float m = -INFINITY;   // running max, scaled log2 units
            float l = 0.f;         // running sum of probabilities
            for (int j = 0; j < c.nt; ++j, ++sp) {
                // every lane tests the barrier itself: no broadcast on the critical path
                if (!(ok = waiter.wait(bar(B_S_FULL + qi), sp & 1, ROLE_SOFTMAX))) break;
                tc_fence_after();
                uint32_t sr[BN];
#pragma unroll
                for (int ch = 0; ch < BN / 32; ++ch) tmem_ld32(tS + 32 * ch, sr + 32 * ch);
                tmem_wait_ld();
#pragma unroll
                for (int ch = 0; ch < BN / 32; ++ch) reg_fence32(sr + 32 * ch);
                if (c.tile(j) == c.nt - 1) {
                    // key mask: columns at or past N + valid in the last tile
#pragma unroll
                    for (int e = 0; e < BN; ++e)
                        if (e >= c.last_lim) sr[e] = __float_as_uint(-INFINITY);
                }
                // row max, two columns per (three-input) max instruction
                float mx0 = fmaxf(__uint_as_float(sr[0]), __uint_as_float(sr[4]));
                float mx1 = fmaxf(__uint_as_float(sr[1]), __uint_as_float(sr[5]));
                float mx2 = fmaxf(__uint_as_float(sr[2]), __uint_as_float(sr[6]));
                float mx3 = fmaxf(__uint_as_float(sr[3]), __uint_as_float(sr[7]));
#pragma unroll
                for (int e = 8; e < BN; e += 8) {
                    mx0 = fmax3(mx0, __uint_as_float(sr[e]), __uint_as_float(sr[e + 4]));
                    mx1 = fmax3(mx1, __uint_as_float(sr[e + 1]), __uint_as_float(sr[e + 5]));
                    mx2 = fmax3(mx2, __uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 6]));
                    mx3 = fmax3(mx3, __uint_as_float(sr[e + 3]), __uint_as_float(sr[e + 7]));
                }
                const float mx_s = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
                float m_new = m, alpha = 1.f;
                if (mx_s - m > RESCALE_THRESHOLD) {
                    m_new = mx_s;
                    alpha = ex2_approx(m - m_new);
                }
                const float nm = -m_new;
                float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
                for (int e = 0; e < BN; e += 4) {
                    float x0, x1, x2, x3;
                    ffma2(x0, x1, __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]), sl2, sl2, nm, nm);
                    ffma2(x2, x3, __uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3]), sl2, sl2, nm, nm);
                    x0 = ex2_approx(x0);
                    x1 = ex2_approx(x1);
                    x2 = ex2_approx(x2);
                    x3 = ex2_approx(x3);
                    fadd2(a0, a1, a0, a1, x0, x1);
                    fadd2(a2, a3, a2, a3, x2, x3);
                    sr[e / 2] = pack_bf16x2(x0, x1);
                    sr[e / 2 + 1] = pack_bf16x2(x2, x3);
                }
                tmem_st32(tS, sr);
                tmem_st32(tS + 32, sr + 32);
                l = l * alpha + ((a0 + a1) + (a2 + a3));
                m = m_new;
                if (__any_sync(0xffffffffu, j > 0 && alpha != 1.f)) {
#pragma unroll 1
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t r[32];
                        tmem_ld32(tO + 32 * ch, r);
                        tmem_wait_ld();
                        reg_fence32(r);
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            float y0, y1;
                            fmul2(y0, y1, __uint_as_float(r[e]), __uint_as_float(r[e + 1]), alpha, alpha);
                            r[e] = __float_as_uint(y0);
                            r[e + 1] = __float_as_uint(y1);
                        }
                        tmem_st32(tO + 32 * ch, r);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_P_READY + qi));
            }
            if (!ok) break;
            // epilogue: out = O / l, one row per thread
            if (!(ok = waiter.wait_warp(bar(B_O_DONE + qi), lu & 1, ROLE_SOFTMAX))) break;
            tc_fence_after();
            const float inv_l = 1.f / l;
            const int srow = c.qu * UNIT_ROWS + qi * BM + row;
            const bool store = srow < p.S;
            const size_t orow = (static_cast<size_t>(c.b) * p.S + (store ? srow : 0)) * p.H + c.h;
            if constexpr (BLOCK) {
                if (p.lse != nullptr && store) p.lse[orow] = (m + log2f(l)) * 0.6931471805599453f;
                if (p.out_f32) {
                    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow * D);
#pragma unroll 1
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t r[32];
                        tmem_ld32(tO + 32 * ch, r);
                        tmem_wait_ld();
                        reg_fence32(r);
                        if (store) {
#pragma unroll
                            for (int v4 = 0; v4 < 8; ++v4)
                                dst[ch * 8 + v4] = make_float4(
                                    __uint_as_float(r[4 * v4]) * inv_l, __uint_as_float(r[4 * v4 + 1]) * inv_l,
                                    __uint_as_float(r[4 * v4 + 2]) * inv_l, __uint_as_float(r[4 * v4 + 3]) * inv_l);
                        }
                    }
                    tc_fence_before();
                    continue;
                }
            }
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + orow * D);
            const uint64_t once = l2_evict_first_policy();   // output rows: written once, evicted first
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint32_t r[32];
                tmem_ld32(tO + 32 * ch, r);
                tmem_wait_ld();
                reg_fence32(r);
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l, __uint_as_float(r[2 * e + 1]) * inv_l);
                if (store) {
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4)
                        stg128_hint(dst + ch * 4 + v4,
                                    make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]), once);
                }
            }
            tc_fence_before();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == WARP_MMA) tmem_dealloc(tmem_base, TMEM_COLS);
}

// Workspace path, first stage: K' = R(K) for every video row, other rows
// copied, [B, S, heads, 128] bf16 in and out. One thread per 16-byte chunk
// (four adjacent channel pairs of one axis segment); the same fp32 rotation
// and bf16 rounding as the attention kernel's in-shared-memory path, with
// (cos, sin) from sincospif of the same angles, so both paths agree bit for
// bit. With the QK RMSNorm prologue (gamma_kv / gamma_kt non-null) every row
// is first normalised as the attention kernel normalises it, and text rows
// are normalised instead of copied. Memory-bound: reads and writes
// B*S*heads*256 bytes once. Warps step through whole pairs of rows (16
// chunks each), so a row's chunks always share a half-warp.
__global__ void __launch_bounds__(256) hv_rope_k_kernel(const uint4* __restrict__ kin, uint4* __restrict__ kout,
                                                        long long n_chunks, int H, int S, int N, int pos0, int Hp,
                                                        int Wp, float theta_log2, const float* __restrict__ gamma_kv,
                                                        const float* __restrict__ gamma_kt, float eps) {
    const long long step = static_cast<long long>(gridDim.x) * blockDim.x;
    const int lane = threadIdx.x & 31;
    const bool norm = gamma_kv != nullptr;
    for (long long e0 = static_cast<long long>(blockIdx.x) * blockDim.x + (threadIdx.x - lane); e0 < n_chunks;
         e0 += step) {
        const long long e = e0 + lane;
        const bool live = e < n_chunks;
        uint4 d = live ? __ldg(kin + e) : make_uint4(0u, 0u, 0u, 0u);
        const int cc = lane & 15;
        const long long row = e >> 4;               // (b * S + s) * H + h
        const int s_idx = static_cast<int>((row / H) % S);
        const bool video = s_idx < N;           // N: leading video rows of this block
        const int g_idx = pos0 + s_idx;         // global token index of a video row
        const int ch0 = cc * 8;
        int i0, dax, pos;
        if (ch0 < 16) {
            i0 = ch0 / 2; dax = 16; pos = g_idx / (Hp * Wp);
        } else if (ch0 < 72) {
            i0 = (ch0 - 16) / 2; dax = 56; pos = (g_idx / Wp) % Hp;
        } else {
            i0 = (ch0 - 72) / 2; dax = 56; pos = g_idx % Wp;
        }
        if (norm) {
            const float* gsrc = (video ? gamma_kv : gamma_kt) + ch0;
            float y[8];
            rms_norm_chunk(d, __ldg(reinterpret_cast<const uint4*>(gsrc)),
                           __ldg(reinterpret_cast<const uint4*>(gsrc + 4)), eps, y);
            uint32_t wv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (video) {
                    float sn, cs;
                    sincospif(angle_over_pi(pos, i0 + q, dax, theta_log2), &sn, &cs);
                    wv[q] = rotate_f(y[2 * q], y[2 * q + 1], cs, sn);
                } else {
                    wv[q] = pack_bf16x2(y[2 * q], y[2 * q + 1]);
                }
            }
            d = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        } else if (video) {
            uint32_t wv[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float sn, cs;
                sincospif(angle_over_pi(pos, i0 + q, dax, theta_log2), &sn, &cs);
                wv[q] = rotate_pair(wv[q], cs, sn);
            }
            d = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
        if (live) kout[e] = d;
    }
}

// Per-row statistics of the QK RMSNorm prologue on load: rinv[(b*H + h)*ld +
// s] = 1/sqrt(mean_j k_j^2 + eps) for every key row (b, s, h) of K [B, S, H,
// 128] bf16, by the same arithmetic as rms_norm_chunk (so the attention
// kernel's normalised keys are bit-identical to those of the two-stage
// form); the entries s in [S, ld) are set to 0, so that rows past the
// sequence scale to zero. Memory-bound: reads K once (B*S*H*256 bytes),
// writes B*H*ld*4 bytes. One half-warp per row, as in hv_rope_k_kernel.
__global__ void __launch_bounds__(256) hv_k_rinv_kernel(const uint4* __restrict__ kin, float* __restrict__ rinv,
                                                        long long n_chunks, int H, int S, int ld, float eps) {
    const long long step = static_cast<long long>(gridDim.x) * blockDim.x;
    const int lane = threadIdx.x & 31;
    for (long long e0 = static_cast<long long>(blockIdx.x) * blockDim.x + (threadIdx.x - lane); e0 < n_chunks;
         e0 += step) {
        const long long e = e0 + lane;
        const bool live = e < n_chunks;
        const uint4 d = live ? __ldg(kin + e) : make_uint4(0u, 0u, 0u, 0u);
        const float r = row_rms_inv(d, eps);
        if (live && (lane & 15) == 0) {
            const long long row = e >> 4;   // (b * S + s) * H + h
            const long long bs = row / H;
            const int h = static_cast<int>(row - bs * H);
            const long long b = bs / S;
            const int s_idx = static_cast<int>(bs - b * S);
            rinv[(b * H + h) * ld + s_idx] = r;
        }
    }
    const long long n_pad = n_chunks / (16ll * S) * (ld - S);   // B * H * (ld - S)
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_pad; i += step) {
        const long long bh = i / (ld - S);
        rinv[bh * ld + S + (i - bh * (ld - S))] = 0.f;
    }
}

// Ring attention, merge step: fold the result (o_part, lse_part) of one more
// key block into the running (o_acc, lse_acc) of the same query rows, as the
// softmax over the union of the keys: with m = max(lse_acc, lse_part),
// w = exp(lse - m), o_acc = (w_acc o_acc + w_part o_part) / (w_acc + w_part)
// and lse_acc = m + log(w_acc + w_part). A block with lse = -inf adds nothing.
// o_part is fp32 (PART_F32) or bf16. One warp per 128-channel row;
// optionally writes the merged row as bf16.
template <bool PART_F32>
__global__ void __launch_bounds__(256) hv_merge_kernel(float* __restrict__ o_acc, float* __restrict__ lse_acc,
                                                       const void* __restrict__ o_part,
                                                       const float* __restrict__ lse_part, uint2* __restrict__ out,
                                                       long long rows) {
    const int lane = threadIdx.x & 31;
    const long long wpb = blockDim.x >> 5;
    const long long step = static_cast<long long>(gridDim.x) * wpb;
    for (long long r = static_cast<long long>(blockIdx.x) * wpb + (threadIdx.x >> 5); r < rows; r += step) {
        const float la = lse_acc[r], lb = lse_part[r];
        __syncwarp();
        const float m = fmaxf(la, lb);
        float4 a = reinterpret_cast<float4*>(o_acc)[r * 32 + lane];
        float lse = m;
        if (m != -INFINITY) {
            const float wa = expf(la - m), wb = expf(lb - m);
            const float tot = wa + wb;
            float b0, b1, b2, b3;
            if constexpr (PART_F32) {
                const float4 pb = reinterpret_cast<const float4*>(o_part)[r * 32 + lane];
                b0 = pb.x; b1 = pb.y; b2 = pb.z; b3 = pb.w;
            } else {
                const uint2 pb = reinterpret_cast<const uint2*>(o_part)[r * 32 + lane];
                b0 = __uint_as_float(pb.x << 16); b1 = __uint_as_float(pb.x & 0xFFFF0000u);
                b2 = __uint_as_float(pb.y << 16); b3 = __uint_as_float(pb.y & 0xFFFF0000u);
            }
            const float inv = 1.f / tot;
            a.x = (a.x * wa + b0 * wb) * inv;
            a.y = (a.y * wa + b1 * wb) * inv;
            a.z = (a.z * wa + b2 * wb) * inv;
            a.w = (a.w * wa + b3 * wb) * inv;
            lse = m + logf(tot);
            reinterpret_cast<float4*>(o_acc)[r * 32 + lane] = a;
            if (lane == 0) lse_acc[r] = lse;
        }
        if (out != nullptr) out[r * 32 + lane] = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
    }
}

__global__ void hv_selftest_timeout_kernel(unsigned long long timeout_ns, unsigned int* status) {
    __shared__ __align__(8) uint64_t mbar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&mbar), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const Waiter w{&abort_flag, timeout_ns, status};
    w.wait_warp(smem_addr(&mbar), 0, ROLE_SELFTEST);
    __syncthreads();
}

// ------------------------------------------------------------------- host

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult qres;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// [B, S, H, 128] bf16 as a 4-D tensor (channel, head, token, batch); a box is
// 64 channels x 1 head x box_rows tokens, landing as box_rows rows of 128
// bytes with the 128-byte swizzle the MMA descriptors expect. Rows past S
// read as zero.
static bool make_qkv_map(CUtensorMap* map, const void* ptr, int B, int S, int H, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(S),
                                static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(H) * D * 2,
                                   static_cast<cuuint64_t>(S) * H * D * 2};
    const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

struct DeviceInfo {
    int ok = -1;   // -1 unknown, 0 unsupported, 1 sm_100
    int sms = 0;
};

// The attention kernel's instantiations: a ring-attention block (plain keys
// only), or the standard call with or without the QK RMSNorm prologue and
// with or without pre-rotated keys; each with and without the rotation table.
using AttnKernel = void (*)(Params);

template <bool BLOCK, bool QKN, bool KROT>
static AttnKernel attn_kernel(bool table) {
    return table ? hv_attn_fwd_kernel<BLOCK, QKN, KROT, true> : hv_attn_fwd_kernel<BLOCK, QKN, KROT, false>;
}

static AttnKernel kernel_for(bool block, bool qkn, bool krot, bool table) {
    if (block) return attn_kernel<true, false, false>(table);
    if (qkn) return krot ? attn_kernel<false, true, true>(table) : attn_kernel<false, true, false>(table);
    return krot ? attn_kernel<false, false, true>(table) : attn_kernel<false, false, false>(table);
}

// Every instantiation, for the per-device set-up.
constexpr int N_KERNELS = 10;
static AttnKernel kernel_at(int i) {
    const bool table = i & 1;
    switch (i >> 1) {
        case 0: return kernel_for(false, false, false, table);
        case 1: return kernel_for(false, false, true, table);
        case 2: return kernel_for(false, true, false, table);
        case 3: return kernel_for(false, true, true, table);
        default: return kernel_for(true, false, false, table);
    }
}

static DeviceInfo& device_info(int dev) {
    static DeviceInfo infos[64];
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    DeviceInfo& di = infos[dev & 63];
    if (di.ok < 0) {
        int major = 0, minor = 0, sms = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        di.sms = sms;
        di.ok = (major == 10 && minor == 0) ? 1 : 0;
        const void* kernels[N_KERNELS];
        for (int i = 0; i < N_KERNELS; ++i) kernels[i] = reinterpret_cast<const void*>(kernel_at(i));
        for (const void* kf : kernels)
            if (di.ok &&
                cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess)
                di.ok = 0;
        // The warpgroups' setmaxnreg split adds up to exactly 512 threads x 128
        // registers; a kernel launched with fewer would wait forever on the
        // increase, so refuse to launch one.
        const int split = static_cast<int>(regs_split(false) > regs_split(true) ? regs_split(false) : regs_split(true));
        for (const void* kf : kernels) {
            cudaFuncAttributes fa;
            if (di.ok && (cudaFuncGetAttributes(&fa, kf) != cudaSuccess || fa.numRegs * NUM_THREADS < split))
                di.ok = 0;
        }
    }
    return di;
}

static bool overlaps(const void* a, const void* b, size_t bytes) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + bytes && y < x + bytes;
}

// [a, a + a_bytes) and [b, b + b_bytes) share a byte
static bool ranges_overlap(const void* a, size_t a_bytes, const void* b, size_t b_bytes) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + b_bytes && y < x + a_bytes;
}

constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;   // 2 s per wait

// Host-visible status words, one 64-byte line per device ordinal, in a static
// page of host memory that is page-locked and mapped into the device's
// address space at first use (registration, not an allocation). A kernel
// wait that runs out stores its code there, so that every later call sees
// it without synchronising; hv_attn_last_device_error clears it.
struct alignas(4096) StatusPage {
    unsigned int word[64 * 16];
};
static StatusPage g_status_page;
static std::mutex g_status_mu;

static unsigned int* status_host(int dev) { return &g_status_page.word[(dev & 63) * 16]; }

// Device address of this device's status word (the current device must be
// `dev`), or nullptr if the page cannot be mapped (then only the device error
// word records a timeout).
static unsigned int* status_word_dev(int dev) {
    std::lock_guard<std::mutex> lock(g_status_mu);
    void* dptr = nullptr;
    if (cudaHostGetDevicePointer(&dptr, status_host(dev), 0) == cudaSuccess) return static_cast<unsigned int*>(dptr);
    (void)cudaGetLastError();   // not registered (yet, or no longer): not an error of the call
    if (cudaHostRegister(&g_status_page, sizeof(g_status_page), cudaHostRegisterMapped | cudaHostRegisterPortable) !=
        cudaSuccess) {
        (void)cudaGetLastError();
        return nullptr;
    }
    if (cudaHostGetDevicePointer(&dptr, status_host(dev), 0) != cudaSuccess) {
        (void)cudaGetLastError();
        return nullptr;
    }
    return static_cast<unsigned int*>(dptr);
}

static bool status_timed_out(int dev) { return *static_cast<volatile unsigned int*>(status_host(dev)) != 0u; }

struct Call {
    int S = 0, N = 0, sms = 0, dev = 0;
    long long units = 0;
    size_t bytes = 0;   // bytes of one [B, S, heads, 128] bf16 tensor
};

// Options of one launch of the attention kernel beyond the call's arguments.
struct LaunchOpts {
    unsigned long long timeout_ns = kWaitTimeoutNs;
    const float* k_rinv = nullptr;   // per-row K statistics (QK RMSNorm on load), see Params
    int k_rinv_ld = 0;
    int withhold_k = -1;   // test hook of hv_attn_selftest_abort
    int h_total = 0;       // heads of the whole call (0: this launch's), for a launch over a head group
    int h_offset = 0;      // first head of the group within the call
};

// Checks of the QK RMSNorm arguments: gamma (device, fp32 [4][128], 16-byte
// aligned, not overlapping out) and eps (finite, >= 0).
static int validate_qk_norm(const float* qk_gamma, float eps, const void* out, size_t out_bytes) {
    if (!qk_gamma) return HV_ERR_NULL_POINTER;
    if (reinterpret_cast<uintptr_t>(qk_gamma) & 15u) return HV_ERR_MISALIGNED;
    if (!std::isfinite(eps) || eps < 0.f) return HV_ERR_BAD_SCALAR;
    if (ranges_overlap(out, out_bytes, qk_gamma, GAMMA_BYTES)) return HV_ERR_ALIAS;
    return HV_OK;
}

// Argument checks (then the device): every error a call can report before
// launching. qk_norm: also check the RMSNorm arguments qk_gamma / qk_eps.
static int validate(const void* q, const void* k, const void* v, const void* out, int B, int heads, int T, int Hp,
                    int Wp, int text_len, const int* text_valid, float rope_theta, float scale, Call& call,
                    bool qk_norm = false, const float* qk_gamma = nullptr, float qk_eps = 0.f) {
    if (!q || !k || !v || !out || !text_valid) return HV_ERR_NULL_POINTER;
    const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                          reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out);
    if (mis & 15u) return HV_ERR_MISALIGNED;
    if (B < 1 || heads < 1 || T < 1 || Hp < 1 || Wp < 1 || B > HV_MAX_BATCH) return HV_ERR_BAD_SHAPE;
    if (text_len < 0 || text_len > HV_MAX_TEXT_LEN) return HV_ERR_BAD_TEXT;
    for (int b = 0; b < B; ++b)
        if (text_valid[b] < 0 || text_valid[b] > text_len) return HV_ERR_BAD_TEXT;
    if (!std::isfinite(rope_theta) || !(rope_theta > 0.f) || !std::isfinite(scale)) return HV_ERR_BAD_SCALAR;
    const long long n_video = static_cast<long long>(T) * Hp * Wp;
    const long long s_len = n_video + text_len;
    const long long units = static_cast<long long>(B) * heads * ((s_len + UNIT_ROWS - 1) / UNIT_ROWS);
    if (s_len + UNIT_ROWS >= (1ll << 31) || s_len * heads * D >= (1ll << 31) || units >= (1ll << 31))
        return HV_ERR_TOO_LARGE;
    const size_t bytes = static_cast<size_t>(B) * s_len * heads * D * 2;
    if (overlaps(out, q, bytes) || overlaps(out, k, bytes) || overlaps(out, v, bytes)) return HV_ERR_ALIAS;
    if (qk_norm) {
        const int st = validate_qk_norm(qk_gamma, qk_eps, out, bytes);
        if (st != HV_OK) return st;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return HV_ERR_LAUNCH;
    DeviceInfo& di = device_info(dev);
    if (di.ok != 1) return HV_ERR_NO_DEVICE;
    if (status_timed_out(dev)) return HV_ERR_DEVICE_TIMEOUT;
    call.S = static_cast<int>(s_len);
    call.N = static_cast<int>(n_video);
    call.sms = di.sms;
    call.dev = dev;
    call.units = units;
    call.bytes = bytes;
    return HV_OK;
}

// Built-in scratch for hv_attn_forward_noalloc: room for the rotated keys of
// problems up to HV_NOALLOC_MAX_BYTES. It is part of the module, so every
// device that loads this library holds it until the process exits; no
// allocation call ever creates it. All calls share it.
static __device__ __align__(256) uint8_t g_noalloc_scratch[HV_NOALLOC_MAX_BYTES];

// Device address of g_noalloc_scratch in the current context. In host code
// the array's name is only a stand-in; the address must come from the
// runtime. It is looked up on every call (a cheap table lookup once the
// module is loaded), so a context that was reset and re-created, where the
// array may sit elsewhere, never sees a stale address.
static void* noalloc_scratch() {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
    return ptr;
}

// Row blocks of a ring-attention step (see Params); the standard call is the
// whole sequence against itself.
struct Blocks {
    int Sk, q_vid, q_pos0, k_vid, k_pos0;
    const int* kv_len;   // host, B entries, each in [1, Sk]
    float* lse;          // device or nullptr
    int out_f32;         // 1: out rows are fp32
};

static int launch_attention(const Call& call, const void* q, const void* k, const void* v, void* out, int B,
                            int heads, int T, int Hp, int Wp, int text_len, const int* text_valid, float rope_theta,
                            float scale, bool k_rotated, const float* qk_gamma, float qk_eps,
                            cudaStream_t stream, const Blocks* blk = nullptr, const LaunchOpts& opts = LaunchOpts()) {
    (void)text_len;
    Params* prm = new Params;   // ~2.5 KB; heap to keep the host stack small
    std::memset(prm, 0, sizeof(Params));
    const int S = call.S;
    const int Sk = blk ? blk->Sk : S;
    if (!make_qkv_map(&prm->tm_q, q, B, S, heads, BM) || !make_qkv_map(&prm->tm_k, k, B, Sk, heads, BN) ||
        !make_qkv_map(&prm->tm_v, v, B, Sk, heads, BN)) {
        delete prm;
        return HV_ERR_LAUNCH;
    }
    prm->out = out;
    prm->B = B;
    prm->H = heads;
    prm->S = S;
    prm->N = call.N;
    prm->T = T;
    prm->Hp = Hp;
    prm->Wp = Wp;
    prm->use_table = (8ll * T + 28ll * (Hp + static_cast<long long>(Wp))) <= TABLE_MAX_ENTRIES ? 1 : 0;
    prm->qk_eps = qk_eps;
    prm->qk_gamma = qk_gamma;
    prm->k_rinv = opts.k_rinv;
    prm->k_rinv_ld = opts.k_rinv_ld;
    prm->HpWp = Hp * Wp;
    prm->n_qunits = (S + UNIT_ROWS - 1) / UNIT_ROWS;
    prm->units = static_cast<int>(call.units);
    prm->theta_log2 = static_cast<float>(std::log2(static_cast<double>(rope_theta)));
    prm->scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    prm->timeout_ns = opts.timeout_ns;
    prm->status = status_word_dev(call.dev);
    prm->withhold_k = opts.withhold_k;
    prm->h_total = opts.h_total > 0 ? opts.h_total : heads;
    prm->h_offset = opts.h_offset;
    prm->round_width = call.sms;
    prm->Sk = Sk;
    if (blk) {
        prm->q_vid = blk->q_vid;
        prm->q_pos0 = blk->q_pos0;
        prm->k_vid = blk->k_vid;
        prm->k_pos0 = blk->k_pos0;
        prm->lse = blk->lse;
        prm->out_f32 = blk->out_f32;
        for (int b = 0; b < B; ++b) prm->kv_len[b] = blk->kv_len[b];
    } else {
        prm->q_vid = prm->k_vid = call.N;
        for (int b = 0; b < B; ++b) prm->kv_len[b] = call.N + text_valid[b];
    }
    // persistent grid: one CTA per SM, at most one per work unit
    const int grid = static_cast<int>(call.units < call.sms ? call.units : call.sms);
    // keys normalised on load always come with their row factors (hv_k_rinv_kernel)
    if (qk_gamma != nullptr && !k_rotated && opts.k_rinv == nullptr) {
        delete prm;
        return HV_ERR_LAUNCH;
    }
    const AttnKernel kern = kernel_for(blk != nullptr, qk_gamma != nullptr, k_rotated, prm->use_table != 0);
    kern<<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(*prm);
    cudaError_t err = cudaSuccess;
    delete prm;
    if (err == cudaSuccess) err = cudaGetLastError();
    return err == cudaSuccess ? HV_OK : HV_ERR_LAUNCH;
}

// First stage of the workspace paths: K' (rotated, and normalised when
// qk_gamma is set) into `dst`.
static int launch_rope_k(const Call& call, const void* k, void* dst, int heads, int Hp, int Wp, float rope_theta,
                         const float* qk_gamma, float qk_eps, cudaStream_t stream) {
    const long long n_chunks = static_cast<long long>(call.bytes / 16);
    hv_rope_k_kernel<<<8 * call.sms, 256, 0, stream>>>(
        static_cast<const uint4*>(k), static_cast<uint4*>(dst), n_chunks, heads, call.S, call.N, 0, Hp, Wp,
        static_cast<float>(std::log2(static_cast<double>(rope_theta))), qk_gamma ? qk_gamma + D : nullptr,
        qk_gamma ? qk_gamma + 3 * D : nullptr, qk_eps);
    return cudaGetLastError() == cudaSuccess ? HV_OK : HV_ERR_LAUNCH;
}

// Streams and events of the host-buffer pipeline, created once per device.
// Streams and events of the host-buffer pipeline, per device: copies in and
// out on their own streams, and the attention launches alternating between
// two compute streams, so that a launch's CTAs take the SMs the previous
// launch's CTAs leave while its last wave finishes (independent heads, no
// kernel waits on another).
struct HostPipe {
    bool ok = false;
    cudaStream_t h2d = nullptr, d2h = nullptr, comp[2] = {};
    cudaEvent_t start = nullptr;
    cudaEvent_t h2d_done[2] = {}, comp_done[2] = {}, d2h_done[2] = {};
};

static std::mutex g_host_pipe_mu;   // also serialises the enqueue of whole calls

static HostPipe* host_pipe(int dev) {
    static HostPipe pipes[64];
    HostPipe& hp = pipes[dev & 63];
    if (!hp.ok) {
        bool good = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) == cudaSuccess &&
                    cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) == cudaSuccess &&
                    cudaStreamCreateWithFlags(&hp.comp[0], cudaStreamNonBlocking) == cudaSuccess &&
                    cudaStreamCreateWithFlags(&hp.comp[1], cudaStreamNonBlocking) == cudaSuccess &&
                    cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming) == cudaSuccess;
        for (int i = 0; i < 2 && good; ++i)
            good = cudaEventCreateWithFlags(&hp.h2d_done[i], cudaEventDisableTiming) == cudaSuccess &&
                   cudaEventCreateWithFlags(&hp.comp_done[i], cudaEventDisableTiming) == cudaSuccess &&
                   cudaEventCreateWithFlags(&hp.d2h_done[i], cudaEventDisableTiming) == cudaSuccess;
        if (!good) return nullptr;
        hp.ok = true;
    }
    return &hp;
}

// bytes of one head group's staging tensor [B, S, heads/groups, 128] bf16
static long long host_group_bytes(int B, int heads, int T, int Hp, int Wp, int text_len, int groups) {
    if (B < 1 || heads < 1 || T < 1 || Hp < 1 || Wp < 1 || text_len < 0 || text_len > HV_MAX_TEXT_LEN ||
        groups < 1 || heads % groups != 0)
        return -1;
    const long long s_len = static_cast<long long>(T) * Hp * Wp + text_len;
    return static_cast<long long>(B) * s_len * (heads / groups) * D * 2;
}

}  // namespace hv

extern "C" {

const char* hv_attn_status_string(int status) {
    switch (status) {
        case HV_OK: return "ok";
        case HV_ERR_NULL_POINTER: return "null pointer";
        case HV_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case HV_ERR_BAD_SHAPE: return "bad shape (B, heads, T, Hp, Wp must be >= 1, B <= HV_MAX_BATCH)";
        case HV_ERR_BAD_TEXT: return "bad text length (0 <= text_valid[b] <= text_len <= 256)";
        case HV_ERR_TOO_LARGE: return "problem too large for int32 TMA coordinates";
        case HV_ERR_ALIAS: return "out overlaps q, k or v";
        case HV_ERR_BAD_SCALAR: return "rope_theta must be finite and > 0, scale finite";
        case HV_ERR_NO_DEVICE: return "current CUDA device is not sm_100";
        case HV_ERR_LAUNCH: return "CUDA launch or driver call failed";
        case HV_ERR_DEVICE_TIMEOUT: return "a kernel-side wait timed out";
        case HV_ERR_WORKSPACE: return "workspace missing, misaligned, too small or overlapping an operand";
        case HV_ERR_NOALLOC_LIMIT:
            return "problem needs more scratch than hv_attn_forward_noalloc's built-in HV_NOALLOC_MAX_BYTES";
        default: return "unknown status";
    }
}

long long hv_video_tokens(int frames, int height, int width) {
    if (frames < 1 || (frames - 1) % 4 != 0) return -1;
    if (height <= 0 || width <= 0 || height % 16 != 0 || width % 16 != 0) return -1;
    const long long t = (frames - 1) / 4 + 1;
    return t * (height / 16) * static_cast<long long>(width / 16);
}

int hv_attn_forward(const void* q, const void* k, const void* v, void* out, int B, int heads, int T, int Hp, int Wp,
                    int text_len, const int* text_valid, float rope_theta, float scale, void* cuda_stream) {
    using namespace hv;
    Call call;
    int st = validate(q, k, v, out, B, heads, T, Hp, Wp, text_len, text_valid, rope_theta, scale, call);
    if (st != HV_OK) return st;
    return launch_attention(call, q, k, v, out, B, heads, T, Hp, Wp, text_len, text_valid, rope_theta, scale, false,
                            nullptr, 0.f, static_cast<cudaStream_t>(cuda_stream));
}

int hv_attn_forward_qknorm(const void* q, const void* k, const void* v, void* out, int B, int heads, int T, int Hp,
                           int Wp, int text_len, const int* text_valid, float rope_theta, float scale,
                           const float* qk_gamma, float qk_eps, void* cuda_stream) {
    using namespace hv;
    Call call;
    int st = validate(q, k, v, out, B, heads, T, Hp, Wp, text_len, text_valid, rope_theta, scale, call, true,
                      qk_gamma, qk_eps);
    if (st != HV_OK) return st;
    const cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    // 1/rms of every key row, once per call, into stream-ordered scratch
    // from the device's default memory pool, released behind the attention
    // kernel on the same stream
    LaunchOpts opts;
    opts.k_rinv_ld = (call.S + BN - 1) / BN * BN;
    const size_t rinv_bytes = static_cast<size_t>(B) * heads * opts.k_rinv_ld * sizeof(float);
    void* rinv = nullptr;
    if (cudaMallocAsync(&rinv, rinv_bytes, stream) != cudaSuccess) {
        (void)cudaGetLastError();
        return HV_ERR_LAUNCH;
    }
    if (reinterpret_cast<uintptr_t>(rinv) & 15u) {   // the tile copies need 16-byte alignment
        (void)cudaFreeAsync(rinv, stream);
        return HV_ERR_LAUNCH;
    }
    opts.k_rinv = static_cast<const float*>(rinv);
    hv_k_rinv_kernel<<<8 * call.sms, 256, 0, stream>>>(static_cast<const uint4*>(k), static_cast<float*>(rinv),
                                                       static_cast<long long>(call.bytes / 16), heads, call.S,
                                                       opts.k_rinv_ld, qk_eps);
    st = cudaGetLastError() == cudaSuccess ? HV_OK : HV_ERR_LAUNCH;
    if (st == HV_OK)
        st = launch_attention(call, q, k, v, out, B, heads, T, Hp, Wp, text_len, text_valid, rope_theta, scale, false,
                              qk_gamma, qk_eps, stream, nullptr, opts);
    if (cudaFreeAsync(rinv, stream) != cudaSuccess && st == HV_OK) st = HV_ERR_LAUNCH;
    return st;
}

long long hv_attn_workspace_bytes(int B, int heads, int T, int Hp, int Wp, int text_len) {
    if (B < 1 || heads < 1 || T < 1 || Hp < 1 || Wp < 1 || text_len < 0 || text_len > HV_MAX_TEXT_LEN) return -1;
    const long long s_len = static_cast<long long>(T) * Hp * Wp + text_len;
    return static_cast<long long>(B) * s_len * heads * hv::D * 2;
}

int hv_attn_forward_ws(const void* q, const void* k, const void* v, void* out, int B, int heads, int T, int Hp,
                       int Wp, int text_len, const int* text_valid, float rope_theta, float scale, void* workspace,
                       size_t workspace_bytes, void* cuda_stream) {
    using namespace hv;
    Call call;
    int st = validate(q, k, v, out, B, heads, T, Hp, Wp, text_len, text_valid, rope_theta, scale, call);
    if (st != HV_OK) return st;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 15u) || workspace_bytes < call.bytes ||
        overlaps(workspace, q, call.bytes) || overlaps(workspace, k, call.bytes) || overlaps(workspace, v, call.bytes) ||
        overlaps(workspace, out, call.bytes))
        return HV_ERR_WORKSPACE;
    const cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    st = launch_rope_k(call, k, workspace, heads, Hp, Wp, rope_theta, nullptr, 0.f, stream);
    if (st != HV_OK) return st;
    return launch_attention(call, q, workspace, v, out, B, heads, T, Hp, Wp, text_len, text_valid, rope_theta, scale,
                            true, nullptr, 0.f, stream);
}

int hv_attn_forward_qknorm_ws(const void* q, const void* k, const void* v, void* out, int B, int heads, int T,
                              int Hp, int Wp, int text_len, const int* text_valid, float rope_theta, float scale,
                              const float* qk_gamma, float qk_eps, void* workspace, size_t workspace_bytes,
                              void* cuda_stream) {
    using namespace hv;
    Call call;
    int st = validate(q, k, v, out, B, heads, T, Hp, Wp, text_len, text_valid, rope_theta, scale, call, true,
                      qk_gamma, qk_eps);
    if (st != HV_OK) return st;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 15u) || workspace_bytes < call.bytes ||
        overlaps(workspace, q, call.bytes) || overlaps(workspace, k, call.bytes) || overlaps(workspace, v, call.bytes) ||
        overlaps(workspace, out, call.bytes) || ranges_overlap(workspace, call.bytes, qk_gamma, GAMMA_BYTES))
        return HV_ERR_WORKSPACE;
    const cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    st = launch_rope_k(call, k, workspace, heads, Hp, Wp, rope_theta, qk_gamma, qk_eps, stream);
    if (st != HV_OK) return st;
    return launch_attention(call, q, workspace, v, out, B, heads, T, Hp, Wp, text_len, text_valid, rope_theta, scale,
                            true, qk_gamma, qk_eps, stream);
}

int hv_attn_forward_noalloc(const void* q, const void* k, const void* v, void* out, int B, int heads, int T,
                            int Hp, int Wp, int text_len, const int* text_valid, float rope_theta, float scale,
                            void* cuda_stream) {
    using namespace hv;
    Call call;
    int st = validate(q, k, v, out, B, heads, T, Hp, Wp, text_len, text_valid, rope_theta, scale, call);
    if (st != HV_OK) return st;
    if (call.bytes > HV_NOALLOC_MAX_BYTES) return HV_ERR_NOALLOC_LIMIT;
    void* scratch = noalloc_scratch();
    if (!scratch) return HV_ERR_LAUNCH;
    // the first stage overwrites every byte of the scratch it uses, so
    // nothing left there by an earlier call needs clearing
    const cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    st = launch_rope_k(call, k, scratch, heads, Hp, Wp, rope_theta, nullptr, 0.f, stream);
    if (st != HV_OK) return st;
    return launch_attention(call, q, scratch, v, out, B, heads, T, Hp, Wp, text_len, text_valid, rope_theta, scale,
                            true, nullptr, 0.f, stream);
}

long long hv_attn_host_workspace_bytes(int B, int heads, int T, int Hp, int Wp, int text_len, int head_groups) {
    const long long g = hv::host_group_bytes(B, heads, T, Hp, Wp, text_len, head_groups);
    return g < 0 ? -1 : 8 * g;   // two slots of q, k, v, out
}

int hv_attn_forward_host(const void* q_host, const void* k_host, const void* v_host, void* out_host, int B,
                         int heads, int T, int Hp, int Wp, int text_len, const int* text_valid, float rope_theta,
                         float scale, int head_groups, void* workspace, size_t workspace_bytes, void* cuda_stream) {
    using namespace hv;
    if (!q_host || !k_host || !v_host || !out_host || !text_valid || !workspace) return HV_ERR_NULL_POINTER;
    if (B < 1 || heads < 1 || T < 1 || Hp < 1 || Wp < 1 || B > HV_MAX_BATCH || head_groups < 1 ||
        heads % head_groups != 0)
        return HV_ERR_BAD_SHAPE;
    const long long gbytes = host_group_bytes(B, heads, T, Hp, Wp, text_len, head_groups);
    if (gbytes < 0) return HV_ERR_BAD_TEXT;
    const int hg = heads / head_groups;
    const size_t full = static_cast<size_t>(gbytes) * head_groups;
    if (overlaps(out_host, q_host, full) || overlaps(out_host, k_host, full) || overlaps(out_host, v_host, full))
        return HV_ERR_ALIAS;
    if ((reinterpret_cast<uintptr_t>(workspace) & 15u) || workspace_bytes < static_cast<size_t>(8 * gbytes))
        return HV_ERR_WORKSPACE;
    // validate one group's device call up front (shapes, text, scalars, device)
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    auto slot_buf = [&](int slot, int t) { return ws + (static_cast<size_t>(slot) * 4 + t) * gbytes; };
    Call call;
    int st = validate(slot_buf(0, 0), slot_buf(0, 1), slot_buf(0, 2), slot_buf(0, 3), B, hg, T, Hp, Wp, text_len,
                      text_valid, rope_theta, scale, call);
    if (st != HV_OK) return st;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return HV_ERR_LAUNCH;
    std::lock_guard<std::mutex> lock(g_host_pipe_mu);
    HostPipe* hp = host_pipe(dev);
    if (!hp) return HV_ERR_LAUNCH;
    const cudaStream_t cs = static_cast<cudaStream_t>(cuda_stream);
    const size_t row = static_cast<size_t>(heads) * D * 2;
    const size_t rows = static_cast<size_t>(B) * call.S;
    bool good = cudaEventRecord(hp->start, cs) == cudaSuccess &&
                cudaStreamWaitEvent(hp->h2d, hp->start, 0) == cudaSuccess &&
                cudaStreamWaitEvent(hp->d2h, hp->start, 0) == cudaSuccess &&
                cudaStreamWaitEvent(hp->comp[0], hp->start, 0) == cudaSuccess &&
                cudaStreamWaitEvent(hp->comp[1], hp->start, 0) == cudaSuccess;
    const void* src[3] = {q_host, k_host, v_host};
    int piece = 0;   // pieces enqueued so far; piece i uses slot i & 1 and compute stream i & 1
    // One piece: heads h0 .. h0 + n - 1 copied in, computed and copied out.
    auto run_piece = [&](int h0, int n) {
        const int slot = piece++ & 1;
        const cudaStream_t comp = hp->comp[slot];
        const size_t col = static_cast<size_t>(h0) * D * 2, grow = static_cast<size_t>(n) * D * 2;
        // inputs of this piece into the slot, once the piece that used it last has been computed
        good = good && cudaStreamWaitEvent(hp->h2d, hp->comp_done[slot], 0) == cudaSuccess;
        for (int t = 0; t < 3 && good; ++t)
            good = cudaMemcpy2DAsync(slot_buf(slot, t), grow, static_cast<const uint8_t*>(src[t]) + col, row, grow,
                                     rows, cudaMemcpyHostToDevice, hp->h2d) == cudaSuccess;
        good = good && cudaEventRecord(hp->h2d_done[slot], hp->h2d) == cudaSuccess;
        // attention of the piece, once its inputs are in and the slot's output has been copied out
        good = good && cudaStreamWaitEvent(comp, hp->h2d_done[slot], 0) == cudaSuccess &&
               cudaStreamWaitEvent(comp, hp->d2h_done[slot], 0) == cudaSuccess;
        if (good) {
            Call pc = call;
            pc.units = static_cast<long long>(B) * n * ((call.S + UNIT_ROWS - 1) / UNIT_ROWS);
            LaunchOpts opts;
            opts.h_total = heads;
            opts.h_offset = h0;
            st = launch_attention(pc, slot_buf(slot, 0), slot_buf(slot, 1), slot_buf(slot, 2), slot_buf(slot, 3), B,
                                  n, T, Hp, Wp, text_len, text_valid, rope_theta, scale, false, nullptr, 0.f, comp,
                                  nullptr, opts);
            if (st != HV_OK) good = false;
        }
        good = good && cudaEventRecord(hp->comp_done[slot], comp) == cudaSuccess;
        // the piece's output back into its columns of out_host
        good = good && cudaStreamWaitEvent(hp->d2h, hp->comp_done[slot], 0) == cudaSuccess &&
               cudaMemcpy2DAsync(static_cast<uint8_t*>(out_host) + col, row, slot_buf(slot, 3), grow, grow, rows,
                                 cudaMemcpyDeviceToHost, hp->d2h) == cudaSuccess &&
               cudaEventRecord(hp->d2h_done[slot], hp->d2h) == cudaSuccess;
    };
    // The head groups in order; the first and the last are cut into one head
    // and the rest, so that only one head's columns are copied in before the
    // first kernel and copied out after the last.
    for (int g = 0; g < head_groups && good; ++g) {
        const int h0 = g * hg;
        if (hg > 1 && g == 0) {
            run_piece(h0, 1);
            run_piece(h0 + 1, hg - 1);
        } else if (hg > 1 && g == head_groups - 1) {
            run_piece(h0, hg - 1);
            run_piece(h0 + hg - 1, 1);
        } else {
            run_piece(h0, hg);
        }
    }
    if (st != HV_OK) return st;
    // the caller's stream completes after the last copy out
    for (int slot = 0; slot < 2 && good; ++slot) good = cudaStreamWaitEvent(cs, hp->d2h_done[slot], 0) == cudaSuccess;
    return good ? HV_OK : HV_ERR_LAUNCH;
}

int hv_attn_forward_block(const void* q, const void* k, const void* v, void* out, float* lse, int B, int heads,
                          int T, int Hp, int Wp, int Sq, int q_video, int q_pos0, int Sk, int k_video, int k_pos0,
                          const int* kv_len, float rope_theta, float scale, int out_fp32, void* cuda_stream) {
    using namespace hv;
    if (!q || !k || !v || !out || !kv_len) return HV_ERR_NULL_POINTER;
    const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                          reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out);
    if ((mis & 15u) || (reinterpret_cast<uintptr_t>(lse) & 3u)) return HV_ERR_MISALIGNED;
    if (B < 1 || heads < 1 || T < 1 || Hp < 1 || Wp < 1 || B > HV_MAX_BATCH || Sq < 1 || Sk < 1 ||
        (out_fp32 != 0 && out_fp32 != 1))
        return HV_ERR_BAD_SHAPE;
    const long long n_video = static_cast<long long>(T) * Hp * Wp;
    if (q_video < 0 || q_video > Sq || k_video < 0 || k_video > Sk || q_pos0 < 0 || k_pos0 < 0 ||
        q_pos0 + static_cast<long long>(q_video) > n_video || k_pos0 + static_cast<long long>(k_video) > n_video)
        return HV_ERR_BAD_SHAPE;
    for (int b = 0; b < B; ++b)
        if (kv_len[b] < 1 || kv_len[b] > Sk) return HV_ERR_BAD_TEXT;
    if (!std::isfinite(rope_theta) || !(rope_theta > 0.f) || !std::isfinite(scale)) return HV_ERR_BAD_SCALAR;
    const long long units = static_cast<long long>(B) * heads * ((Sq + UNIT_ROWS - 1) / UNIT_ROWS);
    const long long big = static_cast<long long>(Sq > Sk ? Sq : Sk);
    if (big + UNIT_ROWS >= (1ll << 31) || big * heads * D >= (1ll << 31) || units >= (1ll << 31) ||
        n_video >= (1ll << 31))
        return HV_ERR_TOO_LARGE;
    const size_t qb = static_cast<size_t>(B) * Sq * heads * D * 2, kb = static_cast<size_t>(B) * Sk * heads * D * 2;
    const size_t ob = out_fp32 ? 2 * qb : qb;
    const size_t lb = static_cast<size_t>(B) * Sq * heads * 4;
    if (ranges_overlap(out, ob, q, qb) || ranges_overlap(out, ob, k, kb) || ranges_overlap(out, ob, v, kb))
        return HV_ERR_ALIAS;
    if (lse && (ranges_overlap(lse, lb, out, ob) || ranges_overlap(lse, lb, q, qb) || ranges_overlap(lse, lb, k, kb) ||
                ranges_overlap(lse, lb, v, kb)))
        return HV_ERR_ALIAS;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return HV_ERR_LAUNCH;
    DeviceInfo& di = device_info(dev);
    if (di.ok != 1) return HV_ERR_NO_DEVICE;
    if (status_timed_out(dev)) return HV_ERR_DEVICE_TIMEOUT;
    Call call;
    call.S = Sq;
    call.N = static_cast<int>(n_video);
    call.sms = di.sms;
    call.dev = dev;
    call.units = units;
    call.bytes = qb;
    const Blocks blk{Sk, q_video, q_pos0, k_video, k_pos0, kv_len, lse, out_fp32};
    return launch_attention(call, q, k, v, out, B, heads, T, Hp, Wp, 0, nullptr, rope_theta, scale, false, nullptr,
                            0.f, static_cast<cudaStream_t>(cuda_stream), &blk);
}

int hv_attn_merge(float* o_acc, float* lse_acc, const void* o_part, int o_part_fp32, const float* lse_part, void* out,
                  long long rows, void* cuda_stream) {
    using namespace hv;
    if (!o_acc || !lse_acc || !o_part || !lse_part) return HV_ERR_NULL_POINTER;
    if ((reinterpret_cast<uintptr_t>(o_acc) & 15u) || (reinterpret_cast<uintptr_t>(o_part) & (o_part_fp32 ? 15u : 7u)) ||
        (reinterpret_cast<uintptr_t>(out) & 7u) || (reinterpret_cast<uintptr_t>(lse_acc) & 3u) ||
        (reinterpret_cast<uintptr_t>(lse_part) & 3u))
        return HV_ERR_MISALIGNED;
    if (rows < 0 || (o_part_fp32 != 0 && o_part_fp32 != 1)) return HV_ERR_BAD_SHAPE;
    if (rows == 0) return HV_OK;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return HV_ERR_LAUNCH;
    DeviceInfo& di = device_info(dev);
    if (di.ok != 1) return HV_ERR_NO_DEVICE;
    if (status_timed_out(dev)) return HV_ERR_DEVICE_TIMEOUT;
    const long long blocks = (rows + 7) / 8;
    const int grid = static_cast<int>(blocks < 16ll * di.sms ? blocks : 16ll * di.sms);
    const cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    if (o_part_fp32)
        hv_merge_kernel<true><<<grid, 256, 0, stream>>>(o_acc, lse_acc, o_part, lse_part, static_cast<uint2*>(out),
                                                        rows);
    else
        hv_merge_kernel<false><<<grid, 256, 0, stream>>>(o_acc, lse_acc, o_part, lse_part, static_cast<uint2*>(out),
                                                         rows);
    return cudaGetLastError() == cudaSuccess ? HV_OK : HV_ERR_LAUNCH;
}

int hv_attn_last_device_error(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    unsigned int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, hv::g_dev_error, sizeof(word)) != cudaSuccess) return -1;
    if (cudaMemcpyToSymbol(hv::g_dev_error, &zero, sizeof(zero)) != cudaSuccess) return -1;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    *static_cast<volatile unsigned int*>(hv::status_host(dev)) = 0u;
    return static_cast<int>(word);
}

int hv_attn_selftest_timeout(int timeout_us) {
    if (timeout_us < 1 || timeout_us > 1000000) return -1;
    if (hv_attn_last_device_error() < 0) return -1;   // clears the words first
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    hv::hv_selftest_timeout_kernel<<<1, 32>>>(static_cast<unsigned long long>(timeout_us) * 1000ull,
                                              hv::status_word_dev(dev));
    if (cudaGetLastError() != cudaSuccess) return -1;
    return hv_attn_last_device_error();
}

int hv_attn_selftest_abort(const void* q, const void* k, const void* v, void* out, int B, int heads, int T, int Hp,
                           int Wp, int text_len, const int* text_valid, int withhold_k, int timeout_us,
                           void* cuda_stream) {
    using namespace hv;
    if (withhold_k < 0 || timeout_us < 1000 || timeout_us > 1000000) return HV_ERR_BAD_SCALAR;
    Call call;
    const int st = validate(q, k, v, out, B, heads, T, Hp, Wp, text_len, text_valid, 256.f, 0.08838834764831843f, call);
    if (st != HV_OK) return st;
    LaunchOpts opts;
    opts.timeout_ns = static_cast<unsigned long long>(timeout_us) * 1000ull;
    opts.withhold_k = withhold_k;
    const cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    const int ls = launch_attention(call, q, k, v, out, B, heads, T, Hp, Wp, text_len, text_valid, 256.f,
                                    0.08838834764831843f, false, nullptr, 0.f, stream, nullptr, opts);
    if (ls != HV_OK) return ls;
    return cudaStreamSynchronize(stream) == cudaSuccess ? HV_OK : HV_ERR_LAUNCH;
}

}  // extern "C"
