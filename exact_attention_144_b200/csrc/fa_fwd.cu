// fa_fwd.cu -- forward pass of exact attention on sm_100a.
//
// O = softmax(scale Q K^T) V and the per-row log-sum-exp, FlashAttention-2
// style (LLM explainer page, sections 4.1-4.3 and 5.2): each work unit holds
// Q tiles of 128 rows of one (batch, head) and walks the K/V tiles; the online
// softmax keeps a running max m and running sum l per row and rescales the O
// accumulator when m grows (YOLO11 page, section 2.2).  S and P live only in
// tensor memory; O is written once per Q tile.
//
// Two persistent kernels, both one block per SM looping over work units:
//
// fa_fwd_pp_kernel (d = 64, 96, 128; 384 threads) -- two 128-row Q tiles per unit
//   warps 0-3  softmax + epilogue of Q tile 0 (thread t owns row t, TMEM lane t)
//   warps 4-7  softmax + epilogue of Q tile 1
//   warp  8    TMA producer: the Q pair once per unit, then K_j, V_j in turn
//   warp  9    TMEM allocator and the single-thread tcgen05.mma issuer
//   warps 10-11 idle (the block is three whole warpgroups so that registers
//              can move from the producer/MMA warpgroup to the softmax ones)
//   TMEM: S0 [0,128), S1 [128,256), O0 [256,256+d), O1 [256+d,256+2d).
//   MMA order per K/V tile j: P0.V_j, Q0 K_{j+1}^T, P1.V_j, Q1 K_{j+1}^T, so
//   the tensor cores work on one tile while the other tile's exponentials run,
//   and both Q tiles share every K/V tile loaded into shared memory.
//
// fa_fwd_kernel (any d, used for d = 256 and short sequences; 224 threads) --
//   one 128-row Q tile per unit, S double buffered in TMEM, 128-key K/V
//   tiles (at d = 256: 2 x 128 S columns + 256 O columns = all of TMEM, and
//   one K and one V stage of 64 KB)
//   warps 0-3 softmax + epilogue (through per-warp staging tiles), warp 4
//   Q/K producer, warp 5 V producer, warp 6 TMEM allocator + MMA issuer.
//
// Shared-memory tiles are rows of 64-element (128-byte, swizzled) chunks.  A
// d = 96 head uses two chunks a row: the second TMA box reaches past the
// head's last element and the tensor map fills those 32 columns with zeros
// (no memory is read for them); Q K^T contracts only the 96 real columns (six
// k-steps of 16) and P.V and the O accumulator are 96 columns wide.
//
// In both, P is consumed by the P.V MMA from tensor memory (A operand): written
// back over the first columns of its S buffer (16-bit P: BN/2 columns; E4M3 P
// from the 8-bit path: BN/4), or, in the d = 64 pair kernel, into its own
// columns.  O is rescaled only when a row's max grows by more than 2^8: until
// then P and l stay relative to the older max (P <= 2^8), which changes
// rounding only.
//
// When the units cannot fill the SMs, the K/V range is split and the partial
// results (fp32, normalised, base-2 LSE) are merged by fa_combine_kernel:
// O = sum_s 2^(LSE_s - LSE) O_s,  LSE = log2 sum_s 2^LSE_s.
#include "fa_common.cuh"
#include "fa_host.h"

namespace fa {

// How a unit's result leaves the block.
enum : int {
  kStoreWhole = 0,    // every K/V tile of the unit (or of its split-mode share)
  kStorePartial = 1,  // K/V tiles [t0 > 0, t1): normalised fp32 rows + LSE to the block's slot
  kStoreMerge = 2     // K/V tiles [0, t1 < n_kvt): merged with the partial rows of the
                      // blocks peer0 .. peer0 + npeer - 1, then stored
};

struct Unit {
  int u;  // unit index
  int b, h, qt, sp, t0, t1;
  int tb;    // batch coordinate of the unit's rows in memory (0 for a varlen batch)
  int tok0;  // first token of the unit's sequence along the token axis (varlen)
  int len;   // tokens in the unit's sequence
  int kind, peer0, npeer;
};

__host__ __device__ __forceinline__ int imin(int a, int b) { return a < b ? a : b; }

// First step of block c's range in the balanced schedule (c <= grid).
__host__ __device__ __forceinline__ int range_begin(const FwdSchedule& s, int c) {
  return c * s.iter_per + imin(c, s.iter_rem);
}

// VARLEN = false compiles the fixed-length location (s.cu is then unused).
template <bool VARLEN>
__host__ __device__ __forceinline__ void locate_seq(const FwdSchedule& s, int b, int& tb,
                                                   int& tok0, int& len) {
  seq_bounds(VARLEN ? s.cu : nullptr, b, s.N, s.total, tb, tok0, len);
}

// Unit u; t1 <= t0 when the unit holds no query row of its sequence (varlen).
template <bool VARLEN>
__host__ __device__ __forceinline__ Unit decode_unit(int u, const FwdSchedule& s) {
  Unit x;
  x.u = u;
  x.kind = kStoreWhole;
  x.peer0 = x.npeer = 0;
  if (s.causal) {
    // longest first: every head's last Q unit, then every head's second last,
    // ...; a unit needs the K/V tiles up to its last query row
    const int bh = u % (s.B * s.H), qi = u / (s.B * s.H);
    x.qt = s.n_qt - 1 - qi;
    x.sp = 0;
    x.h = bh % s.H;
    x.b = bh / s.H;
    locate_seq<VARLEN>(s, x.b, x.tb, x.tok0, x.len);
    x.t0 = 0;
    const int rows_end = imin(x.len, (x.qt + 1) * s.unit_rows);
    x.t1 = x.qt * s.unit_rows < x.len ? (rows_end + s.bn - 1) / s.bn : 0;
    return x;
  }
  x.qt = u % s.n_qt;
  int r = u / s.n_qt;
  x.sp = r % s.n_split;
  r /= s.n_split;
  x.h = r % s.H;
  x.b = r / s.H;
  locate_seq<VARLEN>(s, x.b, x.tb, x.tok0, x.len);
  x.t0 = x.sp * s.kvt_per_split;
  x.t1 = imin(x.t0 + s.kvt_per_split, (x.len + s.bn - 1) / s.bn);
  if (x.qt * s.unit_rows >= x.len) x.t1 = x.t0;  // no query row of this sequence
  return x;
}

// The units (or pieces of units) block `blk` processes, in order.  Every role
// of the block walks its own copy and sees the same sequence.
//   plain:    units blk, blk + grid, blk + 2 grid, ...
//   causal:   units in waves of grid, each wave walked in the opposite
//             direction of the one before (units come longest first, so a
//             block that took a long unit in one wave takes a short one in
//             the next)
//   balanced: the steps [range_begin(blk), range_begin(blk + 1)) cut at unit
//             boundaries.  Only a block's first piece can start inside a unit
//             (kStorePartial); the piece holding K/V tile 0 of a unit cut in
//             pieces is its block's last piece and merges the others
//             (kStoreMerge), whose blocks all come after it.
template <bool VARLEN>
struct UnitIter {
  int i, end, blk;
  __host__ __device__ __forceinline__ UnitIter(const FwdSchedule& s, int blk_) : blk(blk_) {
    if (s.n_iter > 0) {
      i = range_begin(s, blk);
      end = range_begin(s, blk + 1);
    } else if (s.causal) {
      i = 0;  // wave
      end = s.n_units;
    } else {
      i = blk;
      end = s.n_units;
    }
  }
  __host__ __device__ __forceinline__ bool next(const FwdSchedule& s, Unit& x) {
    if (s.n_iter == 0 && s.causal) {
      // a unit past the end in one wave means none in later waves either;
      // units without query rows (varlen) are skipped by every role alike
      for (;;) {
        const int u = i * s.grid + ((i & 1) ? s.grid - 1 - blk : blk);
        if (u >= end) return false;
        x = decode_unit<VARLEN>(u, s);
        ++i;
        if (x.t1 > x.t0) return true;
      }
    }
    if (s.n_iter == 0) {
      for (;;) {
        if (i >= end) return false;
        x = decode_unit<VARLEN>(i, s);
        i += s.grid;
        if (x.t1 > x.t0) return true;
      }
    }
    if (i >= end) return false;
    const int u = i / s.n_kvt;
    const int ubeg = u * s.n_kvt, uend = ubeg + s.n_kvt;
    x = decode_unit<VARLEN>(u, s);  // n_split = 1: the whole K/V range
    x.t0 = i - ubeg;
    x.t1 = imin(end, uend) - ubeg;
    if (x.t0 > 0) {
      x.kind = kStorePartial;
    } else if (x.t1 < s.n_kvt) {
      x.kind = kStoreMerge;
      x.peer0 = blk + 1;
      int c = x.peer0;
      while (c < s.grid && range_begin(s, c) < uend) ++c;
      x.npeer = c - x.peer0;
    }
    i = imin(end, uend);
    return true;
  }
};

struct FwdParams : FwdSchedule {
  void* o;          // [B, N, H, D] 16-bit, direct mode
  float* lse;       // [B, H, N] natural log, direct mode
  float* o_part;    // [S, B, N, H, D] fp32, split mode (null in direct mode)
  float* lse_part;  // [S, B, H, N] base-2 log, split mode
  float* bal_o;     // balanced: [grid, unit_rows, D] fp32 partial rows, normalised
  float* bal_lse;   // balanced: [grid, unit_rows] base-2 LSE of those rows
  unsigned* bal_flag;  // balanced: [grid] warps that have stored their partial rows; zeroed
  float sl2;        // scale * log2(e)
  float o_scale;    // factor applied to O when it is stored (the V descale; 1 for 16-bit)
  unsigned long long limit_ns;
  unsigned long long* status;
};

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* a) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}

// Timeout sites reported in the status word.
enum { kSiteQEmpty = 1, kSiteKEmpty, kSiteVEmpty, kSiteQFull, kSiteKFull, kSitePFull, kSiteVFull,
       kSiteSFull, kSiteODone, kSiteEpi, kSitePeer, kSiteSFree };

// Growth of the running max (base 2) tolerated before O is rescaled.
constexpr float kRescaleThreshold = 8.0f;

// Longest sequence whose forward epilogue goes through the staging tiles.
constexpr int kStagedMaxN = 1024;

// k-steps of a P.V product over K/V tile t that hold keys below the
// sequence's length len (16 keys a step for 16-bit P, 32 for 8-bit P): the
// ragged last tile needs only those, as P and V are zero past the end.
template <int BN, int EB>
__host__ __device__ __forceinline__ int pv_steps(int len, int t) {
  const int keys = len - t * BN < BN ? len - t * BN : BN;
  return (keys * EB + 31) / 32;
}


// ---------------------------------------------------------------------------
// One softmax step for the row a thread owns.  r holds the row's BN raw scores
// (fp32 bits, unscaled); columns >= valid are keys past N.  c = scale*log2(e).
// Updates the reference max m (base 2) and the running sum l, returns the
// factor alpha that O must be multiplied by (1 when the reference max is
// kept), and packs P = 2^(s*c - m) as 16-bit pairs into pk.
// EMU: of every 8 column pairs of a full tile, this many take their
// exponentials on the FMA pipe (ex2_poly2) instead of MUFU.  It pays where one
// softmax warp at a time keeps MUFU busy (the d = 128 ping-pong: 274 -> 266 us
// on the long-sequence workload); where two warps per SM sub-partition run
// their softmax together (d = 64) the extra instructions cost more than MUFU
// time saved (225 -> 241 us), so there it is 0.
// SKIP: partial tiles skip the 32-column chunks that hold no valid column of
// any row of the warp (warp votes; all 32 lanes must call together).
template <class T, int BN, int EMU = 0, bool SKIP = true>
__device__ __forceinline__ float softmax_step(const uint32_t (&r)[BN / 32][32], int valid, float c,
                                              float& m, float& l, uint32_t (&pk)[BN / 2]) {
  auto S = [&](int j) { return __uint_as_float(r[j / 32][j % 32]); };
  // full: every column of the row is valid.  With SKIP it is decided for the
  // whole warp: the partial path then takes warp votes, and a causal
  // diagonal tile holds full and partial rows in one warp (the partial path
  // is exact for full rows too).
  const bool full = SKIP ? __all_sync(0xffffffffu, valid >= BN) : valid >= BN;
  const bool neg = c < 0.f;
  // row max of s*c (the min of s when c < 0): 8 independent chains, two new
  // columns per three-input max
  float mx;
  if (full) {
    // the 8-column groups of the row: group 0 starts the chains, the rest
    // are taken two at a time, and an odd last group alone
    constexpr int NG = BN / 8;
    float part[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) part[q] = S(q);
    if (!neg) {
#pragma unroll
      for (int gi = 1; gi + 1 < NG; gi += 2)
#pragma unroll
        for (int q = 0; q < 8; ++q)
          part[q] = max3f(part[q], S(8 * gi + q), S(8 * gi + 8 + q));
      if constexpr ((NG - 1) % 2 == 1) {
#pragma unroll
        for (int q = 0; q < 8; ++q) part[q] = fmaxf(part[q], S(BN - 8 + q));
      }
      mx = max3f(max3f(part[0], part[1], part[2]), max3f(part[3], part[4], part[5]),
                 fmaxf(part[6], part[7]));
    } else {
#pragma unroll
      for (int gi = 1; gi + 1 < NG; gi += 2)
#pragma unroll
        for (int q = 0; q < 8; ++q)
          part[q] = min3f(part[q], S(8 * gi + q), S(8 * gi + 8 + q));
      if constexpr ((NG - 1) % 2 == 1) {
#pragma unroll
        for (int q = 0; q < 8; ++q) part[q] = fminf(part[q], S(BN - 8 + q));
      }
      mx = min3f(min3f(part[0], part[1], part[2]), min3f(part[3], part[4], part[5]),
                 fminf(part[6], part[7]));
    }
  } else {
    // a partial tile (the ragged end of the keys, or the causal diagonal):
    // 32-column chunks past every valid column of the warp's rows are skipped
    float part[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) part[q] = neg ? INFINITY : -INFINITY;
#pragma unroll
    for (int q = 0; q < BN / 32; ++q)
      if (!SKIP || __any_sync(0xffffffffu, q * 32 < valid)) {
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const int j = q * 32 + jj;
          if (j < valid) part[j & 7] = neg ? fminf(part[j & 7], S(j)) : fmaxf(part[j & 7], S(j));
        }
      }
    if (!neg)
      mx = fmaxf(fmaxf(fmaxf(part[0], part[1]), fmaxf(part[2], part[3])),
                 fmaxf(fmaxf(part[4], part[5]), fmaxf(part[6], part[7])));
    else
      mx = fminf(fminf(fminf(part[0], part[1]), fminf(part[2], part[3])),
                 fminf(fminf(part[4], part[5]), fminf(part[6], part[7])));
  }
  const float mc = mx * c;  // max of s*c over the valid columns
  float alpha = 1.f;
  if (mc > m + kRescaleThreshold) {
    alpha = ex2(m - mc);  // m = -inf on the first tile: alpha = 0
    m = mc;
  }
  const float neg_m = -m;
  float rs;
  if (full) {
    // x = s*c - m two columns per packed FMA; four packed running sums
    const uint64_t c2 = f32x2(c, c), n2 = f32x2(neg_m, neg_m);
    float sum[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) sum[q] = 0.f;
#pragma unroll
    for (int j = 0; j < BN / 2; ++j) {
      float x0, x1, p0, p1;
      fma2(x0, x1, S(2 * j), S(2 * j + 1), c2, n2);
      if ((j & 7) >= 8 - EMU) {
        ex2_poly2(p0, p1, x0, x1);
      } else {
        p0 = ex2(x0);
        p1 = ex2(x1);
      }
      add2(sum[2 * (j & 3)], sum[2 * (j & 3) + 1], p0, p1);
      pk[j] = Elem<T>::pack(p0, p1);
    }
    add2(sum[0], sum[1], sum[4], sum[5]);
    add2(sum[2], sum[3], sum[6], sum[7]);
    add2(sum[0], sum[1], sum[2], sum[3]);
    rs = sum[0] + sum[1];
  } else {
    float sum[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) sum[q] = 0.f;
#pragma unroll
    for (int q = 0; q < BN / 32; ++q) {
      if (!SKIP || __any_sync(0xffffffffu, q * 32 < valid)) {
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const int j = q * 16 + jj;
          const float p0 = (2 * j < valid) ? ex2(fmaf(S(2 * j), c, neg_m)) : 0.f;
          const float p1 = (2 * j + 1 < valid) ? ex2(fmaf(S(2 * j + 1), c, neg_m)) : 0.f;
          sum[j & 7] += p0 + p1;
          pk[j] = Elem<T>::pack(p0, p1);
        }
      } else {
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) pk[q * 16 + jj] = 0u;  // P = 0: finite for P.V
      }
    }
    rs = ((sum[0] + sum[1]) + (sum[2] + sum[3])) + ((sum[4] + sum[5]) + (sum[6] + sum[7]));
  }
  l = l * alpha + rs;
  return alpha;
}

// Writes this thread's packed P row (pk from softmax_step) into tensor memory
// at taddr, where the P.V product reads it as its A operand: 16-bit P two
// keys a column (BN/2 columns); 8-bit P four keys a column (BN/4 columns),
// key 4i in the low byte of column i.
template <class T, int BN>
__device__ __forceinline__ void store_p(uint32_t taddr, const uint32_t (&pk)[BN / 2]) {
  if constexpr (Elem<T>::kBytes == 2) {
#pragma unroll
    for (int q = 0; q < BN / 32; ++q) tmem_st16(taddr + q * 16, &pk[q * 16]);
  } else {
    static_assert(BN % 128 == 0, "8-bit P is written 32 columns at a time");
#pragma unroll
    for (int q = 0; q < BN / 128; ++q) {
      uint32_t w[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) w[i] = pk[q * 64 + 2 * i] | (pk[q * 64 + 2 * i + 1] << 16);
      tmem_st32(taddr + q * 32, w);
    }
  }
}

// Multiplies this thread's O row (D fp32 columns at taddr) by alpha.
template <int D>
__device__ __forceinline__ void rescale_o(uint32_t taddr, float alpha) {
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    uint32_t o[32];
    tmem_ld32(taddr + c * 32, o);
    tmem_wait_ld();
    reg_fence(o);
#pragma unroll
    for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
    tmem_st32(taddr + c * 32, o);
  }
  tmem_wait_st();
}

// Epilogue for one row: O = O_acc / l (16-bit, or fp32 partial in split mode)
// and the LSE (natural log, or base 2 in split mode).  Collective over the warp.
// Balanced schedule: a kStorePartial piece stores its rows into the block's
// slot; a kStoreMerge piece first waits (bounded) until every peer block's 8
// softmax warps have stored theirs, then merges
//   O = sum_x 2^(LSE_x - L) O_x,  L = log2 sum_x 2^LSE_x  (x = own + peers).
// Returns false when a wait gave up.
template <class T, int D>
__device__ __forceinline__ bool store_row(const FwdParams& p, const Unit& un, uint32_t taddr,
                                          int q_row, float m, float l, const WaitCtl& w) {
  const bool live = q_row < un.len;
  // the row's token along the memory token axis (p.total tokens a batch entry)
  const size_t tok = (size_t)un.tb * p.total + un.tok0 + q_row;
  const size_t lse_at = ((size_t)un.tb * p.H + un.h) * p.total + un.tok0 + q_row;
  const float inv_l = p.o_scale / l;
  const float lse2 = m + lg2(l);
  if (un.kind == kStorePartial) {
    const int ur = q_row - un.qt * p.unit_rows;
    float* orow = p.bal_o + ((size_t)blockIdx.x * p.unit_rows + ur) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      tmem_ld32(taddr + c * 32, o);
      tmem_wait_ld();
      reg_fence(o);
      if (live) {
        float4* dst = reinterpret_cast<float4*>(orow + c * 32);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          dst[j] = make_float4(__uint_as_float(o[4 * j]) * inv_l,
                               __uint_as_float(o[4 * j + 1]) * inv_l,
                               __uint_as_float(o[4 * j + 2]) * inv_l,
                               __uint_as_float(o[4 * j + 3]) * inv_l);
      }
    }
    if (live) p.bal_lse[(size_t)blockIdx.x * p.unit_rows + ur] = lse2;
    __threadfence();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) atomicAdd(p.bal_flag + blockIdx.x, 1u);
    return true;
  }
  if (un.kind == kStoreMerge) {
    const int ur = q_row - un.qt * p.unit_rows;
    bool good = true;
    for (int c = un.peer0; c < un.peer0 + un.npeer && good; ++c) {
      const uint64_t t0 = global_ns();
      for (uint32_t it = 1; ld_acquire_gpu(p.bal_flag + c) < 8u; ++it) {
        if ((it & 63u) == 0) {
          if (*w.abort) { good = false; break; }
          if (global_ns() - t0 > w.limit_ns) {
            report_timeout(w.status, kSitePeer);
            *w.abort = 1;
            good = false;
            break;
          }
        }
      }
    }
    if (!__all_sync(0xffffffffu, good)) return false;
    float mx = lse2;
    if (live)
      for (int c = un.peer0; c < un.peer0 + un.npeer; ++c)
        mx = fmaxf(mx, __ldcg(p.bal_lse + (size_t)c * p.unit_rows + ur));
    float tot = ex2(lse2 - mx);
    if (live)
      for (int c = un.peer0; c < un.peer0 + un.npeer; ++c)
        tot += ex2(__ldcg(p.bal_lse + (size_t)c * p.unit_rows + ur) - mx);
    const float L2 = mx + lg2(tot);
    const float w_own = ex2(lse2 - L2) * inv_l;
    T* orow = reinterpret_cast<T*>(p.o) + (tok * p.H + un.h) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      tmem_ld32(taddr + c * 32, o);
      tmem_wait_ld();
      reg_fence(o);
      float acc[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] = __uint_as_float(o[j]) * w_own;
      if (live) {
        for (int pc = un.peer0; pc < un.peer0 + un.npeer; ++pc) {
          const float wp = ex2(__ldcg(p.bal_lse + (size_t)pc * p.unit_rows + ur) - L2);
          const float4* src = reinterpret_cast<const float4*>(
              p.bal_o + ((size_t)pc * p.unit_rows + ur) * D + c * 32);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 v = __ldcg(src + j);
            acc[4 * j] = fmaf(wp, v.x, acc[4 * j]);
            acc[4 * j + 1] = fmaf(wp, v.y, acc[4 * j + 1]);
            acc[4 * j + 2] = fmaf(wp, v.z, acc[4 * j + 2]);
            acc[4 * j + 3] = fmaf(wp, v.w, acc[4 * j + 3]);
          }
        }
        uint4 pkd[4];
        uint32_t* pw = reinterpret_cast<uint32_t*>(pkd);
#pragma unroll
        for (int j = 0; j < 16; ++j) pw[j] = Elem<T>::pack(acc[2 * j], acc[2 * j + 1]);
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[j] = pkd[j];
      }
    }
    if (live) p.lse[lse_at] = L2 * kLn2;
    return true;
  }
  if (p.o_part == nullptr) {
    T* orow = reinterpret_cast<T*>(p.o) + (tok * p.H + un.h) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      tmem_ld32(taddr + c * 32, o);
      tmem_wait_ld();
      reg_fence(o);
      uint4 pkd[4];
      uint32_t* pw = reinterpret_cast<uint32_t*>(pkd);
#pragma unroll
      for (int j = 0; j < 16; ++j)
        pw[j] = Elem<T>::pack(__uint_as_float(o[2 * j]) * inv_l,
                              __uint_as_float(o[2 * j + 1]) * inv_l);
      if (live) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[j] = pkd[j];
      }
    }
    if (live) p.lse[lse_at] = lse2 * kLn2;
  } else {
    float* orow = p.o_part + ((((size_t)un.sp * p.B + un.b) * p.N + q_row) * p.H + un.h) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      tmem_ld32(taddr + c * 32, o);
      tmem_wait_ld();
      reg_fence(o);
      if (live) {
        float4* dst = reinterpret_cast<float4*>(orow + c * 32);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          dst[j] = make_float4(__uint_as_float(o[4 * j]) * inv_l,
                               __uint_as_float(o[4 * j + 1]) * inv_l,
                               __uint_as_float(o[4 * j + 2]) * inv_l,
                               __uint_as_float(o[4 * j + 3]) * inv_l);
      }
    }
    if (live) p.lse_part[(((size_t)un.sp * p.B + un.b) * p.H + un.h) * p.N + q_row] = lse2;
  }
  return true;
}

// Epilogue of a whole unit's row in direct mode (O rounded to 16 bits, LSE
// natural log) through a per-warp staging tile in shared memory: each thread
// writes its row's 16-byte chunks there (chunk u of row r at position
// u ^ (r & 7): conflict-free), then the warp writes the tile back row by row,
// each store instruction covering RPI whole rows (one 16-byte chunk a lane),
// instead of every store touching 32 rows.  stg: the warp's 32 x D x 2-byte
// tile.  Collective over the warp.
template <class T, int D>
__device__ __forceinline__ void store_row_staged(const FwdParams& p, const Unit& un, uint32_t taddr,
                                                 int q_row, float m, float l, uint8_t* stg) {
  constexpr int CPR = D * 2 / 16;  // 16-byte chunks a row
  constexpr int RPI = 32 / CPR;    // rows a warp store instruction covers
  const int lane = threadIdx.x & 31;
  const float inv_l = p.o_scale / l;
  const float lse2 = m + lg2(l);
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    uint32_t o[32];
    tmem_ld32(taddr + c * 32, o);
    tmem_wait_ld();
    reg_fence(o);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint4 v;
      v.x = Elem<T>::pack(__uint_as_float(o[8 * u]) * inv_l, __uint_as_float(o[8 * u + 1]) * inv_l);
      v.y = Elem<T>::pack(__uint_as_float(o[8 * u + 2]) * inv_l,
                          __uint_as_float(o[8 * u + 3]) * inv_l);
      v.z = Elem<T>::pack(__uint_as_float(o[8 * u + 4]) * inv_l,
                          __uint_as_float(o[8 * u + 5]) * inv_l);
      v.w = Elem<T>::pack(__uint_as_float(o[8 * u + 6]) * inv_l,
                          __uint_as_float(o[8 * u + 7]) * inv_l);
      const int chunk = c * 4 + u;
      *reinterpret_cast<uint4*>(stg + lane * (CPR * 16) + ((chunk ^ (lane & 7)) * 16)) = v;
    }
  }
  const int row0 = q_row - lane;  // the warp's first row (q_row = row0 + lane)
  if (q_row < un.len)
    p.lse[((size_t)un.tb * p.H + un.h) * p.total + un.tok0 + q_row] = lse2 * kLn2;
  __syncwarp();
  const int sub = lane / CPR, chunk = lane % CPR;
#pragma unroll
  for (int it = 0; it < 32 / RPI; ++it) {
    const int r = it * RPI + sub;
    const uint4 v = *reinterpret_cast<const uint4*>(stg + r * (CPR * 16) + ((chunk ^ (r & 7)) * 16));
    if (row0 + r < un.len) {
      const size_t tok = (size_t)un.tb * p.total + un.tok0 + row0 + r;
      reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.o) + (tok * p.H + un.h) * D)[chunk] = v;
    }
  }
  __syncwarp();  // the tile is rewritten by the next unit's epilogue
}

// Epilogue of one row in direct or split mode, through the warp's 4 KB
// staging tile, 32 columns at a time: each thread writes its row's 32 output
// values there (16-byte unit u of row r at unit position u ^ (r % units a
// row)), then each warp store instruction covers whole 128-byte row pieces
// (4 rows of fp32 partials, or 8 rows of 16-bit O) instead of 16 bytes of 32
// rows.  PART: normalised fp32 partial rows and base-2 LSE of a K/V split;
// otherwise O rounded to T and the natural-log LSE.  Collective over the warp.
template <class T, int D, bool PART>
__device__ __forceinline__ void store_row_chunked(const FwdParams& p, const Unit& un,
                                                  uint32_t taddr, int q_row, float m, float l,
                                                  uint8_t* stg) {
  constexpr int EBO = PART ? 4 : 2;  // bytes an output element
  constexpr int RB = 32 * EBO;       // bytes of a row's 32-column piece
  constexpr int UPR = RB / 16;       // 16-byte units a piece: 8 or 4
  constexpr int RPI = 32 / UPR;      // rows a warp store instruction covers
  const int lane = threadIdx.x & 31;
  const float inv_l = p.o_scale / l;
  const float lse2 = m + lg2(l);
  const int row0 = q_row - lane;  // the warp's first row
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t o[32];
    tmem_ld32(taddr + c * 32, o);
    tmem_wait_ld();
    reg_fence(o);
#pragma unroll
    for (int u = 0; u < UPR; ++u) {
      uint4 v;
      if constexpr (PART) {
        v = make_uint4(__float_as_uint(__uint_as_float(o[4 * u]) * inv_l),
                       __float_as_uint(__uint_as_float(o[4 * u + 1]) * inv_l),
                       __float_as_uint(__uint_as_float(o[4 * u + 2]) * inv_l),
                       __float_as_uint(__uint_as_float(o[4 * u + 3]) * inv_l));
      } else {
        v.x = Elem<T>::pack(__uint_as_float(o[8 * u]) * inv_l, __uint_as_float(o[8 * u + 1]) * inv_l);
        v.y = Elem<T>::pack(__uint_as_float(o[8 * u + 2]) * inv_l,
                            __uint_as_float(o[8 * u + 3]) * inv_l);
        v.z = Elem<T>::pack(__uint_as_float(o[8 * u + 4]) * inv_l,
                            __uint_as_float(o[8 * u + 5]) * inv_l);
        v.w = Elem<T>::pack(__uint_as_float(o[8 * u + 6]) * inv_l,
                            __uint_as_float(o[8 * u + 7]) * inv_l);
      }
      *reinterpret_cast<uint4*>(stg + lane * RB + ((u ^ (lane & (UPR - 1))) * 16)) = v;
    }
    __syncwarp();
    const int u = lane % UPR;
#pragma unroll
    for (int it = 0; it < 32 / RPI; ++it) {
      const int r = it * RPI + lane / UPR;
      const uint4 v = *reinterpret_cast<const uint4*>(stg + r * RB + ((u ^ (r & (UPR - 1))) * 16));
      const int row = row0 + r;
      if (row < un.len) {
        if constexpr (PART) {
          float* orow =
              p.o_part + ((((size_t)un.sp * p.B + un.b) * p.N + row) * p.H + un.h) * D + c * 32;
          reinterpret_cast<uint4*>(orow)[u] = v;
        } else {
          const size_t tok = (size_t)un.tb * p.total + un.tok0 + row;
          T* orow = reinterpret_cast<T*>(p.o) + (tok * p.H + un.h) * D + c * 32;
          reinterpret_cast<uint4*>(orow)[u] = v;
        }
      }
    }
    __syncwarp();  // the tile is rewritten by the next piece
  }
  if (q_row < un.len) {
    if constexpr (PART)
      p.lse_part[(((size_t)un.sp * p.B + un.b) * p.H + un.h) * p.N + q_row] = lse2;
    else
      p.lse[((size_t)un.tb * p.H + un.h) * p.total + un.tok0 + q_row] = lse2 * kLn2;
  }
}

// ===========================================================================
// fa_fwd_pp_kernel: two Q tiles per unit
// ===========================================================================
template <int D_, int KST_, int VST_, int EB_ = 2, int EMU_ = -1, int DUAL_ = -1>
struct FwdPPTraits {
  static constexpr int D = D_;
  static constexpr int EB = EB_;          // bytes an element of Q, K, V
  static constexpr int CH_ELEMS = 128 / EB;  // elements in a 128-byte chunk
  static constexpr int BM = 128;  // rows per Q tile; a unit holds two
  static constexpr int BN = 128;
  static constexpr int KST = KST_;
  static constexpr int VST = VST_;
  // 128-byte chunks along d; at d = 96 the second chunk's last 32 columns
  // are the tensor map's zero fill and only the first 96 are contracted
  static constexpr int KCH = (D * EB + 127) / 128;
  static constexpr int QT_BYTES = BM * KCH * 128;
  static constexpr int KV_BYTES = BN * KCH * 128;
  static constexpr int P_COLS = BN * EB / 4;  // TMEM columns of one packed P tile
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * QT_BYTES;
  static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
  // d = 64: the epilogue's per-warp O staging tiles (8 warps x 32 rows)
  static constexpr int STG_BYTES = (D == 64 && EB == 2) ? 8 * 32 * D * 2 : 0;
  static constexpr int OFF_STG = OFF_V + VST * KV_BYTES;
  static constexpr int OFF_BAR = OFF_STG + STG_BYTES;
  static constexpr int B_Q_FULL = 0, B_Q_EMPTY = 1, B_K_FULL = 2, B_K_EMPTY = B_K_FULL + KST,
                       B_V_FULL = B_K_EMPTY + KST, B_V_EMPTY = B_V_FULL + VST,
                       B_S_FULL = B_V_EMPTY + VST, B_P_FULL = B_S_FULL + 2,
                       B_O_DONE = B_P_FULL + 2, B_S_FREE = B_O_DONE + 2,
                       B_DRAIN = B_S_FREE + 2, NUM_BARS = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  // P in its own tensor-memory columns when they fit (d = 64: S 2 x 128, P
  // 2 x 64, O 2 x 64 = 512): Q K^T of the next K/V tile may then overwrite S
  // as soon as the softmax warps have read it, before P.V has consumed P.
  // Otherwise (d = 128) P is written over the first BN/2 columns of its S.
  static constexpr bool SEP_P = 2 * BN + 2 * P_COLS + 2 * D <= 512;
  // DUAL: each Q tile's products are issued by its own thread (warp 9:
  // tile 0, warp 10: tile 1); the release barriers of the K and V stages and
  // of the Q pair then count one commit from each.  Where P has its own
  // columns (d = 64): measured on B200, [4,4096,8,64] 228.6 -> 213.7 us.
  // Where P is written over S (d = 96, 128, 8-bit) the products of both
  // tiles share one issuer: two measured far slower there ([1,8192,8,128]:
  // 284.6 -> 363.9 us).
  static constexpr bool DUAL = DUAL_ >= 0 ? DUAL_ != 0 : SEP_P;
  // Short-sequence measures (warps with no live row skip the softmax, the
  // ragged last K/V tile skips its empty 32-column chunks and P.V k-steps):
  // taken where P has its own columns; the d = 96, 128 and 8-bit kernels,
  // bound by the tensor-core issue rate, keep their plain loops (with the
  // measures, [1,8192,8,128] took 284.6 us against 272.9 us).
  static constexpr bool SHORT = SEP_P;
  static_assert(!SHORT || STG_BYTES > 0, "the short-sequence kernel stages its epilogue");
  static constexpr int NISSUE = DUAL ? 2 : 1;
  // exponentials on the FMA pipe per 8 column pairs (see softmax_step): the
  // d = 128 warpgroups take turns, the d = 64 ones run together.  Measured on
  // B200 for d = 128 (bf16 / 8-bit, [1,8192,8,128], us): 1: 269.6 / 243.0,
  // 2: 271.6 / 238.8, 3: 284.0 / 245.1 -- 2 is kept
  static constexpr int EMU = EMU_ >= 0 ? EMU_ : (SEP_P ? 0 : 2);
  static constexpr uint32_t TM_P = 2 * BN;                      // used when SEP_P
  static constexpr uint32_t TM_O = SEP_P ? 3 * BN : 2 * BN;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(TM_O + 2 * D <= 512, "tensor memory budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <class T, class Tr, bool VARLEN>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_pp_kernel(const __grid_constant__ CUtensorMap tmq,
                     const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv, const FwdParams p) {
  constexpr int D = Tr::D, BN = Tr::BN, BM = Tr::BM, KST = Tr::KST, VST = Tr::VST;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + Tr::OFF_Q, sK = base + Tr::OFF_K, sV = base + Tr::OFF_V;
  const uint32_t bars = base + Tr::OFF_BAR;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + Tr::OFF_MISC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + Tr::OFF_MISC + 4);
  auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitCtl w{abort_flag, p.limit_ns, p.status};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(Tr::B_Q_FULL), 1);
    mbar_init(bar(Tr::B_Q_EMPTY), Tr::NISSUE);
    for (int s = 0; s < KST; ++s) {
      mbar_init(bar(Tr::B_K_FULL + s), 1);
      mbar_init(bar(Tr::B_K_EMPTY + s), Tr::NISSUE);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(bar(Tr::B_V_FULL + s), 1);
      mbar_init(bar(Tr::B_V_EMPTY + s), Tr::NISSUE);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(Tr::B_S_FULL + s), 1);
      mbar_init(bar(Tr::B_P_FULL + s), 128);
      mbar_init(bar(Tr::B_O_DONE + s), 1);
      mbar_init(bar(Tr::B_S_FREE + s), 128);
    }
    mbar_init(bar(Tr::B_DRAIN), Tr::NISSUE);
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), Tr::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmq);
    tma_prefetch_desc(&tmk);
    tma_prefetch_desc(&tmv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= 8) {
    regs_shrink();  // all four warps of the producer/MMA warpgroup
  if (warp == 8) {
    // ------------------------------------------------------- producer
    {
      const bool leader = lane == 0;  // issues; all lanes run the loop
      uint32_t kc = 0, vc = 0, qc = 0;
      bool ok = true;
      UnitIter<VARLEN> it(p, blockIdx.x);
      for (Unit un; ok && it.next(p, un);) {
        if (qc > 0 && !(ok = mbar_wait_warp(bar(Tr::B_Q_EMPTY), (qc - 1) & 1u, w, kSiteQEmpty))) break;
        mbar_expect_tx(leader, bar(Tr::B_Q_FULL), 2 * Tr::QT_BYTES);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int c = 0; c < Tr::KCH; ++c)
            tma_load_4d(leader, sQ + t * Tr::QT_BYTES + c * (BM * 128), &tmq, bar(Tr::B_Q_FULL),
                        c * Tr::CH_ELEMS,
                        un.h, un.tok0 + (2 * un.qt + t) * BM, un.tb);
        ++qc;
        for (int t = un.t0; t < un.t1; ++t) {
          const uint32_t ks = kc % KST;
          if (kc >= (uint32_t)KST &&
              !(ok = mbar_wait_warp(bar(Tr::B_K_EMPTY + ks), ((kc / KST) - 1) & 1u, w, kSiteKEmpty)))
            break;
          mbar_expect_tx(leader, bar(Tr::B_K_FULL + ks), Tr::KV_BYTES);
#pragma unroll
          for (int c = 0; c < Tr::KCH; ++c)
            tma_load_4d(leader, sK + ks * Tr::KV_BYTES + c * (BN * 128), &tmk, bar(Tr::B_K_FULL + ks),
                        c * Tr::CH_ELEMS, un.h, un.tok0 + t * BN, un.tb);
          ++kc;
          const uint32_t vs = vc % VST;
          if (vc >= (uint32_t)VST &&
              !(ok = mbar_wait_warp(bar(Tr::B_V_EMPTY + vs), ((vc / VST) - 1) & 1u, w, kSiteVEmpty)))
            break;
          mbar_expect_tx(leader, bar(Tr::B_V_FULL + vs), Tr::KV_BYTES);
#pragma unroll
          for (int c = 0; c < Tr::KCH; ++c)
            tma_load_4d(leader, sV + vs * Tr::KV_BYTES + c * (BN * 128), &tmv, bar(Tr::B_V_FULL + vs),
                        c * Tr::CH_ELEMS, un.h, un.tok0 + t * BN, un.tb);
          ++vc;
        }
      }
      // Every issued load must land before the block exits.
      if (qc > 0) mbar_drain(bar(Tr::B_Q_FULL), (qc - 1) & 1u, p.limit_ns);
      for (uint32_t s = 0; s < (uint32_t)KST; ++s)
        if (kc > s) mbar_drain(bar(Tr::B_K_FULL + s), ((kc - 1 - s) / KST) & 1u, p.limit_ns);
      for (uint32_t s = 0; s < (uint32_t)VST; ++s)
        if (vc > s) mbar_drain(bar(Tr::B_V_FULL + s), ((vc - 1 - s) / VST) & 1u, p.limit_ns);
    }
    __syncwarp();
  } else if (warp == 9 || (Tr::DUAL && warp == 10)) {
    // ---------------------------------------------------- MMA issuer(s)
    {
      const bool leader = lane == 0;  // issues; all lanes run the loop
      constexpr uint32_t kIdescQK = f16_idesc(Elem<T>::kFmt, 128, BN, false);
      constexpr uint32_t kIdescPV = f16_idesc(Elem<T>::kFmt, 128, D, true);
      uint32_t kc = 0, vc = 0, g = 0, uc = 0;
      bool ok = true;
      // Descriptors are built once; each MMA only advances a start address.
      const uint64_t q_desc0 = sw128_desc(sQ, 16, 1024), k_desc0 = sw128_desc(sK, 16, 1024),
                     v_desc0 = sw128_desc(sV, BN * 128, 1024);
      // S_t = Q_t K^T for the K stage of counter kc (t = 0, 1)
      auto issue_qk = [&](int t) {
        const uint64_t kd = desc_advance(k_desc0, (kc % KST) * Tr::KV_BYTES);
        const uint64_t qd = desc_advance(q_desc0, t * Tr::QT_BYTES);
#pragma unroll
        for (int kk = 0; kk < D * Tr::EB / 32; ++kk) {  // 32 bytes of each row a step
          const uint32_t ch = kk >> 2, in = (kk & 3) * 32;
          mma_ss<T>(leader, tmem + t * BN, desc_advance(qd, ch * (BM * 128) + in),
                  desc_advance(kd, ch * (BN * 128) + in), kIdescQK, kk > 0 ? 1u : 0u);
        }
      };
      // O_t (+)= P_t V for the V stage of counter vc; only the k-steps that
      // hold keys below the sequence's end (P and V are zero past it)
      auto issue_pv = [&](int t, bool first, int nsteps) {
        constexpr int kSteps = BN * Tr::EB / 32;  // 32 keys x 16 bits, or 32 x 8 bits
        const uint64_t vd = desc_advance(v_desc0, (vc % VST) * Tr::KV_BYTES);
        const uint32_t pa = Tr::SEP_P ? Tr::TM_P + t * Tr::P_COLS : t * BN;
        if (nsteps >= kSteps) {
#pragma unroll
          for (int kk = 0; kk < kSteps; ++kk)
            mma_ts<T>(leader, tmem + Tr::TM_O + t * D, tmem + pa + kk * 8,
                      desc_advance(vd, kk * (32 / Tr::EB) * 128), kIdescPV,
                      (!first || kk > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < kSteps; ++kk)
            mma_ts<T>(leader && kk < nsteps, tmem + Tr::TM_O + t * D, tmem + pa + kk * 8,
                      desc_advance(vd, kk * (32 / Tr::EB) * 128), kIdescPV,
                      (!first || kk > 0) ? 1u : 0u);
        }
      };
      UnitIter<VARLEN> it(p, blockIdx.x);
      if constexpr (Tr::DUAL) {
        // Issuer t (warp 9 + t) owns Q tile t and walks its chain alone:
        // S_t(j) = Q_t K_j^T -> softmax of warpgroup t -> O_t += P_t(j) V_j, so
        // neither tile waits for the other tile's softmax.  With P in its own
        // columns S_t(j+1) is issued as soon as warpgroup t has read S_t(j)
        // into registers, ahead of P_t(j) V_j (the tensor cores compute the
        // next scores while the exponentials run); with P written over S it
        // follows P_t(j) V_j, which has read P (same thread: in order).
        const int t = warp - 9;
        uint32_t gs = 0;  // S tiles this issuer has issued
        auto issue_s = [&](int j, int n) -> bool {
          if (!mbar_wait_warp(bar(Tr::B_K_FULL + kc % KST), (kc / KST) & 1u, w, kSiteKFull))
            return false;
          if (Tr::SEP_P && gs > 0 &&
              !mbar_wait_warp(bar(Tr::B_S_FREE + t), (gs - 1) & 1u, w, kSiteSFree))
            return false;
          tc_fence_after();
          issue_qk(t);
          umma_commit(leader, bar(Tr::B_S_FULL + t));
          umma_commit(leader, bar(Tr::B_K_EMPTY + kc % KST));
          if (j == n - 1) umma_commit(leader, bar(Tr::B_Q_EMPTY));
          ++kc;
          ++gs;
          return true;
        };
        auto issue_o = [&](const Unit& un, int j) -> bool {
          if (!mbar_wait_warp(bar(Tr::B_P_FULL + t), g & 1u, w, kSitePFull)) return false;
          if (!mbar_wait_warp(bar(Tr::B_V_FULL + vc % VST), (vc / VST) & 1u, w, kSiteVFull))
            return false;
          tc_fence_after();
          issue_pv(t, j == 0, pv_steps<BN, Tr::EB>(un.len, un.t0 + j));
          umma_commit(leader, bar(Tr::B_O_DONE + t));
          umma_commit(leader, bar(Tr::B_V_EMPTY + vc % VST));
          ++vc;
          ++g;
          return true;
        };
        for (Unit un; ok && it.next(p, un);) {
          const int n = un.t1 - un.t0;
          if (!(ok = mbar_wait_warp(bar(Tr::B_Q_FULL), uc & 1u, w, kSiteQFull))) break;
          ok = issue_s(0, n);
          for (int j = 0; j < n && ok; ++j) {
            if (Tr::SEP_P) {
              if (j + 1 < n && !(ok = issue_s(j + 1, n))) break;
              ok = issue_o(un, j);
            } else {
              if (!(ok = issue_o(un, j))) break;
              if (j + 1 < n) ok = issue_s(j + 1, n);
            }
          }
          if (!ok) break;
          ++uc;
        }
      } else
      for (Unit un; ok && it.next(p, un);) {
        const int n = un.t1 - un.t0;
        if (!(ok = mbar_wait_warp(bar(Tr::B_Q_FULL), uc & 1u, w, kSiteQFull))) break;
        if (!(ok = mbar_wait_warp(bar(Tr::B_K_FULL + kc % KST), (kc / KST) & 1u, w, kSiteKFull))) break;
        tc_fence_after();
        issue_qk(0);
        umma_commit(leader, bar(Tr::B_S_FULL + 0));
        issue_qk(1);
        umma_commit(leader, bar(Tr::B_S_FULL + 1));
        umma_commit(leader, bar(Tr::B_K_EMPTY + kc % KST));
        if (n == 1) umma_commit(leader, bar(Tr::B_Q_EMPTY));
        ++kc;
        for (int j = 0; j < n; ++j, ++g) {
          // tile 0: P0 V_j, then S0 for the next K tile
          if (!(ok = mbar_wait_warp(bar(Tr::B_P_FULL + 0), g & 1u, w, kSitePFull))) break;
          if (!(ok = mbar_wait_warp(bar(Tr::B_V_FULL + vc % VST), (vc / VST) & 1u, w, kSiteVFull)))
            break;
          tc_fence_after();
          const int nsteps = Tr::SHORT ? pv_steps<BN, Tr::EB>(un.len, un.t0 + j) : BN * Tr::EB / 32;
          issue_pv(0, j == 0, nsteps);
          umma_commit(leader, bar(Tr::B_O_DONE + 0));
          const bool more = j + 1 < n;
          if (more) {
            if (!(ok = mbar_wait_warp(bar(Tr::B_K_FULL + kc % KST), (kc / KST) & 1u, w, kSiteKFull)))
              break;
            tc_fence_after();
            issue_qk(0);
            umma_commit(leader, bar(Tr::B_S_FULL + 0));
          }
          // tile 1: P1 V_j, then S1 for the next K tile
          if (!(ok = mbar_wait_warp(bar(Tr::B_P_FULL + 1), g & 1u, w, kSitePFull))) break;
          tc_fence_after();
          issue_pv(1, j == 0, nsteps);
          umma_commit(leader, bar(Tr::B_O_DONE + 1));
          umma_commit(leader, bar(Tr::B_V_EMPTY + vc % VST));
          ++vc;
          if (more) {
            issue_qk(1);
            umma_commit(leader, bar(Tr::B_S_FULL + 1));
            umma_commit(leader, bar(Tr::B_K_EMPTY + kc % KST));
            if (j + 2 == n) umma_commit(leader, bar(Tr::B_Q_EMPTY));
            ++kc;
          }
        }
        if (!ok) break;
        ++uc;
      }
      // Every issued MMA must finish before tensor memory is released.
      umma_commit(leader, bar(Tr::B_DRAIN));
      mbar_drain(bar(Tr::B_DRAIN), 0, p.limit_ns);
    }
    __syncwarp();
  }  // warps 10 and 11 have no role
  } else {
    regs_grow();  // both compute warpgroups
    // ------------------------------- softmax and epilogue, Q tile wg
    const int wg = warp >> 2;           // which Q tile
    const int row = threadIdx.x & 127;  // row within the tile = TMEM lane
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t s_col = tl + wg * BN;
    const uint32_t p_col = tl + Tr::TM_P + wg * Tr::P_COLS;  // used when SEP_P
    const uint32_t o_col = tl + Tr::TM_O + wg * D;
    const float c = p.sl2;
    uint32_t g = 0;
    bool ok = true;
    UnitIter<VARLEN> it(p, blockIdx.x);
    for (Unit un; ok && it.next(p, un);) {
      float m = -INFINITY, l = 0.f;
      const int n = un.t1 - un.t0;
      // a warp whose 32 rows all lie past the sequence's end (the ragged last
      // Q tile of short sequences) skips the softmax -- its O rows are never
      // stored -- but takes every barrier step with the other warps
      const bool live =
          !Tr::SHORT || __any_sync(0xffffffffu, (2 * un.qt + wg) * BM + row < un.len);
      if (!live) {
        for (int j = 0; j < n; ++j, ++g) {
          ok = mbar_wait(bar(Tr::B_S_FULL + wg), g & 1u, w, kSiteSFull);
          if (!(ok = __all_sync(0xffffffffu, ok))) break;
          if constexpr (Tr::SEP_P) {
            tc_fence_before();
            mbar_arrive(bar(Tr::B_S_FREE + wg));
          }
          if (Tr::SEP_P ? g > 0 : j > 0) {
            ok = mbar_wait(bar(Tr::B_O_DONE + wg), (g - 1) & 1u, w, kSiteODone);
            if (!(ok = __all_sync(0xffffffffu, ok))) break;
          }
          tc_fence_before();
          mbar_arrive(bar(Tr::B_P_FULL + wg));
        }
      } else
      for (int j = 0; j < n; ++j, ++g) {
        ok = mbar_wait(bar(Tr::B_S_FULL + wg), g & 1u, w, kSiteSFull);
        if (!(ok = __all_sync(0xffffffffu, ok))) break;
        tc_fence_after();
        uint32_t r[BN / 32][32];
#pragma unroll
        for (int q = 0; q < BN / 32; ++q) tmem_ld32(s_col + q * 32, r[q]);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < BN / 32; ++q) reg_fence(r[q]);
        if constexpr (Tr::SEP_P) {
          // S is in registers: the next tile's Q K^T may overwrite it
          tc_fence_before();
          mbar_arrive(bar(Tr::B_S_FREE + wg));
        }
        uint32_t pk[BN / 2];
        // key columns this row sees in K/V tile t: below N, and with the
        // causal mask up to the row's own position
        const int t = un.t0 + j;
        int valid = un.len - t * BN;
        if (p.causal) valid = imin(valid, (2 * un.qt + wg) * BM + row - t * BN + 1);
        const float alpha = softmax_step<T, BN, Tr::EMU, Tr::SHORT>(r, valid, c, m, l, pk);
        if constexpr (Tr::SEP_P) {
          // P has one buffer per Q tile: the previous P.V (the previous tile of
          // this unit, or the last of the previous unit, already waited for by
          // its epilogue) must have read it, and have landed in O before O is
          // rescaled
          if (g > 0) {
            ok = mbar_wait(bar(Tr::B_O_DONE + wg), (g - 1) & 1u, w, kSiteODone);
            if (!(ok = __all_sync(0xffffffffu, ok))) break;
            tc_fence_after();
          }
          store_p<T, BN>(p_col, pk);
          tmem_wait_st();
          if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) rescale_o<D>(o_col, alpha);
        } else {
          store_p<T, BN>(s_col, pk);
          tmem_wait_st();
          if (j > 0) {
            // the previous P.V into this O must have landed before O is touched
            // or the next P.V is issued (every phase is waited once, in order)
            ok = mbar_wait(bar(Tr::B_O_DONE + wg), (g - 1) & 1u, w, kSiteODone);
            if (!(ok = __all_sync(0xffffffffu, ok))) break;
            tc_fence_after();
            if (__any_sync(0xffffffffu, alpha != 1.f)) rescale_o<D>(o_col, alpha);
          }
        }
        tc_fence_before();
        mbar_arrive(bar(Tr::B_P_FULL + wg));
      }
      if (!ok) break;
      ok = mbar_wait(bar(Tr::B_O_DONE + wg), (g - 1) & 1u, w, kSiteEpi);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      // staged for short sequences, where the epilogue is a large share of a
      // unit (B200 [32,400,4,64]: 29.5 -> 27.7 us); long ones keep the direct
      // stores (staged, [4,4096,8,64] measured 212.4 -> 214.9 us)
      if (Tr::SHORT && p.N <= kStagedMaxN && un.kind == kStoreWhole && p.o_part == nullptr)
        store_row_staged<typename Elem<T>::Out, D>(p, un, o_col, (2 * un.qt + wg) * BM + row, m,
                                                   l, gbase + Tr::OFF_STG + warp * (32 * D * 2));
      else
        ok = store_row<typename Elem<T>::Out, D>(p, un, o_col, (2 * un.qt + wg) * BM + row, m, l,
                                                 w);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, Tr::TMEM_COLS);
  }
}

// ===========================================================================
// fa_fwd_kernel: one Q tile per unit, S double buffered
// ===========================================================================
template <int D_, int BN_, int KST_, int VST_, int EB_ = 2>
struct FwdTraits {
  static constexpr int D = D_;
  static constexpr int EB = EB_;             // bytes an element of Q, K, V
  static constexpr int CH_ELEMS = 128 / EB;  // elements in a 128-byte chunk
  static constexpr int BM = 128;
  static constexpr int BN = BN_;
  static constexpr int KST = KST_;
  static constexpr int VST = VST_;
  static constexpr int KCH = (D * EB + 127) / 128;   // 128-byte chunks along d (zero-filled tail)
  static constexpr int Q_BYTES = BM * KCH * 128;
  static constexpr int KV_BYTES = BN * KCH * 128;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr int OFF_STG = OFF_V + VST * KV_BYTES;  // 4 softmax warps x 4 KB (epilogue)
  static constexpr int OFF_BAR = OFF_STG + 4 * 4096;
  static constexpr int B_Q_FULL = 0, B_Q_EMPTY = 1, B_K_FULL = 2, B_K_EMPTY = B_K_FULL + KST,
                       B_V_FULL = B_K_EMPTY + KST, B_V_EMPTY = B_V_FULL + VST,
                       B_S_FULL = B_V_EMPTY + VST, B_P_FULL = B_S_FULL + 2,
                       B_O_DONE = B_P_FULL + 2, B_DRAIN = B_O_DONE + 1, NUM_BARS = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  static constexpr uint32_t TM_O = 2 * BN;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(2 * BN + D <= 512, "tensor memory budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(D % 32 == 0 && BN % 32 == 0, "tile shape");
};

template <class T, class Tr, bool VARLEN>
__global__ void __launch_bounds__(224, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, const FwdParams p) {
  constexpr int D = Tr::D, BN = Tr::BN, KST = Tr::KST, VST = Tr::VST;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + Tr::OFF_Q, sK = base + Tr::OFF_K, sV = base + Tr::OFF_V;
  const uint32_t bars = base + Tr::OFF_BAR;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + Tr::OFF_MISC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + Tr::OFF_MISC + 4);
  auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitCtl w{abort_flag, p.limit_ns, p.status};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(Tr::B_Q_FULL), 1);
    mbar_init(bar(Tr::B_Q_EMPTY), 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(bar(Tr::B_K_FULL + s), 1);
      mbar_init(bar(Tr::B_K_EMPTY + s), 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(bar(Tr::B_V_FULL + s), 1);
      mbar_init(bar(Tr::B_V_EMPTY + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(Tr::B_S_FULL + s), 1);
      mbar_init(bar(Tr::B_P_FULL + s), 128);
    }
    mbar_init(bar(Tr::B_O_DONE), 1);
    mbar_init(bar(Tr::B_DRAIN), 1);
    fence_mbar_init();
  }
  if (warp == 6) {
    tmem_alloc(smem_u32(tmem_slot), Tr::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmq);
    tma_prefetch_desc(&tmk);
    tma_prefetch_desc(&tmv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------ Q and K producer
    {
      const bool leader = lane == 0;  // issues; all lanes run the loop
      uint32_t kc = 0, qc = 0;
      bool ok = true;
      UnitIter<VARLEN> it(p, blockIdx.x);
      for (Unit un; ok && it.next(p, un);) {
        if (qc > 0 && !(ok = mbar_wait_warp(bar(Tr::B_Q_EMPTY), (qc - 1) & 1u, w, kSiteQEmpty))) break;
        mbar_expect_tx(leader, bar(Tr::B_Q_FULL), Tr::Q_BYTES);
#pragma unroll
        for (int c = 0; c < Tr::KCH; ++c)
          tma_load_4d(leader, sQ + c * (Tr::BM * 128), &tmq, bar(Tr::B_Q_FULL), c * Tr::CH_ELEMS, un.h,
                      un.tok0 + un.qt * Tr::BM, un.tb);
        ++qc;
        for (int t = un.t0; t < un.t1; ++t) {
          const uint32_t ks = kc % KST;
          if (kc >= (uint32_t)KST &&
              !(ok = mbar_wait_warp(bar(Tr::B_K_EMPTY + ks), ((kc / KST) - 1) & 1u, w, kSiteKEmpty)))
            break;
          mbar_expect_tx(leader, bar(Tr::B_K_FULL + ks), Tr::KV_BYTES);
#pragma unroll
          for (int c = 0; c < Tr::KCH; ++c)
            tma_load_4d(leader, sK + ks * Tr::KV_BYTES + c * (BN * 128), &tmk, bar(Tr::B_K_FULL + ks),
                        c * Tr::CH_ELEMS, un.h, un.tok0 + t * BN, un.tb);
          ++kc;
        }
      }
      // Every issued load must land before the block exits.
      if (qc > 0) mbar_drain(bar(Tr::B_Q_FULL), (qc - 1) & 1u, p.limit_ns);
      for (uint32_t s = 0; s < (uint32_t)KST; ++s)
        if (kc > s) mbar_drain(bar(Tr::B_K_FULL + s), ((kc - 1 - s) / KST) & 1u, p.limit_ns);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------ V producer
    {
      const bool leader = lane == 0;  // issues; all lanes run the loop
      uint32_t vc = 0;
      bool ok = true;
      UnitIter<VARLEN> it(p, blockIdx.x);
      for (Unit un; ok && it.next(p, un);) {
        for (int t = un.t0; t < un.t1; ++t) {
          const uint32_t vs = vc % VST;
          if (vc >= (uint32_t)VST &&
              !(ok = mbar_wait_warp(bar(Tr::B_V_EMPTY + vs), ((vc / VST) - 1) & 1u, w, kSiteVEmpty)))
            break;
          mbar_expect_tx(leader, bar(Tr::B_V_FULL + vs), Tr::KV_BYTES);
#pragma unroll
          for (int c = 0; c < Tr::KCH; ++c)
            tma_load_4d(leader, sV + vs * Tr::KV_BYTES + c * (BN * 128), &tmv, bar(Tr::B_V_FULL + vs),
                        c * Tr::CH_ELEMS, un.h, un.tok0 + t * BN, un.tb);
          ++vc;
        }
      }
      for (uint32_t s = 0; s < (uint32_t)VST; ++s)
        if (vc > s) mbar_drain(bar(Tr::B_V_FULL + s), ((vc - 1 - s) / VST) & 1u, p.limit_ns);
    }
    __syncwarp();
  } else if (warp == 6) {
    // ----------------------------------------------------- MMA issuer
    {
      const bool leader = lane == 0;  // issues; all lanes run the loop
      constexpr uint32_t kIdescQK = f16_idesc(Elem<T>::kFmt, 128, BN, false);
      constexpr uint32_t kIdescPV = f16_idesc(Elem<T>::kFmt, 128, D, true);
      uint32_t kc = 0, vc = 0, g = 0, uc = 0;
      bool ok = true;
      const uint64_t q_desc0 = sw128_desc(sQ, 16, 1024), k_desc0 = sw128_desc(sK, 16, 1024),
                     v_desc0 = sw128_desc(sV, BN * 128, 1024);
      // O += P_j V_j for the tile whose S/P buffer use counter is gp (nsteps
      // k-steps: those with keys below the sequence's end).
      auto issue_pv = [&](uint32_t gp, bool first, int nsteps) -> bool {
        const uint32_t pb = gp & 1u;
        if (!mbar_wait_warp(bar(Tr::B_P_FULL + pb), (gp >> 1) & 1u, w, kSitePFull)) return false;
        const uint32_t vs = vc % VST;
        if (!mbar_wait_warp(bar(Tr::B_V_FULL + vs), (vc / VST) & 1u, w, kSiteVFull)) return false;
        tc_fence_after();
        const uint64_t vd = desc_advance(v_desc0, vs * Tr::KV_BYTES);
        constexpr int kSteps = BN * Tr::EB / 32;
        if (nsteps >= kSteps) {
#pragma unroll
          for (int kk = 0; kk < kSteps; ++kk)
            mma_ts<T>(leader, tmem + Tr::TM_O, tmem + pb * BN + kk * 8,
                      desc_advance(vd, kk * (32 / Tr::EB) * 128),
                      kIdescPV, (!first || kk > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < kSteps; ++kk)
            mma_ts<T>(leader && kk < nsteps, tmem + Tr::TM_O, tmem + pb * BN + kk * 8,
                      desc_advance(vd, kk * (32 / Tr::EB) * 128),
                      kIdescPV, (!first || kk > 0) ? 1u : 0u);
        }
        umma_commit(leader, bar(Tr::B_V_EMPTY + vs));
        umma_commit(leader, bar(Tr::B_O_DONE));
        ++vc;
        return true;
      };
      UnitIter<VARLEN> it(p, blockIdx.x);
      for (Unit un; ok && it.next(p, un);) {
        if (!(ok = mbar_wait_warp(bar(Tr::B_Q_FULL), uc & 1u, w, kSiteQFull))) break;
        tc_fence_after();
        const int n = un.t1 - un.t0;
        for (int i = 0; i < n; ++i) {
          const uint32_t ks = kc % KST;
          if (!(ok = mbar_wait_warp(bar(Tr::B_K_FULL + ks), (kc / KST) & 1u, w, kSiteKFull))) break;
          tc_fence_after();
          const uint32_t sb = g & 1u;
          const uint64_t kd = desc_advance(k_desc0, ks * Tr::KV_BYTES);
#pragma unroll
          for (int kk = 0; kk < D * Tr::EB / 32; ++kk) {
            const uint32_t ch = kk >> 2, in = (kk & 3) * 32;
            mma_ss<T>(leader, tmem + sb * BN, desc_advance(q_desc0, ch * (Tr::BM * 128) + in),
                    desc_advance(kd, ch * (BN * 128) + in), kIdescQK, kk > 0 ? 1u : 0u);
          }
          umma_commit(leader, bar(Tr::B_K_EMPTY + ks));
          umma_commit(leader, bar(Tr::B_S_FULL + sb));
          if (i == n - 1) umma_commit(leader, bar(Tr::B_Q_EMPTY));
          ++kc;
          if (i > 0 &&
              !(ok = issue_pv(g - 1, i == 1, pv_steps<BN, Tr::EB>(un.len, un.t0 + i - 1))))
            break;
          ++g;
        }
        if (!ok) break;
        if (!(ok = issue_pv(g - 1, n == 1, pv_steps<BN, Tr::EB>(un.len, un.t1 - 1)))) break;
        ++uc;
      }
      // Every issued MMA must finish before tensor memory is released.
      umma_commit(leader, bar(Tr::B_DRAIN));
      mbar_drain(bar(Tr::B_DRAIN), 0, p.limit_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------ softmax and epilogue
    const int row = threadIdx.x;  // 0..127, TMEM lane
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    const float c = p.sl2;
    uint32_t g = 0;
    bool ok = true;
    UnitIter<VARLEN> it(p, blockIdx.x);
    for (Unit un; ok && it.next(p, un);) {
      float m = -INFINITY, l = 0.f;
      const int n = un.t1 - un.t0;
      // a warp whose rows all lie past the sequence's end skips the softmax
      // (its O rows are never stored) but takes every barrier step
      const bool live = __any_sync(0xffffffffu, un.qt * Tr::BM + row < un.len);
      for (int i = 0; i < n; ++i, ++g) {
        const uint32_t sb = g & 1u;
        ok = mbar_wait(bar(Tr::B_S_FULL + sb), (g >> 1) & 1u, w, kSiteSFull);
        if (!(ok = __all_sync(0xffffffffu, ok))) break;
        tc_fence_after();
        const uint32_t scol = tl + sb * BN;
        float alpha = 1.f;
        if (live) {
          uint32_t r[BN / 32][32];
#pragma unroll
          for (int q = 0; q < BN / 32; ++q) tmem_ld32(scol + q * 32, r[q]);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < BN / 32; ++q) reg_fence(r[q]);
          uint32_t pk[BN / 2];
          const int t = un.t0 + i;
          int valid = un.len - t * BN;
          if (p.causal) valid = imin(valid, un.qt * Tr::BM + row - t * BN + 1);
          alpha = softmax_step<T, BN>(r, valid, c, m, l, pk);
          store_p<T, BN>(scol, pk);
          tmem_wait_st();
        }
        if (i > 0) {
          // O holds P_{<j} V_{<j}: once the previous P.V has landed, rescale it
          // (if a row's reference max moved) before this tile's P.V is issued.
          ok = mbar_wait(bar(Tr::B_O_DONE), (g - 1) & 1u, w, kSiteODone);
          if (!(ok = __all_sync(0xffffffffu, ok))) break;
          tc_fence_after();
          if (live && __any_sync(0xffffffffu, alpha != 1.f)) rescale_o<D>(tl + Tr::TM_O, alpha);
        }
        tc_fence_before();
        mbar_arrive(bar(Tr::B_P_FULL + sb));
      }
      if (!ok) break;
      ok = mbar_wait(bar(Tr::B_O_DONE), (g - 1) & 1u, w, kSiteEpi);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      // through the warp's staging tile: one thread a row would make every
      // warp store touch 32 rows ([1,6400,1,256] split mode: the epilogue took
      // a seventh of the kernel)
      uint8_t* stg = gbase + Tr::OFF_STG + warp * 4096;
      if (p.o_part != nullptr)
        store_row_chunked<float, D, true>(p, un, tl + Tr::TM_O, un.qt * Tr::BM + row, m, l, stg);
      else
        store_row_chunked<typename Elem<T>::Out, D, false>(p, un, tl + Tr::TM_O,
                                                            un.qt * Tr::BM + row, m, l, stg);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 6) {
    tc_fence_after();
    tmem_dealloc(tmem, Tr::TMEM_COLS);
  }
}

// Merge of split K/V partial results: one warp per (b, n, h) row.
// o_part rows are normalised by their own sums; lse_part is base 2.
template <class T, int D>
__global__ void __launch_bounds__(256) fa_combine_kernel(const float* __restrict__ o_part,
                                                         const float* __restrict__ lse_part,
                                                         T* __restrict__ o, float* __restrict__ lse,
                                                         int B, int H, int N, int S) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= (long long)B * N * H) return;
  const int h = (int)(row % H);
  const int n = (int)((row / H) % N);
  const int b = (int)(row / ((long long)H * N));
  float mx = -INFINITY;
  for (int s = 0; s < S; ++s)
    mx = fmaxf(mx, lse_part[(((size_t)s * B + b) * H + h) * N + n]);
  float tot = 0.f;
  for (int s = 0; s < S; ++s) tot += ex2(lse_part[(((size_t)s * B + b) * H + h) * N + n] - mx);
  const float L2 = mx + lg2(tot);
  // lane x owns the column pairs 2 (x + 32 j), j < NP (d = 96 leaves lanes
  // 16-31 idle in the second pair)
  constexpr int NP = (D / 2 + 31) / 32;
  float2 acc[NP];
#pragma unroll
  for (int j = 0; j < NP; ++j) acc[j] = make_float2(0.f, 0.f);
  for (int s = 0; s < S; ++s) {
    const float wgt = ex2(lse_part[(((size_t)s * B + b) * H + h) * N + n] - L2);
    const float* src = o_part + ((((size_t)s * B + b) * N + n) * H + h) * D;
#pragma unroll
    for (int j = 0; j < NP; ++j) {
      const int col = 2 * (lane + 32 * j);
      if (col < D) {
        const float2 x = *reinterpret_cast<const float2*>(src + col);
        acc[j].x = fmaf(wgt, x.x, acc[j].x);
        acc[j].y = fmaf(wgt, x.y, acc[j].y);
      }
    }
  }
  T* dst = o + (((size_t)b * N + n) * H + h) * D;
#pragma unroll
  for (int j = 0; j < NP; ++j) {
    const int col = 2 * (lane + 32 * j);
    if (col < D) *reinterpret_cast<uint32_t*>(dst + col) = Elem<T>::pack(acc[j].x, acc[j].y);
  }
  if (lane == 0) lse[((size_t)b * H + h) * N + n] = L2 * kLn2;
}

// ---------------------------------------------------------------- launchers
// Number of K/V splits: only when the units leave most SMs idle, and only so
// far that every split keeps at least 8 K/V tiles.
static int choose_splits(long long base_units, int n_kvt, int sm_count) {
  int n_split = 1;
  if (base_units * 2 <= sm_count) {
    n_split = (int)(sm_count / base_units);
    n_split = n_split < n_kvt / 8 ? n_split : n_kvt / 8;
    n_split = n_split > 1 ? n_split : 1;
  }
  return n_split;
}

// Balanced schedule: when whole units would leave the last wave of blocks
// partly idle (waves = ceil(units / SMs), efficiency = units / (waves * SMs)),
// give every SM the same number of (unit, K/V tile) steps instead.  Units are
// then cut into pieces across neighbouring blocks and merged in the kernel,
// so it is kept for units long enough (>= 16 K/V tiles) that the extra
// Q loads and merges stay small.  With fewer units than SMs nearly every unit
// is cut, which pays only for long units (measured on B200: 128 units of 32
// tiles ran 79 us balanced against 74 us round-robin, while 100 units of 200
// tiles -- one d = 96 head of 25600 rows -- ran 300 us against 397 us).
static bool use_balanced(long long units, int n_kvt, int sm_count) {
  if (n_kvt < 16 || units * n_kvt >= (1ll << 31)) return false;
  if (units <= sm_count && n_kvt < 64) return false;
  const long long waves = (units + sm_count - 1) / sm_count;
  return (double)units / (double)(waves * sm_count) < 0.95;
}

int plan_fwd(int B, int H, int N, int d, unsigned flags, int sm_count, FwdSchedule* s) {
  if (B < 1 || H < 1 || N < 1 || sm_count < 1) return FA_ERR_SHAPE;
  if (d != 64 && d != 96 && d != 128 && d != 256) return FA_ERR_HEADDIM;
  FwdSchedule x{};
  x.B = B;
  x.H = H;
  x.N = N;
  x.d = d;
  x.causal = (flags & 1u) ? 1 : 0;
  x.cu = nullptr;
  x.total = N;
  const bool varlen = (flags & kPlanVarlen) != 0;
  // Two Q tiles per unit once a head has more than one tile's worth of rows;
  // a single tile per unit for short sequences and for d = 256 (whose O
  // accumulator leaves tensor memory room for only one Q tile).
  x.pair = (N > 128 && d <= 128) ? 1 : 0;
  x.unit_rows = x.pair ? 256 : 128;
  x.bn = 128;
  x.n_qt = (N + x.unit_rows - 1) / x.unit_rows;
  x.n_kvt = (N + x.bn - 1) / x.bn;
  const long long base_units = (long long)B * H * x.n_qt;
  if (base_units >= (1ll << 31)) return FA_ERR_SHAPE;
  // causal units differ in length: they are neither split nor cut, and run
  // longest first (decode_unit)
  int n_split = (x.causal || varlen) ? 1 : choose_splits(base_units, x.n_kvt, sm_count);
  x.kvt_per_split = (x.n_kvt + n_split - 1) / n_split;
  x.n_split = (x.n_kvt + x.kvt_per_split - 1) / x.kvt_per_split;  // no empty split
  x.n_units = (int)(base_units * x.n_split);
  const bool balanced =
      !x.causal && !varlen && x.pair && x.n_split == 1 &&
      use_balanced(base_units, x.n_kvt, sm_count);
  x.grid = balanced ? sm_count : (x.n_units < sm_count ? x.n_units : sm_count);
  if (balanced) {
    x.n_iter = (int)(base_units * x.n_kvt);
    x.iter_per = x.n_iter / x.grid;
    x.iter_rem = x.n_iter % x.grid;
  }
  *s = x;
  return FA_OK;
}

size_t fwd_scratch_bytes(const FwdSchedule& s) {
  if (s.n_split > 1)
    return ((size_t)s.n_split * s.B * s.N * s.H * s.d + (size_t)s.n_split * s.B * s.H * s.N) *
           sizeof(float);
  if (s.n_iter > 0)  // one partial slot per block: rows x d fp32, rows LSE, a flag
    return ((size_t)s.grid * s.unit_rows * s.d + (size_t)s.grid * s.unit_rows + s.grid) *
           sizeof(float);
  return 0;
}

int fwd_block_pieces(const FwdSchedule& s, int blk, int* out, int max_pieces) {
  UnitIter<false> it(s, blk);
  int n = 0;
  for (Unit x; it.next(s, x); ++n) {
    if (n < max_pieces) {
      int* o = out + 6 * n;
      o[0] = x.u;
      o[1] = x.t0;
      o[2] = x.t1;
      o[3] = x.kind;
      o[4] = x.peer0;
      o[5] = x.npeer;
    }
  }
  return n;
}

template <class T, int D, int BN, int THREADS, int SMEM, bool SPLIT_REGS, class Kernel>
static int launch_fwd(Kernel kern, const FwdSchedule& s, const void* q, const void* k,
                      const void* v, void* o, float* lse, float scale, float o_scale,
                      long long tok_in, cudaStream_t stream) {
  const int fmt = Elem<T>::kMapFmt;
  CUtensorMap tmq, tmk, tmv;
  int rc;
  // memory view: B batch entries of N tokens, or one entry of all tokens (varlen)
  const int mB = s.cu ? 1 : s.B, mN = s.total;
  if ((rc = make_tmap_bnhd(&tmq, q, fmt, mB, mN, s.H, D, 128, tok_in)) != FA_OK) return rc;
  if ((rc = make_tmap_bnhd(&tmk, k, fmt, mB, mN, s.H, D, BN, tok_in)) != FA_OK) return rc;
  if ((rc = make_tmap_bnhd(&tmv, v, fmt, mB, mN, s.H, D, BN, tok_in)) != FA_OK) return rc;

  FwdParams p{};
  static_cast<FwdSchedule&>(p) = s;
  p.o = o;
  p.lse = lse;
  p.sl2 = scale * kLog2e;
  p.o_scale = o_scale;
  p.limit_ns = 4000000000ull;
  p.status = device_status_ptr();

  void* ws = nullptr;
  const size_t ws_bytes = fwd_scratch_bytes(s);
  if (ws_bytes > 0 && (rc = scratch_alloc(&ws, ws_bytes, stream)) != FA_OK) return rc;
  if (s.n_split > 1) {
    p.o_part = static_cast<float*>(ws);
    p.lse_part = p.o_part + (size_t)s.n_split * s.B * s.N * s.H * D;
  } else if (s.n_iter > 0) {
    p.bal_o = static_cast<float*>(ws);
    p.bal_lse = p.bal_o + (size_t)s.grid * s.unit_rows * D;
    p.bal_flag = reinterpret_cast<unsigned*>(p.bal_lse + (size_t)s.grid * s.unit_rows);
    if (cudaMemsetAsync(p.bal_flag, 0, s.grid * sizeof(unsigned), stream) != cudaSuccess) {
      rc = launch_status(cudaGetLastError());
      scratch_free(ws, stream);
      return rc;
    }
  }
  if (SPLIT_REGS && (rc = check_launch_regs((const void*)kern)) != FA_OK) {
    scratch_free(ws, stream);
    return rc;
  }
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) !=
      cudaSuccess) {
    rc = launch_status(cudaGetLastError());
    scratch_free(ws, stream);
    return rc;
  }
  cudaEvent_t ev0, ev1;
  take_kernel_events(false, &ev0, &ev1);
  if (ev0) cudaEventRecord(ev0, stream);
  if (s.n_iter > 0) {
    // A merging block waits for its neighbours' partial rows, so all blocks
    // must be resident at once: a cooperative launch guarantees it (or fails).
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(s.grid);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    rc = launch_status(cudaLaunchKernelEx(&cfg, kern, tmq, tmk, tmv, p));
  } else {
    kern<<<s.grid, THREADS, SMEM, stream>>>(tmq, tmk, tmv, p);
    rc = launch_status(cudaGetLastError());
  }
  if (ev1) cudaEventRecord(ev1, stream);
  note_launches(1);
  if (rc == FA_OK && s.n_split > 1) {
    const long long rows = (long long)s.B * s.N * s.H;
    fa_combine_kernel<typename Elem<T>::Out, D><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(
        p.o_part, p.lse_part, static_cast<typename Elem<T>::Out*>(o), lse, s.B, s.H, s.N,
        s.n_split);
    rc = launch_status(cudaGetLastError());
    note_launches(1);
  }
  scratch_free(ws, stream);
  return rc;
}

template <class T, class Tr>
static int run_single(const FwdSchedule& s, const void* q, const void* k, const void* v, void* o,
                      float* lse, float scale, float o_scale, long long tok_in,
                      cudaStream_t stream) {
  static_assert(Tr::BM == 128 && Tr::EB == Elem<T>::kBytes, "unit rows, element size");
  return launch_fwd<T, Tr::D, Tr::BN, 224, Tr::SMEM_BYTES, false>(
      s.cu ? fa_fwd_kernel<T, Tr, true> : fa_fwd_kernel<T, Tr, false>, s, q, k, v, o, lse, scale,
      o_scale, tok_in, stream);
}

template <class T, class Tr>
static int run_pp(const FwdSchedule& s, const void* q, const void* k, const void* v, void* o,
                  float* lse, float scale, float o_scale, long long tok_in, cudaStream_t stream) {
  static_assert(2 * Tr::BM == 256 && Tr::EB == Elem<T>::kBytes, "unit rows, element size");
  return launch_fwd<T, Tr::D, Tr::BN, 384, Tr::SMEM_BYTES, true>(
      s.cu ? fa_fwd_pp_kernel<T, Tr, true> : fa_fwd_pp_kernel<T, Tr, false>, s, q, k, v, o, lse,
      scale, o_scale, tok_in, stream);
}

template <class T>
int fwd_launch(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int N, int d, float scale, unsigned flags, long long tok_in, cudaStream_t stream,
               const int* cu, int total, float o_scale) {
  DeviceInfo dev;
  int rc = current_device(&dev);
  if (rc != FA_OK) return rc;
  FwdSchedule s;
  if ((rc = plan_fwd(B, H, N, d, flags | (cu ? kPlanVarlen : 0u), dev.sm_count, &s)) != FA_OK)
    return rc;
  if (cu != nullptr) {
    s.cu = cu;
    s.total = total;
  }
  if constexpr (Elem<T>::kF8) {
    // 8-bit Q, K, V: d = 128 (one 128-byte chunk a row).  Two K and two V
    // stages (measured on B200 at [1,8192,8,128]: 236.8 us, against 238.8 us
    // with four of each)
    if (d != 128) return FA_ERR_HEADDIM;
    return s.pair ? run_pp<T, FwdPPTraits<128, 2, 2, 1>>(s, q, k, v, o, lse, scale, o_scale,
                                                         tok_in, stream)
                  : run_single<T, FwdTraits<128, 128, 3, 2, 1>>(s, q, k, v, o, lse, scale,
                                                                o_scale, tok_in, stream);
  } else {
    switch (d) {
      case 64:
        return s.pair ? run_pp<T, FwdPPTraits<64, 4, 4>>(s, q, k, v, o, lse, scale, o_scale,
                                                         tok_in, stream)
                      : run_single<T, FwdTraits<64, 128, 4, 4>>(s, q, k, v, o, lse, scale,
                                                                 o_scale, tok_in, stream);
      case 96:
        return s.pair ? run_pp<T, FwdPPTraits<96, 2, 2>>(s, q, k, v, o, lse, scale, o_scale,
                                                         tok_in, stream)
                      : run_single<T, FwdTraits<96, 128, 3, 2>>(s, q, k, v, o, lse, scale,
                                                                 o_scale, tok_in, stream);
      case 128:
        return s.pair ? run_pp<T, FwdPPTraits<128, 2, 2>>(s, q, k, v, o, lse, scale, o_scale,
                                                          tok_in, stream)
                      : run_single<T, FwdTraits<128, 128, 3, 2>>(s, q, k, v, o, lse, scale,
                                                                  o_scale, tok_in, stream);
      case 256:
        return run_single<T, FwdTraits<256, 128, 1, 1>>(s, q, k, v, o, lse, scale, o_scale,
                                                          tok_in, stream);
      default:
        return FA_ERR_HEADDIM;
    }
  }
}

template int fwd_launch<__nv_bfloat16>(const void*, const void*, const void*, void*, float*, int,
                                       int, int, int, float, unsigned, long long, cudaStream_t,
                                       const int*, int, float);
template int fwd_launch<__half>(const void*, const void*, const void*, void*, float*, int, int,
                                int, int, float, unsigned, long long, cudaStream_t, const int*,
                                int, float);
template int fwd_launch<__nv_fp8_e4m3>(const void*, const void*, const void*, void*, float*, int,
                                       int, int, int, float, unsigned, long long, cudaStream_t,
                                       const int*, int, float);

}  // namespace fa
