// fa_bwd.cu -- backward pass of exact attention on sm_100a, by recompute.
//
// The forward keeps only O and the per-row LSE; the backward rebuilds P from
// Q, K and the LSE instead of storing it (LLM explainer page, section 6.2,
// recompute strategy; YOLO11 page, section 2.3).  With c = scale * log2(e):
//   P^T  = exp2(c K Q^T - LSE * log2(e))      (no max or sum: LSE is saved)
//   dV  += P^T dO
//   dP^T = V dO^T,   dS^T = P^T o (dP^T - D),   D_i = sum_x dO_ix O_ix
//   dK  += scale dS^T Q
//   dQ  += scale dS K   (fp32, reduced into global memory across K/V tiles)
//
// Five kernels:
//   fa_bwd_pre_kernel   D, minus the base-2 LSE (padded to whole Q tiles) and
//                       a zeroed fp32 dQ accumulator
//   fa_bwd_kernel       d = 64: one block per (K/V tile of 128 keys, head,
//                       batch); its loop walks the Q tiles of 128 queries
//   fa_bwd_tq_kernel    d = 96, 128, 256: 64-query inner tiles with dQ produced
//                       transposed (described where it is defined)
//   fa_bwd_dkv_kernel   sums the fp32 dK, dV partials of split query ranges
//   fa_bwd_dq_kernel    dQ = scale * accumulator, rounded to 16 bits
// The main kernels' grids are 1-D (block = (b * H + h) * blocks per head +
// x, or key-tile major for the causal mask) and may split a key tile's query
// range over several blocks when few key tiles would leave SMs idle.
//
// fa_bwd_kernel layout (384 threads, one block per SM):
//   warps 0-7  compute: warp w owns TMEM lane quadrant w % 4 and half w / 4 of
//              the 128 query columns; P and dS are elementwise in (key, query),
//              so the halves need no exchange.  They recompute P^T and dS^T,
//              drain the dQ tiles (TMEM -> swizzled shared memory -> TMA
//              reduce-add into the fp32 accumulator) and store dK, dV
//   warp  8    TMA producer
//   warp  9    TMEM allocator; issues S^T and dV
//   warp 10    issues dP^T, dK and dQ
//   warp 11    idle (three whole warpgroups, so registers can move from the
//              producer/MMA warpgroup to the compute ones)
// Per Q tile i: dV += P^T dO_i as soon as P^T is written, then S^T for tile
// i+1 (so the next P^T can start while dS^T is computed); dK += dS^T Q_i as
// soon as dS^T is written, then dP^T for tile i+1, then dQ_i = dS K.
// Tensor memory (d = 64): S^T [0,128), dP^T [128,256), dV [256,320),
// dK [320,384), dQ [384,448).  Packed 16-bit P^T and dS^T overwrite the first
// 32 columns of each 64-column query half of S^T and dP^T.
#include "fa_common.cuh"
#include "fa_host.h"

namespace fa {

struct BwdTraits64 {
  static constexpr int NHALF = 1;  // blocks per key tile, one per slice of d
  static constexpr int D = 64;
  static constexpr int BN = 128;  // keys per block
  static constexpr int BM = 128;  // queries per inner tile
  static constexpr int QST = 2;   // Q / dO stages
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int QT_BYTES = BM * D * 2;
  static constexpr int DS_BYTES = BN * BM * 2;       // dS tile, 16-bit
  static constexpr int STAGE_BYTES = BM * D * 4;     // dQ tile, fp32: 8 warps x 4 KiB boxes
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_BYTES;
  static constexpr int OFF_Q = OFF_V + KV_BYTES;
  static constexpr int OFF_DO = OFF_Q + QST * QT_BYTES;
  static constexpr int OFF_DS = OFF_DO + QST * QT_BYTES;
  static constexpr int OFF_STG = OFF_DS + 2 * DS_BYTES;
  static constexpr int OFF_L = OFF_STG + STAGE_BYTES;  // minus the base-2 LSE, per stage
  static constexpr int OFF_DD = OFF_L + QST * BM * 4;  // D per stage
  static constexpr int OFF_BAR = OFF_DD + QST * BM * 4;
  static constexpr int B_KV_FULL = 0, B_Q_FULL = 1, B_Q_EMPTY = B_Q_FULL + QST,
                       B_S_FULL = B_Q_EMPTY + QST, B_DP_FULL = B_S_FULL + 1,
                       B_P_READY = B_DP_FULL + 1, B_DS_READY = B_P_READY + 1,
                       B_DSBUF_FREE = B_DS_READY + 1,
                       B_DQ_FULL = B_DSBUF_FREE + 2, B_DQ_FREE = B_DQ_FULL + 1,
                       B_KV_DONE = B_DQ_FREE + 1, B_DRAIN = B_KV_DONE + 1,
                       NUM_BARS = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DV = 256, TM_DK = 320, TM_DQ = 384;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int ACC_BOX_ROWS = 32;  // dQ reduce box: 32 d columns x 32 queries (one warp's)
  // exponentials on the FMA pipe per 8 column pairs of P^T: the compute
  // warps' exponentials are MUFU-bound (16 a clock per SM).  Measured on
  // B200, [4,4096,8,64] backward kernel: 0: 453.3, 1: 447.2, 2: 436.5,
  // 3: 439.4 us
  static constexpr int EMU = 2;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct BwdParams {
  const float* lse2;  // [B, H, Npad] minus the base-2 LSE, -inf past N
  const float* dvec;  // [B, H, Npad] D, 0 past N
  float* dq_acc;      // [B, H, Npad, D] fp32
  void* dk;           // [B, N, H, D]
  void* dv;
  int B, H, N, Npad, n_qt;  // varlen: B sequences, N = max_seqlen
  long long tok_g;    // token stride of dk, dv (elements): H*D, or 3*H*D when packed
  const int* cu;      // varlen: device [B+1] sequence starts on the token axis; else null
  int total;          // tokens a batch entry holds in memory: N, or all tokens (varlen)
  float sl2;          // scale * log2(e)
  float scale;
  unsigned long long limit_ns;
  unsigned long long* status;
  // split query ranges (kernels instantiated with SPLIT): n_split blocks per
  // key tile, block x = key tile * n_split + split; each writes its fp32
  // partial dK (scaled), dV to dk_part / dv_part + split * part_stride, laid
  // out [B*N tokens, H, D], and fa_bwd_dkv_kernel sums them
  int n_split;
  int n_x;  // blocks per (batch, head); the grid is 1-D: block = (b * H + h) * n_x + x
  float* dk_part;
  float* dv_part;
  long long part_stride;
};

// Stores 32 d columns (from column col) of key row `key`'s dV and scale*dK
// (fp32 TMEM words a, k2): rounded to T at dk/dv + off, or, for a split
// block, as fp32 into its partial slice.
template <class T, bool SPLIT>
__device__ __forceinline__ void store_dkv32(const BwdParams& p, size_t tok, int h, int col, int sp,
                                            const uint32_t (&a)[32], const uint32_t (&k2)[32],
                                            int D) {
  if constexpr (SPLIT) {
    const size_t at = (size_t)sp * p.part_stride + (tok * p.H + h) * D + col;
    float4* dvp = reinterpret_cast<float4*>(p.dv_part + at);
    float4* dkp = reinterpret_cast<float4*>(p.dk_part + at);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      dvp[j] = make_float4(__uint_as_float(a[4 * j]), __uint_as_float(a[4 * j + 1]),
                           __uint_as_float(a[4 * j + 2]), __uint_as_float(a[4 * j + 3]));
      dkp[j] = make_float4(__uint_as_float(k2[4 * j]) * p.scale,
                           __uint_as_float(k2[4 * j + 1]) * p.scale,
                           __uint_as_float(k2[4 * j + 2]) * p.scale,
                           __uint_as_float(k2[4 * j + 3]) * p.scale);
    }
  } else {
    const size_t off = tok * p.tok_g + (size_t)h * D + col;
    uint4 va[4], vk[4];
    uint32_t* pa = reinterpret_cast<uint32_t*>(va);
    uint32_t* pkk = reinterpret_cast<uint32_t*>(vk);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      pa[j] = Elem<T>::pack(__uint_as_float(a[2 * j]), __uint_as_float(a[2 * j + 1]));
      pkk[j] = Elem<T>::pack(__uint_as_float(k2[2 * j]) * p.scale,
                             __uint_as_float(k2[2 * j + 1]) * p.scale);
    }
    uint4* dvp = reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.dv) + off);
    uint4* dkp = reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.dk) + off);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      dvp[j] = va[j];
      dkp[j] = vk[j];
    }
  }
}

enum { kBSiteQEmpty = 0x21, kBSiteKV, kBSiteQFull, kBSiteDsReady, kBSiteDqFree, kBSiteSFull,
       kBSiteDpFull, kBSiteQFullSm, kBSiteDsBuf, kBSiteDqFull, kBSiteKvDone, kBSitePReady };

__device__ __forceinline__ void bulk_load(bool issue, uint32_t dst, const void* src,
                                          uint32_t bytes, uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "@p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      "\n\t}" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar), "r"((uint32_t)issue)
      : "memory");
}
// Reduce-add of a shared-memory tile into global memory through a tensor map
// (element type, box and swizzle come from the map).
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, uint32_t src, int c0,
                                                  int c1) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(c0), "r"(c1), "r"(src)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

template <class T, class Tr, bool CAUSAL, bool VARLEN, bool SPLIT = false>
__global__ void __launch_bounds__(384, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmdo,
                  const __grid_constant__ CUtensorMap tmacc, const BwdParams p) {
  constexpr int D = Tr::D, BN = Tr::BN, BM = Tr::BM, QST = Tr::QST;
  constexpr int HC = BM / 2;  // query columns per compute warp (one half)
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sK = base + Tr::OFF_K, sV = base + Tr::OFF_V, sQ = base + Tr::OFF_Q,
                 sDO = base + Tr::OFF_DO, sDS = base + Tr::OFF_DS, sSTG = base + Tr::OFF_STG;
  const float* sL = reinterpret_cast<const float*>(gbase + Tr::OFF_L);
  const float* sDD = reinterpret_cast<const float*>(gbase + Tr::OFF_DD);
  uint8_t* gDS = gbase + Tr::OFF_DS;
  uint8_t* gSTG = gbase + Tr::OFF_STG;
  const uint32_t bars = base + Tr::OFF_BAR;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + Tr::OFF_MISC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + Tr::OFF_MISC + 4);
  auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitCtl w{abort_flag, p.limit_ns, p.status};
  // a 1-D grid (B * H may exceed the 65,535 limit of gridDim.y and .z); causal
  // key tiles see fewer query tiles the later they are, so there the order is
  // key-tile major: every head's long key tiles start first
  const unsigned n_bh = (unsigned)(p.B * p.H);
  const int bx = CAUSAL ? (int)(blockIdx.x / n_bh) : (int)(blockIdx.x % (unsigned)p.n_x);
  const int bh = CAUSAL ? (int)(blockIdx.x % n_bh) : (int)(blockIdx.x / (unsigned)p.n_x);
  const int sp = SPLIT ? bx % p.n_split : 0;  // split of the query range
  const int kt = SPLIT ? bx / p.n_split : bx;
  const int h = bh % p.H, b = bh / p.H;
  // the block's sequence on the token axis (batch entry tb, tokens tok0 ..
  // tok0 + len); a key tile past a shorter sequence's end has no work
  int tb, tok0, len;
  seq_bounds(VARLEN ? p.cu : nullptr, b, p.N, p.total, tb, tok0, len);
  if (kt * BN >= len) return;  // block-uniform, before any barrier or allocation
  // causal: query tiles wholly before this key tile see none of its keys
  const int q0 = CAUSAL ? (kt * BN) / BM : 0;
  const int q_all = (VARLEN ? (len + BM - 1) / BM : p.n_qt) - q0;
  // tile i is global i0 + i; a split block takes its share of the range
  const int i0 = SPLIT ? q0 + q_all * sp / p.n_split : q0;
  const int n_qt = SPLIT ? q_all * (sp + 1) / p.n_split - q_all * sp / p.n_split : q_all;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(Tr::B_KV_FULL), 1);
    for (int s = 0; s < QST; ++s) {
      mbar_init(bar(Tr::B_Q_FULL + s), 1);
      mbar_init(bar(Tr::B_Q_EMPTY + s), 2);  // one commit from each MMA warp
    }
    mbar_init(bar(Tr::B_S_FULL), 1);
    mbar_init(bar(Tr::B_DP_FULL), 1);
    mbar_init(bar(Tr::B_P_READY), 256);
    mbar_init(bar(Tr::B_DS_READY), 256);
    mbar_init(bar(Tr::B_DSBUF_FREE), 1);
    mbar_init(bar(Tr::B_DSBUF_FREE + 1), 1);
    mbar_init(bar(Tr::B_DQ_FULL), 1);
    mbar_init(bar(Tr::B_DQ_FREE), 256);
    mbar_init(bar(Tr::B_KV_DONE), 2);
    mbar_init(bar(Tr::B_DRAIN), 2);
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), Tr::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= 8) {
    regs_shrink();  // all four warps of the producer/MMA warpgroup
  if (warp == 8) {
    // -------------------------------------------------------- producer
    {
      const bool leader = lane == 0;  // issues; all lanes run the loop
      mbar_expect_tx(leader, bar(Tr::B_KV_FULL), 2 * Tr::KV_BYTES);
      tma_load_4d(leader, sK, &tmk, bar(Tr::B_KV_FULL), 0, h, tok0 + kt * BN, tb);
      tma_load_4d(leader, sV, &tmv, bar(Tr::B_KV_FULL), 0, h, tok0 + kt * BN, tb);
      const size_t row0 = ((size_t)b * p.H + h) * p.Npad;
      int issued = 0;
      for (int i = 0; i < n_qt; ++i) {
        const int qs = i % QST;
        if (i >= QST &&
            !mbar_wait_warp(bar(Tr::B_Q_EMPTY + qs), ((i / QST) - 1) & 1, w, kBSiteQEmpty))
          break;
        const uint32_t fb = bar(Tr::B_Q_FULL + qs);
        mbar_expect_tx(leader, fb, 2 * Tr::QT_BYTES + 2 * BM * 4);
        tma_load_4d(leader, sQ + qs * Tr::QT_BYTES, &tmq, fb, 0, h, tok0 + (i0 + i) * BM, tb);
        tma_load_4d(leader, sDO + qs * Tr::QT_BYTES, &tmdo, fb, 0, h, tok0 + (i0 + i) * BM, tb);
        bulk_load(leader, base + Tr::OFF_L + qs * BM * 4, p.lse2 + row0 + (size_t)(i0 + i) * BM,
                  BM * 4, fb);
        bulk_load(leader, base + Tr::OFF_DD + qs * BM * 4, p.dvec + row0 + (size_t)(i0 + i) * BM,
                  BM * 4, fb);
        ++issued;
      }
      mbar_drain(bar(Tr::B_KV_FULL), 0, p.limit_ns);
      for (int s = 0; s < QST; ++s)
        if (issued > s) mbar_drain(bar(Tr::B_Q_FULL + s), ((issued - 1 - s) / QST) & 1, p.limit_ns);
    }
    __syncwarp();
  } else if (warp == 9 || warp == 10) {
    // ------------------------------------------------------ MMA issuers
    // Two independent streams on two SM sub-partitions (an issuing warp
    // shares its sub-partition's issue slots with two compute warps):
    //   warp 9:  S^T = K Q_i^T and dV += P^T dO_i   (TMEM S^T and dV only)
    //   warp 10: dP^T = V dO_i^T, dK += dS^T Q_i, dQ_i = dS K  (dP^T, dK, dQ)
    // They share no TMEM columns; the Q/dO stage release and the final
    // "all done" barriers count one commit from each.
    {
      const bool stream_a = warp == 9;
      const bool leader = lane == 0;  // issues; all lanes run the loop
      constexpr uint32_t fmt = Elem<T>::kFmt;
      constexpr uint32_t kIdescSP = f16_idesc(fmt, 128, BM, false);            // K-major x K-major
      constexpr uint32_t kIdescAcc = f16_idesc(fmt, 128, D, true);             // TS, B MN-major
      constexpr uint32_t kIdescDQ = f16_idesc(fmt, 128, D, true) | (1u << 15);  // A, B MN-major
      // Packed 16-bit P^T / dS^T: query half hf sits in the first 32 columns of
      // its own 64-column half of the S^T / dP^T region (a half never writes
      // columns that the other half may still be reading).
      auto packed_col = [](int kk) -> uint32_t {
        return (uint32_t)((kk / (HC / 16)) * HC + (kk % (HC / 16)) * 8);
      };
      // Descriptors are built once; each MMA only advances a start address.
      const uint64_t k_kmaj = sw128_desc(sK, 16, 1024), v_kmaj = sw128_desc(sV, 16, 1024),
                     q_kmaj = sw128_desc(sQ, 16, 1024), do_kmaj = sw128_desc(sDO, 16, 1024),
                     q_mn = sw128_desc(sQ, BM * 128, 1024), do_mn = sw128_desc(sDO, BM * 128, 1024),
                     ds_mn = sw128_desc(sDS, BN * 128, 1024), k_mn = sw128_desc(sK, BN * 128, 1024);
      // S^T = K Q_i^T into TM_S (stream a); dP^T = V dO_i^T into TM_DP (stream b)
      auto issue_first = [&](int i) {
        const uint64_t a0 = stream_a ? k_kmaj : v_kmaj;
        const uint64_t b0 = desc_advance(stream_a ? q_kmaj : do_kmaj, (i % QST) * Tr::QT_BYTES);
        const uint32_t d_tmem = tmem + (stream_a ? Tr::TM_S : Tr::TM_DP);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ch = kk >> 2, in = (kk & 3) * 32;
          umma_ss(leader, d_tmem, desc_advance(a0, ch * (BN * 128) + in),
                  desc_advance(b0, ch * (BM * 128) + in), kIdescSP, kk > 0 ? 1u : 0u);
        }
        umma_commit(leader, bar(stream_a ? Tr::B_S_FULL : Tr::B_DP_FULL));
      };
      bool ok = mbar_wait_warp(bar(Tr::B_KV_FULL), 0, w, kBSiteKV);
      if (ok && n_qt > 0 && (ok = mbar_wait_warp(bar(Tr::B_Q_FULL), 0, w, kBSiteQFull))) {
        tc_fence_after();
        issue_first(0);
      }
      for (int i = 0; i < n_qt && ok; ++i) {
        const bool more = i + 1 < n_qt;
        if (stream_a) {
          // dV += P^T dO_i  (A = P^T from TMEM, B = dO_i: queries x d, MN-major)
          if (!(ok = mbar_wait_warp(bar(Tr::B_P_READY), i & 1, w, kBSitePReady))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk)
            umma_ts(leader, tmem + Tr::TM_DV, tmem + Tr::TM_S + packed_col(kk),
                    desc_advance(do_mn, (i % QST) * Tr::QT_BYTES + kk * 16 * 128), kIdescAcc,
                    (i > 0 || kk > 0) ? 1u : 0u);
          umma_commit(leader, bar(Tr::B_Q_EMPTY + i % QST));
        } else {
          // dK += dS^T Q_i  (A = dS^T from TMEM, B = Q_i MN-major)
          if (!(ok = mbar_wait_warp(bar(Tr::B_DS_READY), i & 1, w, kBSiteDsReady))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk)
            umma_ts(leader, tmem + Tr::TM_DK, tmem + Tr::TM_DP + packed_col(kk),
                    desc_advance(q_mn, (i % QST) * Tr::QT_BYTES + kk * 16 * 128), kIdescAcc,
                    (i > 0 || kk > 0) ? 1u : 0u);
          umma_commit(leader, bar(Tr::B_Q_EMPTY + i % QST));
        }
        // the next S^T (dP^T) overwrites TM_S (TM_DP) after dV (dK) has read
        // P^T (dS^T): same issuing thread, so the tensor pipe keeps the order.
        // Stream b issues it ahead of dQ_i, which reads dS from its own
        // shared-memory buffer: the compute warps' next dS^T then waits only
        // for dK, not for dQ and the dQ drain
        if (more) {
          if (!(ok = mbar_wait_warp(bar(Tr::B_Q_FULL + (i + 1) % QST), ((i + 1) / QST) & 1, w,
                                    kBSiteQFull)))
            break;
          tc_fence_after();
          issue_first(i + 1);
        }
        if (!stream_a) {
          // dQ_i = dS K  (A = dS from shared memory, queries contiguous; B = K, d contiguous)
          if (i > 0 && !(ok = mbar_wait_warp(bar(Tr::B_DQ_FREE), (i - 1) & 1, w, kBSiteDqFree)))
            break;
          tc_fence_after();
          const uint64_t dsd = desc_advance(ds_mn, (i & 1) * Tr::DS_BYTES);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            umma_ss(leader, tmem + Tr::TM_DQ, desc_advance(dsd, kk * 16 * 128),
                    desc_advance(k_mn, kk * 16 * 128), kIdescDQ, kk > 0 ? 1u : 0u);
          umma_commit(leader, bar(Tr::B_DQ_FULL));
          umma_commit(leader, bar(Tr::B_DSBUF_FREE + (i & 1)));
        }
      }
      umma_commit(leader, bar(Tr::B_KV_DONE));
      umma_commit(leader, bar(Tr::B_DRAIN));
      mbar_drain(bar(Tr::B_DRAIN), 0, p.limit_ns);
    }
    __syncwarp();
  }  // warp 11 has no role
  } else {
    regs_grow();  // both compute warpgroups
    // ----------------------------- compute warps 0-7: P^T, dS^T, dQ drain
    // Warp w owns TMEM lane quadrant w % 4 (key rows of S^T/dP^T, query rows
    // of dQ) and half hf = w / 4 of the columns.
    const int quad = warp & 3, hf = warp >> 2;
    const int r = quad * 32 + lane;  // key row (S^T, dP^T) and query row (dQ)
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
    const bool key_valid = kt * BN + r < len;
    const float c = p.sl2;
    bool ok = true;

    // dQ tile i: TMEM -> this warp's swizzled fp32 staging box (its 32 query
    // rows x 32 d columns) -> TMA reduce-add issued by its lane 0.  Each warp
    // only waits for its own previous reduce: no barrier across warps.
    uint8_t* gbox = gSTG + warp * 4096;
    auto drain_dq = [&](int i) -> bool {
      bool good = mbar_wait(bar(Tr::B_DQ_FULL), i & 1, w, kBSiteDqFull);
      if (!__all_sync(0xffffffffu, good)) return false;
      uint32_t v[32];
      tc_fence_after();
      tmem_ld32(tl + Tr::TM_DQ + hf * 32, v);
      tmem_wait_ld();
      reg_fence(v);
      tc_fence_before();
      mbar_arrive(bar(Tr::B_DQ_FREE));
      if (lane == 0) bulk_wait_read_all();  // the previous reduce has read the box
      __syncwarp();
#pragma unroll
      for (int u = 0; u < 8; ++u)
        *reinterpret_cast<float4*>(gbox + lane * 128 + ((u ^ (lane & 7)) * 16)) =
            make_float4(__uint_as_float(v[4 * u]), __uint_as_float(v[4 * u + 1]),
                        __uint_as_float(v[4 * u + 2]), __uint_as_float(v[4 * u + 3]));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && *abort_flag == 0) {
        const int row = (int)(((size_t)b * p.H + h) * p.Npad + (size_t)(i0 + i) * BM + quad * 32);
        tma_reduce_add_2d(&tmacc, sSTG + warp * 4096, hf * 32, row);
        bulk_commit();
      }
      return true;
    };

    for (int i = 0; i < n_qt; ++i) {
      const int qs = i % QST;
      // ---- P^T = 2^(c S^T - LSE2) for this warp's 64 query columns
      ok = mbar_wait(bar(Tr::B_S_FULL), i & 1, w, kBSiteSFull);
      ok = ok && mbar_wait(bar(Tr::B_Q_FULL + qs), (i / QST) & 1, w, kBSiteQFullSm);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      const float4* l4 = reinterpret_cast<const float4*>(sL + qs * BM + hf * HC);
      const float4* d4 = reinterpret_cast<const float4*>(sDD + qs * BM + hf * HC);
      float pr[HC];
      {
        uint32_t sr[2][32];
        tmem_ld32(tl + Tr::TM_S + hf * HC, sr[0]);
        tmem_ld32(tl + Tr::TM_S + hf * HC + 32, sr[1]);
        tmem_wait_ld();
        reg_fence(sr[0]);
        reg_fence(sr[1]);
        const uint64_t c2 = f32x2(c, c);
#pragma unroll
        for (int j4 = 0; j4 < HC / 4; ++j4) {
          const float4 L = l4[j4];  // minus the base-2 LSE of four queries
          const int j = 4 * j4;
          fma2(pr[j], pr[j + 1], __uint_as_float(sr[j / 32][j % 32]),
               __uint_as_float(sr[j / 32][j % 32 + 1]), c2, f32x2(L.x, L.y));
          fma2(pr[j + 2], pr[j + 3], __uint_as_float(sr[j / 32][j % 32 + 2]),
               __uint_as_float(sr[j / 32][j % 32 + 3]), c2, f32x2(L.z, L.w));
          // of every 8 column pairs, EMU take the FMA-pipe exponential
          if (((j / 2) & 7) >= 8 - Tr::EMU) {
            ex2_poly2(pr[j], pr[j + 1], pr[j], pr[j + 1]);
          } else {
            pr[j] = ex2(pr[j]);
            pr[j + 1] = ex2(pr[j + 1]);
          }
          if ((((j + 2) / 2) & 7) >= 8 - Tr::EMU) {
            ex2_poly2(pr[j + 2], pr[j + 3], pr[j + 2], pr[j + 3]);
          } else {
            pr[j + 2] = ex2(pr[j + 2]);
            pr[j + 3] = ex2(pr[j + 3]);
          }
        }
        // P = 0 for keys past N, and with the causal mask for the columns
        // whose query comes before this key (query - key < 0: the first
        // `hidden` of this warp's columns)
        int hidden = key_valid ? 0 : HC;
        if (CAUSAL) hidden = max(hidden, min(HC, (kt * BN + r) - ((i0 + i) * BM + hf * HC)));
        if (hidden > 0) {
#pragma unroll
          for (int j = 0; j < HC; ++j)
            if (j < hidden) pr[j] = 0.f;
        }
        uint32_t pk[HC / 2];
#pragma unroll
        for (int j = 0; j < HC / 2; ++j) pk[j] = Elem<T>::pack(pr[2 * j], pr[2 * j + 1]);
        tmem_st16(tl + Tr::TM_S + hf * HC, &pk[0]);
        tmem_st16(tl + Tr::TM_S + hf * HC + 16, &pk[16]);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(bar(Tr::B_P_READY));
      // ---- dS^T = P^T o (dP^T - D) for the same columns
      ok = mbar_wait(bar(Tr::B_DP_FULL), i & 1, w, kBSiteDpFull);
      if (i >= 2)
        ok = ok && mbar_wait(bar(Tr::B_DSBUF_FREE + (i & 1)), ((i >> 1) - 1) & 1, w, kBSiteDsBuf);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      uint32_t dk16[HC / 2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {  // 32 columns at a time: fewer live registers
        uint32_t dr[32];
        tmem_ld32(tl + Tr::TM_DP + hf * HC + hh * 32, dr);
        tmem_wait_ld();
        reg_fence(dr);
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
          const float4 Dv = d4[hh * 8 + j4];
          const int j = 32 * hh + 4 * j4;
          float ds[4];
          sub_mul2(ds[0], ds[1], __uint_as_float(dr[4 * j4]), __uint_as_float(dr[4 * j4 + 1]),
                   Dv.x, Dv.y, pr[j], pr[j + 1]);
          sub_mul2(ds[2], ds[3], __uint_as_float(dr[4 * j4 + 2]), __uint_as_float(dr[4 * j4 + 3]),
                   Dv.z, Dv.w, pr[j + 2], pr[j + 3]);
          dk16[16 * hh + 2 * j4] = Elem<T>::pack(ds[0], ds[1]);
          dk16[16 * hh + 2 * j4 + 1] = Elem<T>::pack(ds[2], ds[3]);
        }
      }
      tmem_st16(tl + Tr::TM_DP + hf * HC, &dk16[0]);
      tmem_st16(tl + Tr::TM_DP + hf * HC + 16, &dk16[16]);
      // dS row r, query chunk hf, into the 128-byte-swizzled shared tile
      uint8_t* ds_g = gDS + (i & 1) * Tr::DS_BYTES + hf * (BN * 128) + r * 128;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        *reinterpret_cast<uint4*>(ds_g + ((u ^ (r & 7)) * 16)) =
            make_uint4(dk16[4 * u], dk16[4 * u + 1], dk16[4 * u + 2], dk16[4 * u + 3]);
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(Tr::B_DS_READY));
      // ---- dQ of the previous tile
      if (i > 0 && !(ok = drain_dq(i - 1))) break;
    }
    if (ok && n_qt > 0) ok = drain_dq(n_qt - 1);
    if (lane == 0) bulk_wait_all();
    // ---- epilogue: dV and scale * dK, this warp's key rows and 32 of the d columns
    if (ok) ok = mbar_wait(bar(Tr::B_KV_DONE), 0, w, kBSiteKvDone);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const int key = kt * BN + r;
      uint32_t a[32], k2[32];
      tmem_ld32(tl + Tr::TM_DV + hf * 32, a);
      tmem_ld32(tl + Tr::TM_DK + hf * 32, k2);
      tmem_wait_ld();
      reg_fence(a);
      reg_fence(k2);
      if (key_valid)
        store_dkv32<T, SPLIT>(p, (size_t)tb * p.total + tok0 + key, h, hf * 32, sp, a, k2, D);
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
// fa_bwd_tq_kernel: d = 96, 128 and 256.  At 128 queries per inner tile the five
// accumulators (S^T, dP^T, dQ, dV, dK: 5 x 128 columns) exceed tensor memory,
// so the inner tile holds 64 queries and dQ is produced transposed,
//   dQ_i^T = K^T dS_i^T   (M = d = 128 lanes, N = 64 queries, K = 128 keys),
// into one of two 64-column buffers; the compute warps drain it through a
// per-warp staging box (32 queries x 32 d, fp32) that the warp reduce-adds
// into the accumulator itself.
// Tensor memory: S^T [0,64), dP^T [64,128), dQ^T [128,256) (two buffers),
// dV [256,384), dK [384,512).  Warps as in fa_bwd_kernel; compute warp w owns
// lane quadrant w % 4 and query half w / 4 (32 columns) of S^T and dP^T, and
// d quadrant w % 4, query half w / 4 of dQ^T.
// The single dS^T staging tile is released by a barrier committed after the
// dQ^T MMA of its tile: dP^T of tile i + 1 is issued right after dK of tile i,
// ahead of dQ_i^T, so the compute warps may already build dS^T of tile i + 1
// in registers and tensor memory while dQ_i^T still reads the tile.
// At d = 96 the tiles keep the d = 128 layout: the second 64-column chunk of
// every shared-memory row is half zero fill from the tensor map; S^T and dP^T
// contract the 96 real columns, dV and dK are 96 columns wide (dK at
// [352,448)), and dQ^T is still a 128-lane tile whose lanes 96-127 (K^T rows
// of zeros) are never drained.
// At d = 256 two blocks share each key tile, block half dh producing columns
// [128 dh, 128 dh + 128) of dK, dV and rows of dQ^T (the same tensor memory
// layout as d = 128); S^T and dP^T contract all 256 columns in both.  The
// resident 64 KB K and V tiles leave room for one Q/dO stage and four dQ
// staging boxes, which warps 0-3 use for both query halves of their quadrant.
// ===========================================================================
template <int D_, int QST_>
struct BwdTqTraits {
  static constexpr int D = D_;
  static constexpr int BN = 128;  // keys per block
  static constexpr int BM = 64;   // queries per inner tile
  static constexpr int QST = QST_;
  // d columns of dK, dV (and d rows of dQ^T) a block produces: all of them up
  // to d = 128; at d = 256 two blocks per key tile take one 128-wide half
  // each (S^T and dP^T still contract all 256)
  static constexpr int DW = D < 128 ? D : 128;
  static constexpr int NHALF = D / DW;
  // dQ staging: one 32 x 32 fp32 box per compute warp, or (d = 256, where the
  // full K, V tiles leave less room) one per lane quadrant, drained by warps
  // 0-3 for both query halves
  static constexpr int NBOX = NHALF > 1 ? 4 : 8;
  // 128-byte chunks along d; at d = 96 the last 32 columns of the second
  // chunk are the tensor map's zero fill
  static constexpr int KCH = (D + 63) / 64;
  static constexpr int KV_BYTES = BN * KCH * 128;
  static constexpr int QT_BYTES = BM * KCH * 128;
  static constexpr int DS_BYTES = BN * BM * 2;       // dS^T tile: keys x 64 queries, 16-bit
  static constexpr int BOX_BYTES = 32 * 32 * 4;      // a warp's dQ staging box
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_BYTES;
  static constexpr int OFF_Q = OFF_V + KV_BYTES;
  static constexpr int OFF_DO = OFF_Q + QST * QT_BYTES;
  static constexpr int OFF_DS = OFF_DO + QST * QT_BYTES;
  static constexpr int OFF_STG = OFF_DS + DS_BYTES;
  static constexpr int OFF_L = OFF_STG + NBOX * BOX_BYTES;  // minus the base-2 LSE, per stage
  static constexpr int OFF_DD = OFF_L + QST * BM * 4;    // D per stage
  static constexpr int OFF_BAR = OFF_DD + QST * BM * 4;
  static constexpr int B_KV_FULL = 0, B_Q_FULL = 1, B_Q_EMPTY = B_Q_FULL + QST,
                       B_S_FULL = B_Q_EMPTY + QST, B_DP_FULL = B_S_FULL + 1,
                       B_P_READY = B_DP_FULL + 1, B_DS_READY = B_P_READY + 1,
                       B_DQ_FULL = B_DS_READY + 1, B_DQ_FREE = B_DQ_FULL + 2,
                       B_DSBUF_FREE = B_DQ_FREE + 2, B_KV_DONE = B_DSBUF_FREE + 1,
                       B_DRAIN = B_KV_DONE + 1, NUM_BARS = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr uint32_t TM_S = 0, TM_DP = 64, TM_DQ = 128, TM_DV = 256, TM_DK = 256 + DW;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int ACC_BOX_ROWS = 32;  // dQ reduce box: 32 d columns x 32 queries
  // dP^T of the next tile ahead of dQ^T (below).  At d = 256 the single Q/dO
  // stage already serialises the tiles, and the early order measured slower
  // (B200, [1,6400,1,256] backward: 279.8 against 274.0 us)
  static constexpr bool EARLY_DP = NHALF == 1;
  // dQ^T has DW rows: one 128-lane MMA tile (rows past d are zero and never drained)
  static_assert(D == 96 || D == 128 || D == 256, "head sizes of the transposed-dQ kernel");
  static_assert(TM_DK + DW <= TMEM_COLS, "tensor memory budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(OFF_Q % 1024 == 0 && OFF_DO % 1024 == 0 && OFF_DS % 1024 == 0 &&
                    OFF_STG % 1024 == 0 && QT_BYTES % 1024 == 0,
                "swizzled tiles start on 1024-byte boundaries");
};

using BwdTq128 = BwdTqTraits<128, 3>;
using BwdTq96 = BwdTqTraits<96, 3>;
using BwdTq256 = BwdTqTraits<256, 1>;  // resident 64 KB K and V tiles leave one Q/dO stage

template <class T, class Tr, bool CAUSAL, bool VARLEN, bool SPLIT = false>
__global__ void __launch_bounds__(384, 1)
    fa_bwd_tq_kernel(const __grid_constant__ CUtensorMap tmq,
                     const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv,
                     const __grid_constant__ CUtensorMap tmdo,
                     const __grid_constant__ CUtensorMap tmacc, const BwdParams p) {
  constexpr int D = Tr::D, BN = Tr::BN, BM = Tr::BM, QST = Tr::QST, KCH = Tr::KCH;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sK = base + Tr::OFF_K, sV = base + Tr::OFF_V, sQ = base + Tr::OFF_Q,
                 sDO = base + Tr::OFF_DO, sDS = base + Tr::OFF_DS, sSTG = base + Tr::OFF_STG;
  const float* sL = reinterpret_cast<const float*>(gbase + Tr::OFF_L);
  const float* sDD = reinterpret_cast<const float*>(gbase + Tr::OFF_DD);
  uint8_t* gDS = gbase + Tr::OFF_DS;
  uint8_t* gSTG = gbase + Tr::OFF_STG;
  const uint32_t bars = base + Tr::OFF_BAR;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + Tr::OFF_MISC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + Tr::OFF_MISC + 4);
  auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitCtl w{abort_flag, p.limit_ns, p.status};
  // a 1-D grid (B * H may exceed the 65,535 limit of gridDim.y and .z); within
  // a (batch, head): x = (key tile * n_split + split) * NHALF + d half.  Causal
  // key tiles see fewer query tiles the later they are, so there the order is
  // x-major: every head's long key tiles start first
  constexpr int DW = Tr::DW, NHALF = Tr::NHALF;
  const unsigned n_bh = (unsigned)(p.B * p.H);
  const int bx = CAUSAL ? (int)(blockIdx.x / n_bh) : (int)(blockIdx.x % (unsigned)p.n_x);
  const int bh = CAUSAL ? (int)(blockIdx.x % n_bh) : (int)(blockIdx.x / (unsigned)p.n_x);
  const int dh = NHALF > 1 ? bx % NHALF : 0;  // d half this block produces
  const int xs = NHALF > 1 ? bx / NHALF : bx;
  const int sp = SPLIT ? xs % p.n_split : 0;  // split of the query range
  const int kt = SPLIT ? xs / p.n_split : xs;
  const int h = bh % p.H, b = bh / p.H;
  // the block's sequence on the token axis (batch entry tb, tokens tok0 ..
  // tok0 + len); a key tile past a shorter sequence's end has no work
  int tb, tok0, len;
  seq_bounds(VARLEN ? p.cu : nullptr, b, p.N, p.total, tb, tok0, len);
  if (kt * BN >= len) return;  // block-uniform, before any barrier or allocation
  // causal: query tiles wholly before this key tile see none of its keys
  const int q0 = CAUSAL ? (kt * BN) / BM : 0;
  const int q_all = (VARLEN ? (len + BM - 1) / BM : p.n_qt) - q0;
  // tile i is global i0 + i; a split block takes its share of the range
  const int i0 = SPLIT ? q0 + q_all * sp / p.n_split : q0;
  const int n_qt = SPLIT ? q_all * (sp + 1) / p.n_split - q_all * sp / p.n_split : q_all;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(Tr::B_KV_FULL), 1);
    for (int s = 0; s < QST; ++s) {
      mbar_init(bar(Tr::B_Q_FULL + s), 1);
      mbar_init(bar(Tr::B_Q_EMPTY + s), 2);  // one commit from each MMA warp
    }
    mbar_init(bar(Tr::B_S_FULL), 1);
    mbar_init(bar(Tr::B_DP_FULL), 1);
    mbar_init(bar(Tr::B_P_READY), 256);
    mbar_init(bar(Tr::B_DS_READY), 256);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(Tr::B_DQ_FULL + s), 1);
      mbar_init(bar(Tr::B_DQ_FREE + s), 32 * Tr::NBOX);  // the draining warps
    }
    mbar_init(bar(Tr::B_DSBUF_FREE), 1);
    mbar_init(bar(Tr::B_KV_DONE), 2);
    mbar_init(bar(Tr::B_DRAIN), 2);
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
    tma_prefetch_desc(&tmdo);
    tma_prefetch_desc(&tmacc);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= 8) {
    regs_shrink();  // all four warps of the producer/MMA warpgroup
  if (warp == 8) {
    // -------------------------------------------------------- producer
    {
      const bool leader = lane == 0;  // issues; all lanes run the loop
      mbar_expect_tx(leader, bar(Tr::B_KV_FULL), 2 * Tr::KV_BYTES);
#pragma unroll
      for (int c = 0; c < KCH; ++c) {
        tma_load_4d(leader, sK + c * (BN * 128), &tmk, bar(Tr::B_KV_FULL), c * 64, h,
                    tok0 + kt * BN, tb);
        tma_load_4d(leader, sV + c * (BN * 128), &tmv, bar(Tr::B_KV_FULL), c * 64, h,
                    tok0 + kt * BN, tb);
      }
      const size_t row0 = ((size_t)b * p.H + h) * p.Npad;
      int issued = 0;
      for (int i = 0; i < n_qt; ++i) {
        const int qs = i % QST;
        if (i >= QST &&
            !mbar_wait_warp(bar(Tr::B_Q_EMPTY + qs), ((i / QST) - 1) & 1, w, kBSiteQEmpty))
          break;
        const uint32_t fb = bar(Tr::B_Q_FULL + qs);
        mbar_expect_tx(leader, fb, 2 * Tr::QT_BYTES + 2 * BM * 4);
#pragma unroll
        for (int c = 0; c < KCH; ++c) {
          tma_load_4d(leader, sQ + qs * Tr::QT_BYTES + c * (BM * 128), &tmq, fb, c * 64, h,
                      tok0 + (i0 + i) * BM, tb);
          tma_load_4d(leader, sDO + qs * Tr::QT_BYTES + c * (BM * 128), &tmdo, fb, c * 64, h,
                      tok0 + (i0 + i) * BM, tb);
        }
        bulk_load(leader, base + Tr::OFF_L + qs * BM * 4, p.lse2 + row0 + (size_t)(i0 + i) * BM,
                  BM * 4, fb);
        bulk_load(leader, base + Tr::OFF_DD + qs * BM * 4, p.dvec + row0 + (size_t)(i0 + i) * BM,
                  BM * 4, fb);
        ++issued;
      }
      mbar_drain(bar(Tr::B_KV_FULL), 0, p.limit_ns);
      for (int s = 0; s < QST; ++s)
        if (issued > s) mbar_drain(bar(Tr::B_Q_FULL + s), ((issued - 1 - s) / QST) & 1, p.limit_ns);
    }
    __syncwarp();
  } else if (warp == 9 || warp == 10) {
    // ------------------------------------------------------ MMA issuers
    //   warp 9:  S^T = K Q_i^T and dV += P^T dO_i         (TMEM S^T, dV)
    //   warp 10: dP^T = V dO_i^T, dK += dS^T Q_i, dQ_i^T  (TMEM dP^T, dK, dQ^T)
    {
      const bool stream_a = warp == 9;
      const bool leader = lane == 0;  // issues; all lanes run the loop
      constexpr uint32_t fmt = Elem<T>::kFmt;
      constexpr uint32_t kIdescSP = f16_idesc(fmt, 128, BM, false);              // K-major x K-major
      constexpr uint32_t kIdescAcc = f16_idesc(fmt, 128, DW, true);              // TS, B MN-major
      constexpr uint32_t kIdescDQ = f16_idesc(fmt, 128, BM, true) | (1u << 15);  // A, B MN-major
      // Packed 16-bit P^T / dS^T: query half hf sits in the first 16 columns of
      // its own 32-column half of the S^T / dP^T region.
      auto packed_col = [](int kk) -> uint32_t { return (uint32_t)((kk >> 1) * 32 + (kk & 1) * 8); };
      const uint64_t k_kmaj = sw128_desc(sK, 16, 1024), v_kmaj = sw128_desc(sV, 16, 1024),
                     q_kmaj = sw128_desc(sQ, 16, 1024), do_kmaj = sw128_desc(sDO, 16, 1024),
                     q_mn = sw128_desc(sQ, BM * 128, 1024), do_mn = sw128_desc(sDO, BM * 128, 1024),
                     k_mn = sw128_desc(sK, BN * 128, 1024), ds_mn = sw128_desc(sDS, BN * 128, 1024);
      // the block's d half starts DW/64 chunks into the Q, dO and K tiles
      const uint32_t d_off_q = (uint32_t)(dh * (DW / 64) * (BM * 128));
      const uint32_t d_off_k = (uint32_t)(dh * (DW / 64) * (BN * 128));
      // S^T = K Q_i^T into TM_S (stream a); dP^T = V dO_i^T into TM_DP (stream b)
      auto issue_first = [&](int i) {
        const uint64_t a0 = stream_a ? k_kmaj : v_kmaj;
        const uint64_t b0 = desc_advance(stream_a ? q_kmaj : do_kmaj, (i % QST) * Tr::QT_BYTES);
        const uint32_t d_tmem = tmem + (stream_a ? Tr::TM_S : Tr::TM_DP);
        // (at d = 256 partly unrolled: the issuing warps run on 88 registers)
        constexpr int kUnroll = D > 128 ? 4 : D / 16;
#pragma unroll kUnroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ch = kk >> 2, in = (kk & 3) * 32;
          umma_ss(leader, d_tmem, desc_advance(a0, ch * (BN * 128) + in),
                  desc_advance(b0, ch * (BM * 128) + in), kIdescSP, kk > 0 ? 1u : 0u);
        }
        umma_commit(leader, bar(stream_a ? Tr::B_S_FULL : Tr::B_DP_FULL));
      };
      bool ok = mbar_wait_warp(bar(Tr::B_KV_FULL), 0, w, kBSiteKV);
      if (ok && n_qt > 0 && (ok = mbar_wait_warp(bar(Tr::B_Q_FULL), 0, w, kBSiteQFull))) {
        tc_fence_after();
        issue_first(0);
      }
      for (int i = 0; i < n_qt && ok; ++i) {
        const bool more = i + 1 < n_qt;
        const int qs = i % QST;
        if (stream_a) {
          // dV += P^T dO_i  (A = P^T from TMEM, B = dO_i: queries x d, MN-major)
          if (!(ok = mbar_wait_warp(bar(Tr::B_P_READY), i & 1, w, kBSitePReady))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk)
            umma_ts(leader, tmem + Tr::TM_DV, tmem + Tr::TM_S + packed_col(kk),
                    desc_advance(do_mn, qs * Tr::QT_BYTES + d_off_q + kk * 16 * 128), kIdescAcc,
                    (i > 0 || kk > 0) ? 1u : 0u);
          umma_commit(leader, bar(Tr::B_Q_EMPTY + qs));
        } else {
          // dK += dS^T Q_i  (A = dS^T from TMEM, B = Q_i MN-major)
          if (!(ok = mbar_wait_warp(bar(Tr::B_DS_READY), i & 1, w, kBSiteDsReady))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk)
            umma_ts(leader, tmem + Tr::TM_DK, tmem + Tr::TM_DP + packed_col(kk),
                    desc_advance(q_mn, qs * Tr::QT_BYTES + d_off_q + kk * 16 * 128), kIdescAcc,
                    (i > 0 || kk > 0) ? 1u : 0u);
          umma_commit(leader, bar(Tr::B_Q_EMPTY + qs));
        }
        // the next S^T (dP^T) after dV (dK) has read P^T (dS^T): same thread,
        // in order.  With EARLY_DP stream b issues it ahead of dQ_i^T: the
        // compute warps may then build the next dS^T while dQ_i^T runs, and
        // wait for DSBUF_FREE before they rewrite the shared dS^T tile it reads
        if (more && (stream_a || Tr::EARLY_DP)) {
          if (!(ok = mbar_wait_warp(bar(Tr::B_Q_FULL + (i + 1) % QST), ((i + 1) / QST) & 1, w,
                                    kBSiteQFull)))
            break;
          tc_fence_after();
          issue_first(i + 1);
        }
        if (!stream_a) {
          // dQ_i^T = K^T dS_i^T  (A = K: d contiguous, MN-major; B = dS^T: queries
          // contiguous, MN-major) into buffer i & 1, once its previous tile is drained
          const int qb = i & 1;
          if (i >= 2 &&
              !(ok = mbar_wait_warp(bar(Tr::B_DQ_FREE + qb), ((i >> 1) - 1) & 1, w, kBSiteDqFree)))
            break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            umma_ss(leader, tmem + Tr::TM_DQ + qb * BM,
                    desc_advance(k_mn, d_off_k + kk * 16 * 128),
                    desc_advance(ds_mn, kk * 16 * 128), kIdescDQ, kk > 0 ? 1u : 0u);
          umma_commit(leader, bar(Tr::B_DQ_FULL + qb));
          umma_commit(leader, bar(Tr::B_DSBUF_FREE));
          if (more && !Tr::EARLY_DP) {
            if (!(ok = mbar_wait_warp(bar(Tr::B_Q_FULL + (i + 1) % QST), ((i + 1) / QST) & 1, w,
                                      kBSiteQFull)))
              break;
            tc_fence_after();
            issue_first(i + 1);
          }
        }
      }
      umma_commit(leader, bar(Tr::B_KV_DONE));
      umma_commit(leader, bar(Tr::B_DRAIN));
      mbar_drain(bar(Tr::B_DRAIN), 0, p.limit_ns);
    }
    __syncwarp();
  }  // warp 11 has no role
  } else {
    regs_grow();  // both compute warpgroups
    // ----------------------------- compute warps 0-7: P^T, dS^T, dQ drain
    const int quad = warp & 3, hf = warp >> 2;
    const int r = quad * 32 + lane;  // key row (S^T, dP^T), d row (dQ^T)
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
    const bool key_valid = kt * BN + r < len;
    const float c = p.sl2;
    // staging box: one per warp, or (NBOX = 4) one per lane quadrant, whose
    // warp 0-3 drains both query halves
    constexpr int NH = 8 / Tr::NBOX;  // query halves a draining warp handles
    const bool drains = warp < Tr::NBOX;
    const uint32_t box = sSTG + (Tr::NBOX == 8 ? warp : quad) * Tr::BOX_BYTES;
    uint8_t* gbox = gSTG + (Tr::NBOX == 8 ? warp : quad) * Tr::BOX_BYTES;
    bool ok = true;

    // dQ^T tile i: TMEM -> the warp's swizzled fp32 staging box (32 queries x
    // 32 d) -> TMA reduce-add into the accumulator, issued by lane 0.
    auto drain_dq = [&](int i) -> bool {
      const int qb = i & 1;
      bool good = mbar_wait(bar(Tr::B_DQ_FULL + qb), (i >> 1) & 1, w, kBSiteDqFull);
      if (!__all_sync(0xffffffffu, good)) return false;
      tc_fence_after();
#pragma unroll
      for (int e = 0; e < NH; ++e) {
        const int half = NH == 1 ? hf : e;
        uint32_t v[32];
        tmem_ld32(tl + Tr::TM_DQ + qb * BM + half * 32, v);
        tmem_wait_ld();
        reg_fence(v);
        if (e == NH - 1) {  // every read of this dQ^T buffer is done
          tc_fence_before();
          mbar_arrive(bar(Tr::B_DQ_FREE + qb));
        }
        if (lane == 0) bulk_wait_read_all();  // the previous reduce has read the box
        __syncwarp();
        // v[j] = dQ[query 32 half + j][d = 32 quad + lane]; box row j holds query j
#pragma unroll
        for (int j = 0; j < 32; ++j)
          *reinterpret_cast<float*>(gbox + j * 128 + ((((lane >> 2) ^ (j & 7))) << 4) +
                                    (lane & 3) * 4) = __uint_as_float(v[j]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && *abort_flag == 0 && quad * 32 < DW) {  // d rows past d are padding
          const int row =
              (int)(((size_t)b * p.H + h) * p.Npad + (size_t)(i0 + i) * BM + half * 32);
          tma_reduce_add_2d(&tmacc, box, dh * DW + quad * 32, row);
          bulk_commit();
        }
      }
      return true;
    };

    for (int i = 0; i < n_qt; ++i) {
      const int qs = i % QST;
      // ---- P^T = 2^(c S^T - LSE2) for this warp's 32 query columns
      ok = mbar_wait(bar(Tr::B_S_FULL), i & 1, w, kBSiteSFull);
      ok = ok && mbar_wait(bar(Tr::B_Q_FULL + qs), (i / QST) & 1, w, kBSiteQFullSm);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      const float4* l4 = reinterpret_cast<const float4*>(sL + qs * BM + hf * 32);
      const float4* d4 = reinterpret_cast<const float4*>(sDD + qs * BM + hf * 32);
      float pr[32];
      {
        uint32_t sr[32];
        tmem_ld32(tl + Tr::TM_S + hf * 32, sr);
        tmem_wait_ld();
        reg_fence(sr);
        const uint64_t c2 = f32x2(c, c);
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
          const float4 L = l4[j4];  // minus the base-2 LSE of four queries
          fma2(pr[4 * j4], pr[4 * j4 + 1], __uint_as_float(sr[4 * j4]),
               __uint_as_float(sr[4 * j4 + 1]), c2, f32x2(L.x, L.y));
          fma2(pr[4 * j4 + 2], pr[4 * j4 + 3], __uint_as_float(sr[4 * j4 + 2]),
               __uint_as_float(sr[4 * j4 + 3]), c2, f32x2(L.z, L.w));
#pragma unroll
          for (int e = 0; e < 4; ++e) pr[4 * j4 + e] = ex2(pr[4 * j4 + e]);
        }
        int hidden = key_valid ? 0 : 32;  // as in fa_bwd_kernel
        if (CAUSAL) hidden = max(hidden, min(32, (kt * BN + r) - ((i0 + i) * BM + hf * 32)));
        if (hidden > 0) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < hidden) pr[j] = 0.f;
        }
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) pk[j] = Elem<T>::pack(pr[2 * j], pr[2 * j + 1]);
        tmem_st16(tl + Tr::TM_S + hf * 32, pk);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(bar(Tr::B_P_READY));
      // ---- dS^T = P^T o (dP^T - D) for the same columns
      ok = mbar_wait(bar(Tr::B_DP_FULL), i & 1, w, kBSiteDpFull);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      uint32_t ds16[16];
      {
        uint32_t dr[32];
        tmem_ld32(tl + Tr::TM_DP + hf * 32, dr);
        tmem_wait_ld();
        reg_fence(dr);
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
          const float4 Dv = d4[j4];
          float ds[4];
          sub_mul2(ds[0], ds[1], __uint_as_float(dr[4 * j4]), __uint_as_float(dr[4 * j4 + 1]),
                   Dv.x, Dv.y, pr[4 * j4], pr[4 * j4 + 1]);
          sub_mul2(ds[2], ds[3], __uint_as_float(dr[4 * j4 + 2]), __uint_as_float(dr[4 * j4 + 3]),
                   Dv.z, Dv.w, pr[4 * j4 + 2], pr[4 * j4 + 3]);
          ds16[2 * j4] = Elem<T>::pack(ds[0], ds[1]);
          ds16[2 * j4 + 1] = Elem<T>::pack(ds[2], ds[3]);
        }
      }
      tmem_st16(tl + Tr::TM_DP + hf * 32, ds16);
      // the shared dS^T tile is rewritten only after dQ^T of the previous tile
      // has read it (without EARLY_DP, dP^T of this tile already followed it)
      if (Tr::EARLY_DP && i > 0) {
        ok = mbar_wait(bar(Tr::B_DSBUF_FREE), (i - 1) & 1, w, kBSiteDsBuf);
        if (!(ok = __all_sync(0xffffffffu, ok))) break;
      }
      // dS^T row r (key), queries [32 hf, 32 hf + 32): 16-byte chunks 4 hf .. 4 hf + 3
      // of the 128-byte-swizzled row
      uint8_t* ds_row = gDS + r * 128;
#pragma unroll
      for (int u = 0; u < 4; ++u)
        *reinterpret_cast<uint4*>(ds_row + (((4 * hf + u) ^ (r & 7)) * 16)) =
            make_uint4(ds16[4 * u], ds16[4 * u + 1], ds16[4 * u + 2], ds16[4 * u + 3]);
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(Tr::B_DS_READY));
      // ---- dQ of the previous tile
      if (drains && i > 0 && !(ok = drain_dq(i - 1))) break;
    }
    if (drains && ok && n_qt > 0) ok = drain_dq(n_qt - 1);
    if (lane == 0) bulk_wait_all();
    // ---- epilogue: dV and scale * dK, key row r, the 32-column d chunks
    // hf, hf + 2, ... (d = 96: chunks 0 and 2 for hf = 0, chunk 1 for hf = 1)
    if (ok) ok = mbar_wait(bar(Tr::B_KV_DONE), 0, w, kBSiteKvDone);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const int key = kt * BN + r;
#pragma unroll
      for (int cc = hf; cc < DW / 32; cc += 2) {  // this block's d slice, from dh * DW
        const int col = cc * 32;
        uint32_t a[32], k2[32];
        tmem_ld32(tl + Tr::TM_DV + col, a);
        tmem_ld32(tl + Tr::TM_DK + col, k2);
        tmem_wait_ld();
        reg_fence(a);
        reg_fence(k2);
        if (key_valid)
          store_dkv32<T, SPLIT>(p, (size_t)tb * p.total + tok0 + key, h, dh * DW + col, sp, a, k2,
                                D);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, Tr::TMEM_COLS);
  }
}

// Lanes of fa_bwd_pre_kernel per row: d / 8 rounded up to a power of two.
constexpr int bwd_pre_lanes(int d) { return d <= 64 ? 8 : d <= 128 ? 16 : 32; }

// D_i = sum_x dO_ix O_ix; minus the base-2 LSE; zero the dQ accumulator.
// Accumulator rows are (b, h, i) with i < Npad for every sequence b; rows past
// the sequence's length get D = 0 and -LSE = -inf (so P = 0 there).  A row
// takes bwd_pre_lanes(D) lanes, each with 16 bytes of O and of dO (the last
// four lanes of a d = 96 row have none).
template <class T, int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const T* __restrict__ o,
                                                         const T* __restrict__ dout,
                                                         const float* __restrict__ lse,
                                                         float* __restrict__ lse2,
                                                         float* __restrict__ dvec,
                                                         float* __restrict__ dq_acc, int B, int H,
                                                         int N, int Npad, const int* cu,
                                                         int total) {
  constexpr int LPR = bwd_pre_lanes(D);  // lanes per row (a power of two)
  constexpr int RPW = 32 / LPR;          // rows per warp
  const int lane = threadIdx.x & 31, sub = lane % LPR;
  const long long row = ((long long)blockIdx.x * 8 + (threadIdx.x >> 5)) * RPW + lane / LPR;
  const bool in = row < (long long)B * H * Npad;
  const bool part = sub * 8 < D;  // d = 96: 12 of a row's 16 lanes hold data
  int i = 0, h = 0, tb = 0, tok0 = 0, len = 0;
  float acc = 0.f;
  if (in) {
    i = (int)(row % Npad);
    h = (int)((row / Npad) % H);
    const int b = (int)(row / ((long long)Npad * H));
    seq_bounds(cu, b, N, total, tb, tok0, len);
    if (i < len && part) {
      const size_t at = (((size_t)tb * total + tok0 + i) * H + h) * D + sub * 8;
      const uint4 a = *reinterpret_cast<const uint4*>(o + at);
      const uint4 c = *reinterpret_cast<const uint4*>(dout + at);
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 x = Elem<T>::unpack(aw[j]), y = Elem<T>::unpack(cw[j]);
        acc += x.x * y.x + x.y * y.y;
      }
    }
  }
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (in) {
    if (part) {
      float4* arow = reinterpret_cast<float4*>(dq_acc + (size_t)row * D + sub * 8);
      arow[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      arow[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (sub == 0) {
      dvec[row] = acc;
      lse2[row] = (i < len) ? -(lse[((size_t)tb * H + h) * total + tok0 + i] * kLog2e) : -INFINITY;
    }
  }
}

// dQ = scale * accumulator, rounded; 8 elements per thread, over the
// accumulator rows (b, h, i < Npad), written for i below the sequence length.
// dq rows are tok_g elements apart (H*D, or 3*H*D inside a packed dQKV).
template <class T, int D>
__global__ void __launch_bounds__(256) fa_bwd_dq_kernel(const float* __restrict__ dq_acc,
                                                        T* __restrict__ dq, int B, int H, int N,
                                                        int Npad, float scale, long long tok_g,
                                                        const int* cu, int total) {
  const long long e = ((long long)blockIdx.x * 256 + threadIdx.x) * 8;
  if (e >= (long long)B * H * Npad * D) return;
  const long long row = e / D;
  const int x = (int)(e % D);
  const int i = (int)(row % Npad);
  const int h = (int)((row / Npad) % H);
  const int b = (int)(row / ((long long)Npad * H));
  int tb, tok0, len;
  seq_bounds(cu, b, N, total, tb, tok0, len);
  if (i >= len) return;
  const float4 a = *reinterpret_cast<const float4*>(dq_acc + e);
  const float4 c = *reinterpret_cast<const float4*>(dq_acc + e + 4);
  uint4 out;
  out.x = Elem<T>::pack(a.x * scale, a.y * scale);
  out.y = Elem<T>::pack(a.z * scale, a.w * scale);
  out.z = Elem<T>::pack(c.x * scale, c.y * scale);
  out.w = Elem<T>::pack(c.z * scale, c.w * scale);
  *reinterpret_cast<uint4*>(dq + ((size_t)tb * total + tok0 + i) * tok_g + (size_t)h * D + x) = out;
}

// dK, dV = sum over the splits of the fp32 partials, rounded; 8 elements per
// thread over the [B*N tokens, H, D] partial layout.  dk, dv rows are tok_g
// elements apart.
template <class T, int D>
__global__ void __launch_bounds__(256) fa_bwd_dkv_kernel(const float* __restrict__ dk_part,
                                                         const float* __restrict__ dv_part,
                                                         int n_split, long long part_stride,
                                                         T* __restrict__ dk, T* __restrict__ dv,
                                                         int H, long long tok_g) {
  const long long e = ((long long)blockIdx.x * 256 + threadIdx.x) * 8;
  if (e >= part_stride) return;
  const long long tok = e / ((long long)H * D);
  const int hx = (int)(e % ((long long)H * D));
  float a[8], c[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) a[j] = c[j] = 0.f;
  for (int sp = 0; sp < n_split; ++sp) {
    const float4* pk = reinterpret_cast<const float4*>(dk_part + sp * part_stride + e);
    const float4* pv = reinterpret_cast<const float4*>(dv_part + sp * part_stride + e);
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const float4 x = __ldcs(pk + h2), y = __ldcs(pv + h2);
      a[4 * h2] += x.x; a[4 * h2 + 1] += x.y; a[4 * h2 + 2] += x.z; a[4 * h2 + 3] += x.w;
      c[4 * h2] += y.x; c[4 * h2 + 1] += y.y; c[4 * h2 + 2] += y.z; c[4 * h2 + 3] += y.w;
    }
  }
  uint4 ok, ov;
  ok.x = Elem<T>::pack(a[0], a[1]); ok.y = Elem<T>::pack(a[2], a[3]);
  ok.z = Elem<T>::pack(a[4], a[5]); ok.w = Elem<T>::pack(a[6], a[7]);
  ov.x = Elem<T>::pack(c[0], c[1]); ov.y = Elem<T>::pack(c[2], c[3]);
  ov.z = Elem<T>::pack(c[4], c[5]); ov.w = Elem<T>::pack(c[6], c[7]);
  *reinterpret_cast<uint4*>(dk + tok * tok_g + hx) = ok;
  *reinterpret_cast<uint4*>(dv + tok * tok_g + hx) = ov;
}

// Number of blocks per key tile: one, unless splitting each key tile's query
// range over s blocks fills the waves of one-block-per-SM launches clearly
// better (efficiency = blocks / (waves * SMs), less 0.03 per extra split for
// the partial dK/dV traffic and pipeline refills), keeping >= 8 query tiles
// a block.
static int choose_bwd_split(long long blocks, int n_qt, int sm_count) {
  auto eff = [&](long long b) {
    const long long waves = (b + sm_count - 1) / sm_count;
    return (double)b / (double)(waves * sm_count);
  };
  int best = 1;
  double best_e = eff(blocks);
  for (int sp = 2; sp <= 4 && n_qt / sp >= 8; ++sp) {
    const double e = eff(blocks * sp) - 0.03 * (sp - 1);
    if (e > best_e + 0.02) {
      best = sp;
      best_e = e;
    }
  }
  return best;
}

// The three launches of one backward pass with scratch at ws (ws_bytes from
// bwd_scratch_bytes): pre-pass, main kernel, dQ conversion.  With n_split > 1
// the main kernel is the SPLIT instantiation and a fourth launch sums its
// partial dK, dV.
template <class T, class Tr>
static int launch_bwd(void (*kern)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                                   const CUtensorMap, const CUtensorMap, const BwdParams),
                      void* ws, const void* q, const void* k, const void* v, const void* o,
                      const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                      int H, int N, float scale, long long tok_in, long long tok_g,
                      cudaStream_t stream, bool timed, const int* cu, int total,
                      int n_split = 1) {
  constexpr int D = Tr::D;
  const bool bf16 = Elem<T>::kFmt == 1;
  CUtensorMap tmq, tmk, tmv, tmdo, tmacc;
  int rc;
  // memory view: B batch entries of N tokens, or one entry of all tokens (varlen)
  if (cu == nullptr) total = N;
  const int mB = cu ? 1 : B;
  if ((rc = make_tmap_bnhd(&tmq, q, bf16, mB, total, H, D, Tr::BM, tok_in)) != FA_OK) return rc;
  if ((rc = make_tmap_bnhd(&tmk, k, bf16, mB, total, H, D, Tr::BN, tok_in)) != FA_OK) return rc;
  if ((rc = make_tmap_bnhd(&tmv, v, bf16, mB, total, H, D, Tr::BN, tok_in)) != FA_OK) return rc;
  if ((rc = make_tmap_bnhd(&tmdo, dout, bf16, mB, total, H, D, Tr::BM, (long long)H * D)) != FA_OK)
    return rc;
  const int n_qt = (N + Tr::BM - 1) / Tr::BM;
  const int Npad = n_qt * Tr::BM;
  const size_t rows = (size_t)B * H * Npad;
  BwdParams p{};
  p.dq_acc = static_cast<float*>(ws);
  float* lse2 = p.dq_acc + rows * D;
  float* dvec = lse2 + rows;
  p.lse2 = lse2;
  p.dvec = dvec;
  p.dk = dk;
  p.dv = dv;
  p.B = B;
  p.H = H;
  p.N = N;
  p.Npad = Npad;
  p.n_qt = n_qt;
  p.tok_g = tok_g;
  p.cu = cu;
  p.total = total;
  p.sl2 = scale * kLog2e;
  p.scale = scale;
  p.limit_ns = 4000000000ull;
  p.status = device_status_ptr();
  p.n_split = n_split;
  if (n_split > 1) {  // partials after the rows' D: bwd_scratch_bytes counts them
    p.part_stride = (long long)B * N * H * D;
    p.dk_part = dvec + rows;
    p.dv_part = p.dk_part + (size_t)n_split * p.part_stride;
  }
  if ((rc = make_tmap_f32_rows(&tmacc, p.dq_acc, rows, D, 32, Tr::ACC_BOX_ROWS)) != FA_OK)
    return rc;
  if ((rc = check_launch_regs((const void*)kern)) != FA_OK) return rc;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Tr::SMEM_BYTES) !=
      cudaSuccess)
    return launch_status(cudaGetLastError());

  // The pre-pass rewrites every scratch word the pass reads (it zeroes the
  // accumulator), so earlier contents of the scratch never leak in.
  constexpr int kPreRowsPerBlock = 8 * (32 / bwd_pre_lanes(D));
  fa_bwd_pre_kernel<T, D>
      <<<(unsigned)((rows + kPreRowsPerBlock - 1) / kPreRowsPerBlock), 256, 0, stream>>>(
          static_cast<const T*>(o), static_cast<const T*>(dout), lse, lse2, dvec, p.dq_acc, B, H,
          N, Npad, cu, total);
  note_launches(1);
  if ((rc = launch_status(cudaGetLastError())) != FA_OK) return rc;
  cudaEvent_t ev0 = nullptr, ev1 = nullptr;
  if (timed) take_kernel_events(true, &ev0, &ev1);
  if (ev0) cudaEventRecord(ev0, stream);
  p.n_x = (N + Tr::BN - 1) / Tr::BN * n_split * Tr::NHALF;
  const long long blocks = (long long)p.n_x * H * B;
  if (blocks >= (1ll << 31)) return FA_ERR_SHAPE;
  kern<<<(unsigned)blocks, 384, Tr::SMEM_BYTES, stream>>>(tmq, tmk, tmv, tmdo, tmacc, p);
  rc = launch_status(cudaGetLastError());
  if (ev1) cudaEventRecord(ev1, stream);
  note_launches(1);
  if (rc != FA_OK) return rc;
  if (n_split > 1) {
    fa_bwd_dkv_kernel<T, D><<<(unsigned)((p.part_stride / 8 + 255) / 256), 256, 0, stream>>>(
        p.dk_part, p.dv_part, n_split, p.part_stride, static_cast<T*>(dk), static_cast<T*>(dv), H,
        tok_g);
    note_launches(1);
    if ((rc = launch_status(cudaGetLastError())) != FA_OK) return rc;
  }
  const long long acc_elems = (long long)rows * D;
  fa_bwd_dq_kernel<T, D><<<(unsigned)((acc_elems / 8 + 255) / 256), 256, 0, stream>>>(
      p.dq_acc, static_cast<T*>(dq), B, H, N, Npad, scale, tok_g, cu, total);
  note_launches(1);
  return launch_status(cudaGetLastError());
}

template <class Tr>
static size_t bwd_scratch_bytes(int B, int H, int N, int n_split = 1) {
  const size_t rows = (size_t)B * H * ((N + Tr::BM - 1) / Tr::BM) * Tr::BM;
  const size_t parts = n_split > 1 ? 2 * (size_t)n_split * B * N * H * Tr::D : 0;
  return (rows * Tr::D + 2 * rows + parts) * sizeof(float);
}

template <class T, class Tr>
static int run_bwd(void (*kern)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                                const CUtensorMap, const CUtensorMap, const BwdParams),
                   const void* q, const void* k, const void* v, const void* o, const void* dout,
                   const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, float scale,
                   long long tok_in, long long tok_g, cudaStream_t stream, const int* cu,
                   int total, int n_split = 1) {
  void* ws = nullptr;
  int rc = scratch_alloc(&ws, bwd_scratch_bytes<Tr>(B, H, N, n_split), stream);
  if (rc != FA_OK) return rc;
  rc = launch_bwd<T, Tr>(kern, ws, q, k, v, o, dout, lse, dq, dk, dv, B, H, N, scale, tok_in, tok_g,
                         stream, true, cu, total, n_split);
  scratch_free(ws, stream);
  return rc;
}

// Split choice for a fixed-length, non-causal batch (causal key tiles see
// unequal query ranges and varlen sequences unequal lengths: those keep one
// block per key tile).
template <class Tr>
static int bwd_split(int B, int H, int N, unsigned flags, const int* cu, int sm_count) {
  if ((flags & 1u) || cu != nullptr) return 1;
  const long long blocks = (long long)((N + Tr::BN - 1) / Tr::BN) * Tr::NHALF * H * B;
  return choose_bwd_split(blocks, (N + Tr::BM - 1) / Tr::BM, sm_count);
}

int plan_bwd(int B, int H, int N, int d, unsigned flags, int sm_count, int* n_split,
             int* grid_blocks) {
  if (B < 1 || H < 1 || N < 1 || sm_count < 1) return FA_ERR_SHAPE;
  int ns, bn;
  switch (d) {
    case 64:
      ns = bwd_split<BwdTraits64>(B, H, N, flags, nullptr, sm_count);
      bn = BwdTraits64::BN;
      break;
    case 96:
      ns = bwd_split<BwdTq96>(B, H, N, flags, nullptr, sm_count);
      bn = BwdTq96::BN;
      break;
    case 128:
      ns = bwd_split<BwdTq128>(B, H, N, flags, nullptr, sm_count);
      bn = BwdTq128::BN;
      break;
    case 256:  // two blocks per key tile and split, one per half of d
      ns = bwd_split<BwdTq256>(B, H, N, flags, nullptr, sm_count);
      bn = BwdTq256::BN;
      break;
    default:
      return FA_ERR_HEADDIM;
  }
  *n_split = ns;
  *grid_blocks = (int)((long long)((N + bn - 1) / bn) * ns * (d == 256 ? 2 : 1) * H * B);
  return FA_OK;
}

template <class T>
int bwd_launch(const void* q, const void* k, const void* v, const void* o, const void* dout,
               const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
               float scale, unsigned flags, long long tok_in, long long tok_g,
               cudaStream_t stream, const int* cu, int total) {
  DeviceInfo dev;
  int rc = current_device(&dev);
  if (rc != FA_OK) return rc;
  switch (d) {
    case 64: {
      const int ns = bwd_split<BwdTraits64>(B, H, N, flags, cu, dev.sm_count);
      auto kern = (flags & 1u) ? (cu ? fa_bwd_kernel<T, BwdTraits64, true, true>
                                     : fa_bwd_kernel<T, BwdTraits64, true, false>)
                               : (cu ? fa_bwd_kernel<T, BwdTraits64, false, true>
                                     : ns > 1 ? fa_bwd_kernel<T, BwdTraits64, false, false, true>
                                              : fa_bwd_kernel<T, BwdTraits64, false, false>);
      return run_bwd<T, BwdTraits64>(kern, q, k, v, o, dout, lse, dq, dk, dv, B, H, N, scale,
                                     tok_in, tok_g, stream, cu, total, ns);
    }
    case 96: {
      const int ns = bwd_split<BwdTq96>(B, H, N, flags, cu, dev.sm_count);
      auto kern = (flags & 1u) ? (cu ? fa_bwd_tq_kernel<T, BwdTq96, true, true>
                                     : fa_bwd_tq_kernel<T, BwdTq96, true, false>)
                               : (cu ? fa_bwd_tq_kernel<T, BwdTq96, false, true>
                                     : ns > 1 ? fa_bwd_tq_kernel<T, BwdTq96, false, false, true>
                                              : fa_bwd_tq_kernel<T, BwdTq96, false, false>);
      return run_bwd<T, BwdTq96>(kern, q, k, v, o, dout, lse, dq, dk, dv, B, H, N, scale, tok_in,
                                 tok_g, stream, cu, total, ns);
    }
    case 128: {
      const int ns = bwd_split<BwdTq128>(B, H, N, flags, cu, dev.sm_count);
      auto kern = (flags & 1u) ? (cu ? fa_bwd_tq_kernel<T, BwdTq128, true, true>
                                     : fa_bwd_tq_kernel<T, BwdTq128, true, false>)
                               : (cu ? fa_bwd_tq_kernel<T, BwdTq128, false, true>
                                     : ns > 1 ? fa_bwd_tq_kernel<T, BwdTq128, false, false, true>
                                              : fa_bwd_tq_kernel<T, BwdTq128, false, false>);
      return run_bwd<T, BwdTq128>(kern, q, k, v, o, dout, lse, dq, dk, dv, B, H, N, scale, tok_in,
                                  tok_g, stream, cu, total, ns);
    }
    case 256: {
      const int ns = bwd_split<BwdTq256>(B, H, N, flags, cu, dev.sm_count);
      auto kern = (flags & 1u) ? (cu ? fa_bwd_tq_kernel<T, BwdTq256, true, true>
                                     : fa_bwd_tq_kernel<T, BwdTq256, true, false>)
                               : (cu ? fa_bwd_tq_kernel<T, BwdTq256, false, true>
                                     : ns > 1 ? fa_bwd_tq_kernel<T, BwdTq256, false, false, true>
                                              : fa_bwd_tq_kernel<T, BwdTq256, false, false>);
      return run_bwd<T, BwdTq256>(kern, q, k, v, o, dout, lse, dq, dk, dv, B, H, N, scale, tok_in,
                                  tok_g, stream, cu, total, ns);
    }
    default:
      return FA_ERR_HEADDIM;
  }
}

template int bwd_launch<__nv_bfloat16>(const void*, const void*, const void*, const void*,
                                       const void*, const float*, void*, void*, void*, int, int,
                                       int, int, float, unsigned, long long, long long,
                                       cudaStream_t, const int*, int);
template int bwd_launch<__half>(const void*, const void*, const void*, const void*, const void*,
                                const float*, void*, void*, void*, int, int, int, int, float,
                                unsigned, long long, long long, cudaStream_t, const int*, int);

// ------------------------------------------------------------------------
// Fixed-scratch backward (fa_bwd_noalloc).  Same kernels as run_bwd, but the
// scratch (dQ accumulator, minus the base-2 LSE, D) lives in a file-scope device array
// instead of a stream-ordered allocation, for callers that cannot allocate.
// Host code cannot pass g_fixed_scratch itself to a kernel (in host code the
// name denotes a host-side stand-in); its device address is looked up with
// cudaGetSymbolAddress, with the device current, once per CUDA context (the
// address belongs to the context: a reset device or another context gets its
// own lookup).
static constexpr size_t kFixedScratchBytes = (size_t)64 << 20;
static __device__ __align__(256) unsigned char g_fixed_scratch[kFixedScratchBytes];

static int fixed_scratch_address(void** out) { return symbol_address(&g_fixed_scratch, out); }

template <class T, class Tr>
static int run_bwd_fixed_scratch(const void* q, const void* k, const void* v, const void* o,
                                 const void* dout, const float* lse, void* dq, void* dk, void* dv,
                                 int B, int H, int N, float scale, cudaStream_t stream) {
  if (bwd_scratch_bytes<Tr>(B, H, N) > kFixedScratchBytes) return FA_ERR_SCRATCH;
  void* ws = nullptr;
  int rc = fixed_scratch_address(&ws);
  if (rc != FA_OK) return rc;
  return launch_bwd<T, Tr>(fa_bwd_kernel<T, Tr, false, false>, ws, q, k, v, o, dout, lse, dq, dk, dv, B,
                           H, N, scale, (long long)H * Tr::D, (long long)H * Tr::D, stream, false,
                           nullptr, N);
}

}  // namespace fa

extern "C" __attribute__((visibility("default"))) int fa_bwd_noalloc(
    const void* q, const void* k, const void* v, const void* o, const void* dout,
    const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale,
    cudaStream_t stream) {
  int rc = fa::check_bwd_args(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale);
  if (rc != FA_OK) return rc;
  fa::DeviceInfo dev;
  if ((rc = fa::current_device(&dev)) != FA_OK) return rc;
  if (d != 64) return FA_ERR_HEADDIM;
  return fa::run_bwd_fixed_scratch<__nv_bfloat16, fa::BwdTraits64>(q, k, v, o, dout, lse, dq, dk,
                                                                   dv, B, H, N, scale, stream);
}
