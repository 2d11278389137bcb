// fa_host.h -- host-side pieces shared by the forward and backward launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa_b200.h"  // include/ is on the include path

namespace fa {

// Properties of the current device that the launchers need.
struct DeviceInfo {
  int device;
  int sm_count;
  int max_smem_optin;
};

// FA_OK, or FA_ERR_DEVICE when the current device is not compute capability
// 10.0, or FA_ERR_LAUNCH when the runtime cannot be queried.
int current_device(DeviceInfo* info);

// FA_OK when e is cudaSuccess; otherwise records e (fa_last_cuda_error) and
// returns FA_ERR_LAUNCH.
int launch_status(cudaError_t e);

// FA_OK when the kernel was compiled with the register count its warpgroup
// register split assumes (kLaunchRegs a thread at 384 threads).
int check_launch_regs(const void* kernel);

// Counts kernel launches (fa_kernel_launches).
void note_launches(unsigned n);

// Takes (and disarms) the event pair armed for the next forward (bwd=false)
// or backward (bwd=true) main kernel; both are null when none is armed.
void take_kernel_events(bool bwd, cudaEvent_t* start, cudaEvent_t* stop);

// Stream-ordered scratch from this library's own memory pool on the current
// device (created on first use).  The pool keeps up to kScratchRetainBytes of
// freed scratch mapped across synchronisations, so repeated calls do not map
// and unmap device memory each time (the default pool releases everything at
// every synchronisation).  FA_OK or FA_ERR_NOMEM.
constexpr unsigned long long kScratchRetainBytes = 1ull << 30;
int scratch_alloc(void** ptr, size_t bytes, cudaStream_t stream);
void scratch_free(void* ptr, cudaStream_t stream);

// Device address of this library's status word in the current context.
unsigned long long* device_status_ptr();

// Unique ID of the CUDA context current on the calling thread (cuCtxGetId);
// false when none is current or the driver cannot report it.
bool current_context_id(unsigned long long* id);

// Device address of a __device__ variable of this library in the current
// context: looked up with cudaGetSymbolAddress once per context (keyed by the
// context's unique ID, so a reset device or another context never gets a
// stale address).  FA_OK or FA_ERR_LAUNCH.
int symbol_address(const void* symbol, void** out);

// Number of scratch_alloc calls since the library was loaded.
unsigned long long scratch_allocs();

// Tensor map over a contiguous [B, N, H, d] tensor for TMA tile loads of
// `box_rows` tokens x 128 bytes of one head (64 16-bit or 128 8-bit elements,
// 128-byte swizzle).  fmt: 0 fp16, 1 bf16, 2 one-byte elements (E4M3).
// Rows past N, and elements past d, are filled with zeros by the hardware.
// tok_stride: elements from one token to the next (H*d for [B,N,H,d]; 3*H*d
// for one of Q, K, V inside a packed [B,N,3,H,d] tensor).
int make_tmap_bnhd(CUtensorMap* map, const void* base, int fmt, int B, int N, int H, int d,
                   int box_rows, long long tok_stride);

// Tensor map over a contiguous [rows, cols] fp32 matrix for TMA tiles of
// box_rows x box_cols (box_cols * 4 = 128 bytes, 128-byte swizzle).
int make_tmap_f32_rows(CUtensorMap* map, const void* base, size_t rows, int cols, int box_cols,
                       int box_rows);

// The backward entry points' argument checks (FA_OK or an FA_ERR_* code).
int check_bwd_args(const void* q, const void* k, const void* v, const void* o, const void* dout,
                   const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                   float scale);

// Flags of the *_ex entry points that the library knows (FA_FLAG_* bits).
constexpr unsigned kKnownFlags = 1u;  // FA_FLAG_CAUSAL
// Internal plan_fwd flag (never accepted from callers): a varlen batch, whose
// units are neither split nor cut.
constexpr unsigned kPlanVarlen = 0x100u;

// Work decomposition of one forward call (fa_fwd.cu).  A unit is unit_rows
// query rows of one (batch, head), possibly limited to one share of the K/V
// tiles (split mode); blocks walk units round-robin, or in the balanced
// schedule each block takes a contiguous range of (unit, K/V tile) steps.
struct FwdSchedule {
  int B, H, N, d;     // varlen: B sequences of at most N (max_seqlen) tokens
  int causal;         // 1: row i sees keys j <= i (units ordered longest first)
  const int* cu;      // varlen: device [B+1] sequence starts in the packed token axis; else null
  int total;          // tokens a batch entry holds in memory: N, or all B sequences' (varlen)
  int pair;           // 1: fa_fwd_pp_kernel (two 128-row Q tiles a unit), 0: fa_fwd_kernel
  int unit_rows;      // 256 (pair) or 128
  int bn;             // K/V tile rows
  int n_qt;           // units per (b, h) along the queries
  int n_kvt;          // K/V tiles per head
  int n_split;        // K/V shares per unit (> 1: partials merged by fa_combine_kernel)
  int kvt_per_split;
  int n_units;        // B * H * n_qt * n_split
  int grid;           // blocks launched (at most one per SM)
  int n_iter;         // balanced: n_units * n_kvt steps (0 = round-robin schedule)
  int iter_per, iter_rem;  // balanced: block c takes iter_per (+1 if c < iter_rem) steps
};

// Fills *s for a forward call on a device with sm_count SMs (pure host logic).
// FA_OK, or FA_ERR_SHAPE / FA_ERR_HEADDIM for shapes the forward rejects.
int plan_fwd(int B, int H, int N, int d, unsigned flags, int sm_count, FwdSchedule* s);

// Scratch bytes the forward needs for schedule s (split partials, or the
// balanced schedule's partial-row slots and flags).
size_t fwd_scratch_bytes(const FwdSchedule& s);

// The pieces block `blk` of schedule s processes, in order: for each, the
// unit index, first and end K/V tile, store kind (0 whole, 1 partial,
// 2 merge), first peer block and peer count, written as 6 ints to out.
// Returns the number of pieces (writes at most max_pieces).
int fwd_block_pieces(const FwdSchedule& s, int blk, int* out, int max_pieces);

// Backward decomposition for fixed-length batches: blocks per key tile
// (n_split; > 1 splits each key tile's query range) and blocks in the grid.
int plan_bwd(int B, int H, int N, int d, unsigned flags, int sm_count, int* n_split,
             int* grid_blocks);

// Launchers (argument validation is done by the callers in fa_api.cu).
// tok_in: token stride of q, k, v (elements); tok_g: of dq, dk, dv.  o, lse,
// dout are always contiguous [B,N,H,d] / [B,H,N].
// cu (varlen): device [B+1] sequence starts, N = max_seqlen, total tokens; else null.
// T = __nv_fp8_e4m3: q, k, v are E4M3 (d = 128 only), o is bf16, and o_scale
// multiplies O as it is stored (the V descale; the Q, K descales are in scale).
template <class T>
int fwd_launch(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int N, int d, float scale, unsigned flags, long long tok_in, cudaStream_t stream,
               const int* cu = nullptr, int total = 0, float o_scale = 1.f);
template <class T>
int bwd_launch(const void* q, const void* k, const void* v, const void* o, const void* dout,
               const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
               float scale, unsigned flags, long long tok_in, long long tok_g,
               cudaStream_t stream, const int* cu = nullptr, int total = 0);

}  // namespace fa
