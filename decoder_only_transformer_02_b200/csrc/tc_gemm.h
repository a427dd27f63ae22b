// Host interface of the tcgen05 bf16 GEMM (internal to the library).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stddef.h>

namespace tcg {

enum Epi : int {
  EPI_BF16 = 0,         // out(bf16)  = acc (+ bias)
  EPI_F32 = 1,          // out(fp32)  = acc (+ bias)
  EPI_RESID_F32 = 2,    // out(fp32)  = resid + acc (+ bias)
  EPI_GELU = 3,         // out(bf16)  = u = acc + bias ; out2(bf16) = gelu_tanh(u)
  EPI_DGELU = 4,        // out(bf16)  = acc * gelu_tanh'(aux)
  EPI_ACCUM_F32 = 5,    // out(fp32) += acc   (split-K through `workspace` when given)
  EPI_PARTIAL_F32 = 6,  // internal: split-K partial tiles
  EPI_CE_STATS = 7,     // internal: out(bf16) = acc, plus per-(row, half tile) softmax statistics of the
                        // stored (bf16-rounded) values into ce_part
  EPI_ROWDOT = 8,       // out(bf16) = acc, plus per (row, 64 columns) the dot product of the stored
                        // values with aux (bf16, same layout), into rd_out (see GemmArgs)
};

// Logical problem: D[M,N] = sum_k A[m,k] B[n,k].
//  a_mn = 0: A stored [M][lda] (k contiguous); a_mn = 1: A stored [K][lda] (m contiguous)
//  b_mn = 0: B stored [N][ldb] (k contiguous); b_mn = 1: B stored [K][ldb] (n contiguous)
// out / resid / aux are [M][ldc].  lda, ldb, ldc multiples of 8; A, B, out 16-byte aligned.
struct GemmArgs {
  const __nv_bfloat16* A = nullptr;
  long lda = 0;
  int a_mn = 0;
  const __nv_bfloat16* B = nullptr;
  long ldb = 0;
  int b_mn = 0;
  int M = 0, N = 0, K = 0;
  int epi = EPI_BF16;
  const float* bias = nullptr;
  const float* resid = nullptr;
  void* out = nullptr;
  __nv_bfloat16* out2 = nullptr;
  const __nv_bfloat16* aux = nullptr;
  long ldc = 0;
  float* workspace = nullptr;   // split-K scratch for EPI_ACCUM_F32 (may be null)
  size_t workspace_bytes = 0;
  int bn = 0;                   // 0: automatic (256 unless N <= 128), or 128 / 256
  float* ce_part = nullptr;     // EPI_CE_STATS: [M][ce_halves(N)][3] (max, sum of exp(z - max), argmax bits)
  // EPI_ACCUM_F32 over K splits into persistent per-split accumulators (no
  // reduction here): split s adds its share of the sum into
  // slots[s][M][N] (ldc == N); at most slot_splits splits.  The caller folds
  // the slots into the final sum later, in split order.  out is unused.
  float* slots = nullptr;
  int slot_splits = 0;
  // EPI_ROWDOT (N = 64 H, M = B T, T % 128 == 0): for row m = b T + q and
  // column group h, rd_out[((b H + h) nqb + q / 128) 256 + 128 + q % 128] =
  // sum of out[m][64h + c] * aux[m][64h + c] over c, and the entry 128 below
  // it = rd_lse[(b H + h) T + q] * log2(e) (nqb = T / 128): the rows of
  // lse*log2(e) and D = rowsum(dO * O) of the attention backward.
  float* rd_out = nullptr;
  const float* rd_lse = nullptr;
  int rd_T = 0;
};

// Number of softmax-statistics partials per row that EPI_CE_STATS writes.
inline int ce_halves(int N) { return 2 * ((N + 255) / 256); }

struct Params {
  int M, N, K;
  int a_mn, b_mn;
  int num_m, num_n, splits, kb_total, kb_per_split;
  int total_tiles;
  int epi;
  const float* bias;
  const float* resid;
  void* out;
  __nv_bfloat16* out2;
  const __nv_bfloat16* aux;
  long ldc;
  float* partial;
  int vec32;  // 1: every 32-column chunk is 32-byte aligned (vector epilogue)
  float* ce_part;
  int ce_nh;
  long split_stride;  // EPI_ACCUM_F32: elements between the accumulators of consecutive splits (0: one)
  float* rd_out;      // EPI_ROWDOT
  const float* rd_lse;
  int rd_T;
};

// Returns 0 on success, -1 bad arguments, -2 tensor-map encode failure, -3 launch failure.
int gemm(const GemmArgs& g, cudaStream_t stream);
// Bytes of split-K scratch that an EPI_ACCUM_F32 call of this shape would use.
size_t splitk_workspace_bytes(int M, int N, int K, int bn);
// K splits that an EPI_ACCUM_F32 call of this shape uses with per-split
// accumulators (1: none needed).
int accum_slot_splits(int M, int N, int K);
int choose_splits(int tiles, int kb_total, int units);

}  // namespace tcg
