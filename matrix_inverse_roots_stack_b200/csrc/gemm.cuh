// Batched square GEMM on split-fp16 operands with a fused epilogue.
//
// Every product on the hot path of the batched block-Shampoo step is a
// B x B x B product of two matrices from stacked (N, B, B) tensors (the DASH
// explainer's "Building blocks": stack blocks into (N, B, B), run batched
// products).  Operands are held as two fp16 planes (hi, lo * 2^11); for every
// K=16 step the kernel computes hi*lo + lo*hi and then hi*hi + 2^-11 * that in
// fp32 tensor memory (tcgen05, kind::f16) and adds the step's product into
// fp32 registers, which gives about fp32 accuracy at the fp16 tensor-core rate.
//
// Problem p computes
//     out_p = s_p * (alpha * a_p * A_p op(B_p) + beta * Cin_p + gamma * I)
// (s_p, a_p optional per-problem scalars) where A_p is a row-major matrix of
// the A stack (read K-major) and op(B_p)
// is B_p (b_mn = 1: the stored row-major B is read MN-major, giving A B) or
// B_p^T (b_mn = 0: read K-major, giving A B^T).  A launch carries one or two
// "ops" (groups of problems) with their own operand stacks and epilogues.
// With sym = 1 only upper-triangle tiles are computed and each off-diagonal
// tile is also written mirrored (for results that are symmetric by
// construction).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace dash {

// One Shampoo block in parameter layout (used by the preconditioner epilogue
// that scatters U into the parameter-shaped buffer).
struct BlockDesc {
  long long off;  // element offset of the owning parameter in the flat buffer
  int pitch;      // row length (columns) of the owning parameter
  int r0, c0;     // block origin inside the parameter
  int br, bc;     // block extent (<= B)
  int param;      // owning parameter index
};

// Matrix index of problem p: base + stride * (p % mod); mod <= 0 means no
// modulo and stride 0 means 1, so a zero-initialised Idx maps p to p.
struct Idx {
  int base, mod, stride;
};

struct GemmOp {
  int nprob;
  Idx a, b;                  // operand matrices in this op's A / B stacks
  int b_mn;                  // 1: out = A B ; 0: out = A B^T
  float alpha, beta, gamma;
  const float* scale;        // per-problem multiplier s_p (nullptr: 1)
  Idx scale_i;
  const float* acc_scale;    // per-problem multiplier of alpha alone (nullptr: 1)
  Idx accs_i;
  const __half* cin_split;   // split Cin stack (nullptr: none)
  Idx cin_i;
  const float* cin_f32;      // fp32 Cin stack (nullptr: none)
  Idx cinf_i;
  __half* out_split;         // split output (+ mirror if sym)
  Idx out_i;
  int split_norm;            // 1: the split output is out_p * 2^-e with 2^(e-1) <= s_p < 2^e
  float* out_f32;            // fp32 output (+ mirror if sym)
  Idx outf_i;
  const BlockDesc* blocks;   // non-null: scatter out_p into u_out (parameter layout); with
                             // 128 x 256 tiles such an op may have no Cin
  float* u_out;
  float* unorm;              // per-problem sum of squares of the scattered out_p
};

struct GemmArgs {
  int B;      // matrix size; multiple of 128
  int sym;    // 1: symmetric outputs (upper-triangle tiles + mirrored writes)
  int nops;   // 1 or 2
  int single_pass;  // 1: fp16 operands (hi planes only), one MMA per product, fp32 accumulation
  int skip_loads;  // test hook: the producer issues no loads (bounded waits expire)
  GemmOp op[2];
  unsigned* status;  // device status word (non-finite / timeout bits)
};

// Operand stacks of one op: split stacks of B x B matrices, layout
// [matrix][plane][row][col] fp16.
struct OpBuffers {
  const __half* a;
  int a_nmat;
  const __half* b;
  int b_nmat;
};

// Launch one batched GEMM (args.nops ops).  Returns cudaSuccess or the
// launch / encode error.
cudaError_t launch_gemm_split(const OpBuffers* bufs, const GemmArgs& args, cudaStream_t stream);

// Newton-DB iterations on a stack of n factors of 128 held in shared memory
// (one CTA per factor), in place on the split stacks Y and Zhat (layout as
// OpBuffers), in this order: if first, Y <- Y + Y D with D read from the
// split stack D; `iters` times D = alpha_d Zhat Y + I/2, Y <- Y + Y D,
// Zhat <- Zhat + D Zhat; if last_y, once more D = alpha_d Zhat Y + I/2,
// Y <- Y + Y D.  Zhat is written back only when the launch ends with a full
// iteration (with last_y, or first alone, the Zhat stack keeps what it held
// before the launch).  The products' arithmetic is
// that of launch_gemm_split.  Returns cudaErrorNotSupported unless B == 128
// and first, last_y are 0 or 1.
cudaError_t launch_ndb_fused(__half* Y, __half* Zhat, const __half* D, int n, int B, float alpha_d, int first,
                             int iters, int last_y, unsigned* status, cudaStream_t stream);

// Arm a one-shot test fault: the next launch of a tensor-core product kernel
// (the GEMM, or Newton-DB on resident factors) withholds its operand loads,
// so its waits run into their time limit and it reports a timeout.
void arm_load_fault();
// Consume the armed fault: true once after arm_load_fault.
bool take_load_fault();

}  // namespace dash
