/*
 * tp.h -- C ABI of libtp: the Megatron-style tensor-parallel MLP over t virtual shards held in one
 * GPU's memory, ring-order collectives over those shards, and the four sharded-matmul cases.
 *
 * Sources (pages cited by title and section):
 *   [TPSP] "张量并行与序列并行" (hs-black.github.io, scaling-tensor-parallel)
 *   [CH06] "Scaling Book 入门第 6 章：分片矩阵乘法 — 分布式计算的核心" (r00kie-liu.github.io, scaling-infra-ch06)
 *   [CH05] "Scaling Book 入门第 5 章：Sharded Matrices 上篇 — 集合通信原语" (r00kie-liu.github.io, scaling-infra-ch05)
 *   [PFY]  pufanyi.com "ml-revisit-infra", section "Tensor Parallel"
 *
 * Conventions shared by every entry point
 *   - All matrices are row-major. Weights are [in, out] (a linear layer is Y = X W, W of shape [k, n]).
 *   - "bf16" buffers are uint16_t bit patterns of bfloat16; "f32" buffers are IEEE binary32.
 *   - Every data pointer is a DEVICE pointer, except arrays of shard pointers ("const T* const* p"),
 *     which are HOST arrays of t device pointers. t (the TP degree) is 1..TP_MAX_SHARDS.
 *   - The caller allocates and frees every buffer. The library allocates no device memory; it keeps
 *     one device status word and the code it needs.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Every call is asynchronous on it.
 *     Argument errors are returned before anything is launched; a failed launch returns TP_ECUDA.
 *     tp_last_error() gives a one-line message for the last failure on the calling host thread.
 *   - Device pointers must be 16-byte aligned and row strides a multiple of 16 bytes (8 bf16 or 4 f32
 *     elements) where a function says "aligned"; otherwise TP_EALIGN. A dimension that t must divide
 *     and does not gives TP_EDIVIS (nothing is padded).
 *   - Buffers must not overlap unless a function states otherwise.
 *   - Empty inputs: a call whose token count / row count (or, for a GEMM or collective, any output
 *     dimension) is zero returns TP_OK: t and the sizes are still checked, but no data pointer is
 *     read and nothing is launched. A negative size, and an empty contraction (K, h or F of zero,
 *     which would leave the output undefined rather than empty), give TP_EINVAL.
 *   - Device-side waits are bounded; a wait that runs out records TP_ETIMEOUT in the device status
 *     word (read it with tp_device_status) and the kernel returns without finishing its work.
 */
#ifndef TP_H_
#define TP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TP_MAX_SHARDS 16

typedef enum {
  TP_OK = 0,
  TP_EINVAL = 1,        /* null pointer, negative size, empty contraction, bad enum value */
  TP_ESHAPE = 2,        /* sizes inconsistent with each other */
  TP_EDIVIS = 3,        /* t does not divide a dimension it must split */
  TP_EALIGN = 4,        /* pointer or row stride not 16-byte aligned */
  TP_ECUDA = 5,         /* a CUDA runtime/driver call failed */
  TP_ETIMEOUT = 6,      /* a bounded device-side wait ran out (reported by tp_device_status) */
  TP_EUNSUPPORTED = 7,  /* valid request the library does not implement */
  TP_ENOSPACE = 8       /* a workspace is too small: the caller's, or the built-in array of
                           tp_mlp_fwd_noalloc */
} tp_status;

/* Element types. TP_BF16_RING is bf16 storage for the ring collectives only (tp_reduce_scatter,
 * tp_all_reduce, tp_all_gather): the running partial is rounded to bf16 after every add, as a ring
 * whose links carry bf16 does. The default bf16 mode (TP_BF16) keeps the partial in binary32 and
 * rounds once at the end. */
typedef enum { TP_F32 = 0, TP_BF16 = 1, TP_BF16_RING = 2 } tp_dtype;

/* Activation applied in the column-parallel GEMM's epilogue. It is element-wise, so each shard
 * applies it to its own columns ([TPSP] §MLP：先列后行，只通信一次). GELU is the exact erf form.
 * SWIGLU reads a fused [gate | up] operand and writes SiLU(gate) * up (one output per pair). */
typedef enum { TP_ACT_NONE = 0, TP_ACT_GELU = 1, TP_ACT_GELU_TANH = 2, TP_ACT_SWIGLU = 3 } tp_act;

/* What tp_mlp_fwd returns after the row-parallel GEMM. */
typedef enum {
  TP_OUT_PARTIALS = 0,  /* the t unreduced partial sums {U} ([TPSP] §矩阵乘法的两种切法, row-parallel) */
  TP_OUT_RS = 1,        /* ReduceScatter along tokens: shard r gets rows [rN/t,(r+1)N/t) of sum U */
  TP_OUT_AR = 2,        /* AllReduce in one pass: every shard gets sum U */
  TP_OUT_RS_AG = 3      /* AllReduce as ReduceScatter along tokens then AllGather (bit-identical to AR) */
} tp_reduce;

/* Strategies of tp_sharded_matmul ([CH06] §6.2, four cases of C[B,F] = X[B,D] W[D,F]). */
typedef enum {
  TP_CASE1_LOCAL = 0,
  TP_CASE2_ALLGATHER = 0, TP_CASE2_ALLREDUCE = 1,
  TP_CASE3_ALLREDUCE = 0, TP_CASE3_RS_B = 1, TP_CASE3_RS_F = 2,
  TP_CASE4_GATHER_X = 0, TP_CASE4_GATHER_W = 1
} tp_strategy;

/* ------------------------------------------------------------------------------------------------
 * Status and diagnostics
 * ------------------------------------------------------------------------------------------------ */
const char* tp_status_str(tp_status s);
/* One-line description of the last failure returned on the calling host thread ("" if none). */
const char* tp_last_error(void);
/* Synchronises the current device, then returns TP_ETIMEOUT if any kernel recorded a wait that ran
 * out since the last clear (TP_OK otherwise, TP_ECUDA if synchronising failed). clear != 0 resets
 * the word. *where (optional, host) receives the code of the wait that ran out. */
tp_status tp_device_status(int clear, uint32_t* where);
/* Budget, in SM clock cycles, of every bounded device-side wait issued by later launches
 * (0 restores the default of about two seconds). */
void tp_set_wait_budget(uint64_t cycles);
/* Launches one kernel that waits, bounded by `budget_cycles`, on a device flag that nothing sets,
 * so that the wait runs out and records TP_ETIMEOUT in the status word (failure-path self test). */
tp_status tp_selftest_wait_timeout(uint64_t budget_cycles, void* stream);
/* Number of streaming multiprocessors of the current device (grid sizing), or -1 on error. */
int tp_num_sms(void);

/* ------------------------------------------------------------------------------------------------
 * Weight shard layouts (bit copies). Outputs are stacked: shard r starts at out + r * (shard size).
 * All aligned (inputs' row strides ld_* in elements). One-off conversions, not on the hot loop.
 * ------------------------------------------------------------------------------------------------ */
/* Column-parallel split of W[K, N] (row stride ld): out[r] = W[:, rN/t:(r+1)N/t], shape [K, N/t].
 * ([TPSP] §矩阵乘法的两种切法, first identity; [CH06] §6.7 Column Parallel Linear.) */
tp_status tp_shard_cols(const uint16_t* w, int64_t ld, int64_t K, int64_t N, int t, uint16_t* out, void* stream);
/* Row-parallel split of W[K, N] (row stride ld): out[r] = W[rK/t:(r+1)K/t, :], shape [K/t, N].
 * ([TPSP] §矩阵乘法的两种切法, second identity; [CH06] §6.7 Row Parallel Linear.) */
tp_status tp_shard_rows(const uint16_t* w, int64_t ld, int64_t K, int64_t N, int t, uint16_t* out, void* stream);
/* Fused SwiGLU gate|up layout of W_gate[h, F] and W_up[h, F] (row strides ld_g, ld_u):
 * out[r] = [W_gate[:, F-range r] | W_up[:, F-range r]], shape [h, 2F/t] -- a rank's gate and up
 * columns cover the same F indices ([TPSP] §MLP, SwiGLU paragraph). Gate first, then up. */
tp_status tp_shard_gate_up(const uint16_t* w_gate, int64_t ld_g, const uint16_t* w_up, int64_t ld_u,
                           int64_t h, int64_t F, int t, uint16_t* out, void* stream);
/* Rank-grouped fused QKV layout ([TPSP] §注意力：按头切 fused-QKV bullet, §GQA). W_q[h, n_h*d_h],
 * W_k/W_v[h, n_kv*d_h] (row strides ld_q, ld_k, ld_v). out[r] = [Q heads of rank r | its K heads | its
 * V heads], heads ascending, d_h columns each; shape [h, (n_h/t + 2*kv)*d_h] with kv = n_kv/t when
 * t <= n_kv, else kv = 1 and rank r takes KV head floor(r*n_kv/t) (replication for n_kv < t <= n_h).
 * t must divide n_h, n_kv must divide n_h, and t | n_kv or n_kv | t (TP_EDIVIS otherwise). */
tp_status tp_shard_qkv(const uint16_t* w_q, int64_t ld_q, const uint16_t* w_k, int64_t ld_k,
                       const uint16_t* w_v, int64_t ld_v, int64_t h, int n_h, int n_kv, int d_h, int t,
                       uint16_t* out, void* stream);

/* ------------------------------------------------------------------------------------------------
 * Ring collectives over t shard buffers resident in this GPU's memory ([CH05] §5.2 环形算法, §5.3;
 * [CH06] §6.4). `in` and `out` are host arrays of t device pointers; buffers are contiguous
 * [rows, cols] matrices of `dtype`.
 *
 * Summation order (the pages fix the ring, device i passing to i+1 and accumulating at every step,
 * and that device r ends with chunk r; the order of the adds follows from that): chunk c is
 * (((U[c+1] + U[c+2]) + U[c+3]) + ... ) + U[c], indices mod t, one binary32 add at a time. bf16 inputs
 * are widened to binary32, summed in that order and rounded once to bf16 (nearest-even). With
 * TP_BF16_RING (optional, NCCL-like) every add is followed by a rounding to bf16 instead: the partial
 * a device passes on ([CH05] §5.2, §5.3) is held in the payload's type.
 * Chunk r is the row block [r*rows/t, (r+1)*rows/t) (axis 0) or column block (axis 1).
 * Results are bit-exact and independent of launch shape; no atomics are used.
 * ------------------------------------------------------------------------------------------------ */
/* ReduceScatter: in[s] is [rows, cols]; out[r] receives chunk r of the sum: [rows/t, cols] (axis 0)
 * or [rows, cols/t] (axis 1). */
tp_status tp_reduce_scatter(const void* const* in, void* const* out, int64_t rows, int64_t cols, int axis,
                            tp_dtype dtype, int t, void* stream);
/* AllGather: in[r] is shard r of the gathered [rows, cols] matrix ([rows/t, cols] for axis 0,
 * [rows, cols/t] for axis 1); every out[s] receives the whole [rows, cols] in shard order. In-place is
 * allowed for axis 0 when in[r] == out[r] + r*(rows/t)*cols (each shard's piece already in place). */
tp_status tp_all_gather(const void* const* in, void* const* out, int64_t rows, int64_t cols, int axis,
                        tp_dtype dtype, int t, void* stream);
/* AllReduce (= ReduceScatter + AllGather, done in one pass): every out[s] receives the ring-ordered
 * sum of the t in[] buffers; all replicas are bit-identical. in[s] == out[s] (in place) is allowed. */
tp_status tp_all_reduce(const void* const* in, void* const* out, int64_t rows, int64_t cols,
                        tp_dtype dtype, int t, void* stream);

/* AllToAll ([CH05] §5.3 AllToAll; [CH06] §6.4): every in[i] is a [rows, cols] buffer, split into t
 * pieces along split_axis; out[j] receives piece j of every shard, concatenated along concat_axis in
 * shard order. Output shape: [t*rows, cols/t] (split 1, concat 0: moves the sharding from rows to
 * columns, A[I_X, J] -> A[I, J_X]); [rows/t, t*cols] (split 0, concat 1); [rows, cols] otherwise.
 * A bit copy: reads t*M, writes t*M. Buffers must not overlap. */
tp_status tp_all_to_all(const void* const* in, void* const* out, int64_t rows, int64_t cols, int split_axis,
                        int concat_axis, tp_dtype dtype, int t, void* stream);

/* ------------------------------------------------------------------------------------------------
 * GEMMs on the tensor cores (bf16 inputs, fp32 accumulation)
 * ------------------------------------------------------------------------------------------------ */
/* Grouped GEMM: for g < groups, c[g] = act(a[g] . b[g]) with a[g] [M, K] bf16, b[g] [K, Nb] bf16
 * (Nb = N, or 2N for TP_ACT_SWIGLU where b[g] = [gate | up]) and c[g] [M, N] of c_dtype
 * (TP_ACT_NONE may write f32 or bf16; the activations write bf16). a[] entries may repeat (a shared
 * input). Aligned; K and N must be multiples of 8. groups <= TP_MAX_SHARDS. */
tp_status tp_grouped_gemm(int groups, const uint16_t* const* a, const uint16_t* const* b, void* const* c,
                          int64_t M, int64_t N, int64_t K, tp_act act, tp_dtype c_dtype, void* stream);
/* Grouped GEMM with transposed operand storage (no activation): c[g] = op(a[g]) . op(b[g]), where
 * op(a) = a [M, K] (trans_a = 0) or a holds A^T as [K, M] (trans_a = 1), and op(b) = b [K, N]
 * (trans_b = 0) or b holds B^T as [N, K] (trans_b = 1). Row strides are the stored row lengths.
 * Used by the backward pass for X^T dH, Z^T dY and dY W^T. M, N and K multiples of 8, aligned. */
tp_status tp_grouped_gemm_t(int groups, const uint16_t* const* a, int trans_a, const uint16_t* const* b, int trans_b,
                            void* const* c, int64_t M, int64_t N, int64_t K, tp_dtype c_dtype, void* stream);
/* Column-parallel linear ([TPSP] §矩阵乘法的两种切法; [CH06] §6.7): y[r] = act(x . w[r]) for every
 * shard r, from the full x [N, k] (shared by all shards) and the stacked shards w [t][k][n/t]
 * ([t][k][2n/t] = [gate_r | up_r] for SWIGLU, as written by tp_shard_gate_up). y is stacked
 * [t][N][n/t] bf16. No communication. */
tp_status tp_column_linear(const uint16_t* x, int64_t N, int64_t k, int64_t n, int t, tp_act act,
                           const uint16_t* w, uint16_t* y, void* stream);
/* Row-parallel linear: partials[r] = x[r] . w[r], fp32 [N, n], from stacked x [t][N][k/t] and
 * w [t][k/t][n]. The true output is sum_r partials[r] (a following AllReduce or ReduceScatter). */
tp_status tp_row_linear(const uint16_t* x, int64_t N, int64_t k, int64_t n, int t, const uint16_t* w,
                        float* const* partials, void* stream);

/* Row-parallel linear fused with its collective: the one-GPU form of collective matmul ([CH06] §6.6;
 * [TPSP] §把通信藏到计算后面). out = Reduce_r(x[r] . w[r]) with x stacked [t][N][k/t] and w stacked
 * [t][k/t][n], without materialising the fp32 partials. The kernel computes each output tile's t
 * shard products in ring order (c+1, ..., c for the tile's chunk c), accumulates them in binary32
 * exactly as tp_reduce_scatter would, and writes the tile once:
 *   TP_OUT_RS           out[r] receives chunk r: [N/t, n] (axis 0) or [N, n/t] (axis 1)
 *   TP_OUT_AR           every out[r] receives the whole [N, n] sum: a ReduceScatter along `axis`
 *                       (which fixes each element's summation order: its row chunk for 0, its
 *                       column chunk for 1; [CH06] §6.4) with its AllGather folded into the same
 *                       epilogue
 *   TP_OUT_RS_AG        as TP_OUT_AR with the ReduceScatter along tokens (axis 0), whatever `axis` says
 * Results are bit-identical to tp_row_linear followed by tp_reduce_scatter(axis) (and, for the
 * AllReduce modes, tp_all_gather(axis); for axis 0 that is tp_all_reduce).
 * The fused kernel needs (N/t) % 128 == 0 for axis 0, or (n/t) % 256 == 0 for axis 1. Otherwise
 * `partials` (t fp32 [N, n] buffers, else NULL) is used for the unfused path, and without it the
 * call returns TP_EUNSUPPORTED. Aligned; k/t and n multiples of 8. */
tp_status tp_row_linear_reduce(const uint16_t* x, int64_t N, int64_t k, int64_t n, int t, const uint16_t* w,
                               tp_reduce mode, int axis, float* const* out, float* const* partials, void* stream);

/* ------------------------------------------------------------------------------------------------
 * The tensor-parallel MLP forward ([TPSP] §MLP：先列后行，只通信一次; [PFY] §Tensor Parallel;
 * [CH06] §6.9 Problem 5): Z_r = act(X W_in[r]) (column-parallel, local), U_r = Z_r W_down[r]
 * (row-parallel, full-shape partial), then the collective `mode` selects.
 *   x       bf16 [N, h], shared by all shards
 *   w_in    bf16 stacked [t][h][F/t] (GELU/NONE) or [t][h][2F/t] (SWIGLU, from tp_shard_gate_up)
 *   w_down  bf16 stacked [t][F/t][h] (from tp_shard_rows)
 *   z_ws    bf16 workspace [t][N][F/t] (the activations Z_r)
 *   partials t fp32 [N, h] buffers (the {U}): the result in TP_OUT_PARTIALS mode. The reducing modes
 *           fuse the row GEMM with its collective (tp_row_linear_reduce) whenever (N/t) % 128 == 0,
 *           and then never touch partials, which may be NULL. Otherwise they are scratch.
 *   out     t fp32 buffers: unused for PARTIALS; [N/t, h] for RS (t | N); [N, h] for AR and RS_AG
 * Aligned; h and F/t multiples of 8. */
tp_status tp_mlp_fwd(const uint16_t* x, int64_t N, int64_t h, int64_t F, int t, tp_act act,
                     const uint16_t* w_in, const uint16_t* w_down, uint16_t* z_ws, float* const* partials,
                     tp_reduce mode, float* const* out, void* stream);

/* Backward of the tensor-parallel MLP ([TPSP] §矩阵乘法的两种切法, backward bullets, and §f 和 g; [PFY]
 * §Tensor Parallel, the gradient identities). dY is replicated, since g's backward is the identity:
 *   dZ_r = dY W_down[r]^T;  dW_down[r] = Z_r^T dY;  dH_r = act'(H_r) * dZ_r (SwiGLU: dG = dZ*U*SiLU'(G),
 *   dU = dZ*SiLU(G));  dW_in[r] = X^T dH_r;  dX = sum_r dH_r W_in[r]^T (f's backward: a ring AllReduce).
 *   x, dy   bf16 [N, h];  w_in / w_down as in tp_mlp_fwd
 *   h_pre   bf16 stacked [t][N][wn], the forward pre-activations H_r = X W_in[r] (wn = F/t, or 2F/t for
 *           SwiGLU: [G | U]; e.g. from tp_column_linear with TP_ACT_NONE)
 *   z       bf16 stacked [t][N][F/t], the forward activations Z_r
 *   dz_ws   bf16 workspace [t][N][F/t];  dh_ws bf16 workspace [t][N][wn]
 *   dw_in   fp32 stacked [t][h][wn];  dw_down fp32 stacked [t][F/t][h];  dx  t fp32 [N, h] (identical replicas)
 * N, h and F/t multiples of 8; t | N. */
tp_status tp_mlp_bwd(const uint16_t* x, const uint16_t* dy, int64_t N, int64_t h, int64_t F, int t, tp_act act,
                     const uint16_t* w_in, const uint16_t* w_down, const uint16_t* h_pre, const uint16_t* z,
                     uint16_t* dz_ws, uint16_t* dh_ws, float* dw_in, float* dw_down, float* const* dx, void* stream);

/* ------------------------------------------------------------------------------------------------
 * Tensor + sequence parallelism ([TPSP] §序列并行：把剩下的激活也切开). In the replicated region each
 * shard holds only its own block of tokens, x[r] = rows [rN/t, (r+1)N/t) of X. The entry g is an
 * AllGather along tokens and the exit g-bar a ReduceScatter along tokens. Same bytes as pure TP.
 * ------------------------------------------------------------------------------------------------ */
/* Column-parallel linear whose input is the AllGather of the t token shards x[r] (bf16 [N/t, k], host
 * array of device pointers): y[r] = act(AllGather(x) . w[r]), stacked [t][N][n/t] bf16, with w as in
 * tp_column_linear. The gathered X is never materialised: every 128-row tile of the GEMM's input is
 * read from the shard that holds it. Needs (N/t) % 128 == 0 (TP_EUNSUPPORTED otherwise). */
tp_status tp_column_linear_sp(const uint16_t* const* x, int64_t N, int64_t k, int64_t n, int t, tp_act act,
                              const uint16_t* w, uint16_t* y, void* stream);
/* The MLP under TP+SP: out[r] (fp32 [N/t, h]) = rows r of act(AllGather(x) W_in) W_down, i.e.
 * tp_column_linear_sp, then the row GEMM fused with the ReduceScatter along tokens. x[r] bf16 [N/t, h];
 * w_in, w_down and z_ws as in tp_mlp_fwd. Bit-identical to tp_mlp_fwd(TP_OUT_RS) on the gathered X.
 * Needs (N/t) % 128 == 0. */
tp_status tp_mlp_fwd_sp(const uint16_t* const* x, int64_t N, int64_t h, int64_t F, int t, tp_act act,
                        const uint16_t* w_in, const uint16_t* w_down, uint16_t* z_ws, float* const* out,
                        void* stream);

/* ------------------------------------------------------------------------------------------------
 * The four sharded-matmul cases of C[B,F] = X[B,D] . W[D,F] over t shards ([CH06] §6.2, §6.9
 * Problems 4 and 9). x[] and w[] are host arrays of t device pointers (bf16, row-major); entries of a
 * replicated operand may point to the same buffer. c[] receives t outputs of c_dtype.
 *   case 1 X[B_X, D] . W[D, F]: x[i] [B/t, D], w[i] [D, F] -> c[i] [B/t, F]; no communication.
 *   case 2 X[B, D_X] . W[D, F]: x[i] [B, D/t], w[i] [D, F] (replicated)
 *       ALLGATHER: every shard gathers X and computes the full C -> c[i] [B, F] (t x the FLOPs)
 *       ALLREDUCE: shard i multiplies by its row block of W, then AllReduce -> c[i] [B, F]
 *   case 3 X[B, D_X] . W[D_X, F]: x[i] [B, D/t], w[i] [D/t, F] -> partial C{U_X}, then
 *       ALLREDUCE -> c[i] [B, F]; RS_B -> c[i] [B/t, F]; RS_F -> c[i] [B, F/t]
 *   case 4 X[B_X, D] . W[D, F_X] (only diagonal blocks as is), fixed by
 *       GATHER_X -> c[i] [B, F/t]; GATHER_W -> c[i] [B/t, F]
 * Partial sums are fp32 and reduced in the ring order above; a bf16 c_dtype rounds once at the end.
 * The workspace (device, >= tp_sharded_matmul_ws_bytes) holds gathered operands or partials. It is
 * 0 bytes (ws may be NULL)
 *   - when the fused row GEMM + ring reduction computes case 2 AllReduce or a case-3 strategy, i.e.
 *     when every reduction chunk is a whole number of 128-row tiles (256-column tiles for RS_F);
 *   - when the GEMM reads the gathered operand's pieces where they lie instead of a gathered copy
 *     ([CH06] §6.6, the gather folded into the matmul): case 2 AllGather with (D/t) % 64 == 0
 *     (each k-block of X read from the shard that holds it), case 4 GATHER_X with (B/t) % 128 == 0
 *     (each 128-row tile of X likewise), case 4 GATHER_W with (F/t) % 64 == 0 (each 64-column box
 *     of W likewise). Otherwise the gather is materialised in the workspace, one copy per shard. */
size_t tp_sharded_matmul_ws_bytes(int case_id, int strategy, int64_t B, int64_t D, int64_t F, int t);
/* The strategy that the pages' cost rule picks ([CH06] §6.2 cases 2 and 4, §6.9 Problem 4), written
 * to *strategy. The rule compares the elements a ring of t devices would move, taking operands and
 * output to have the same element type:
 *   case 1  TP_CASE1_LOCAL: nothing moves;
 *   case 2  TP_CASE2_ALLGATHER when gathering X (B*D elements) moves no more than the AllReduce of
 *           C (about 2*B*F), else TP_CASE2_ALLREDUCE. For the weight-gathering orientation of
 *           Problem 4 this is the page's "AllReduce when D > 2B";
 *   case 4  gather the smaller operand: TP_CASE4_GATHER_X when B*D <= D*F, else TP_CASE4_GATHER_W;
 *   case 3  TP_EUNSUPPORTED: its three strategies reduce the same partials, and the sharding the
 *           caller wants for C decides among them (replicated, rows or columns).
 * On one GPU the gathers cost no traffic (the GEMM reads the pieces in place); this reports the
 * multi-device choice. Host-only; sizes must be positive, 1 <= t <= TP_MAX_SHARDS (TP_EINVAL). */
tp_status tp_sharded_matmul_choose(int case_id, int64_t B, int64_t D, int64_t F, int t, int* strategy);
tp_status tp_sharded_matmul(int case_id, int strategy, const uint16_t* const* x, const uint16_t* const* w,
                            int64_t B, int64_t D, int64_t F, int t, void* const* c, tp_dtype c_dtype,
                            void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------------------------
 * One tensor-parallel transformer layer without its attention core ([TPSP] §注意力：按头切 and §MLP;
 * 2 AllReduces per layer forward): qkv[r] = X W_qkv[r] (column-parallel; its output feeds the
 * attention core, which is outside this library); attn = AllReduce_r(O[r] W_o[r]); h1 = X + attn (fp32);
 * the MLP (SwiGLU) runs on bf16(h1); y = h1 + AllReduce_r(MLP partials).
 *   x      bf16 [N, h];  o: t device pointers, bf16 [N, n_h*d_h/t] (each shard's attention output)
 *   w_qkv  bf16 stacked [t][h][(n_h/t + 2kv)*d_h] (tp_shard_qkv); w_o bf16 stacked [t][n_h*d_h/t][h]
 *   w_gu   bf16 stacked [t][h][2F/t];  w_down bf16 stacked [t][F/t][h]
 *   qkv_out bf16 stacked [t][N][(n_h/t + 2kv)*d_h]
 *   h1     t fp32 [N, h] (replicas of the residual stream after attention); h1_bf16 bf16 [N, h]
 *   z_ws   bf16 [t][N][F/t]; y t fp32 [N, h]
 *   partials t fp32 [N, h] scratch, needed only when neither (h/t) % 256 == 0 nor (N/t) % 128 == 0;
 *          otherwise both row GEMMs are fused with their AllReduce (and residual) and partials may
 *          be NULL
 * Both AllReduces scatter along h (their summation order follows column chunks of h/t) when
 * (h/t) % 256 == 0, else along tokens: along h, all row-tiles of a chunk read the same shard's weight
 * panel at the same time, so the weights stream from DRAM about once rather than once per row-tile.
 * ------------------------------------------------------------------------------------------------ */
tp_status tp_layer_fwd(const uint16_t* x, const uint16_t* const* o, int64_t N, int64_t h, int n_h, int n_kv,
                       int d_h, int64_t F, int t, const uint16_t* w_qkv, const uint16_t* w_o,
                       const uint16_t* w_gu, const uint16_t* w_down, uint16_t* qkv_out, float* const* h1,
                       uint16_t* h1_bf16, uint16_t* z_ws, float* const* partials, float* const* y, void* stream);

/* ------------------------------------------------------------------------------------------------
 * tp_mlp_fwd without caller-provided scratch. The pages have no counterpart: this entry point exists
 * for callers that cannot allocate device memory. Examples are code inside a host framework whose
 * caching pool owns the GPU's memory, where an allocation behind the pool's back can fail or escape
 * its accounting, and serving loops that forbid cudaMalloc/cudaFree after start-up because those
 * calls can synchronise the device.
 * Same computation, arguments and results as tp_mlp_fwd, minus z_ws and partials. The activations
 * and the fp32 partials live in one array of TP_MLP_NOALLOC_SCRATCH_BYTES compiled into the library,
 * which every GPU that loads the library holds until the process exits.
 *   - The scratch needed is N*F*2 bytes (Z), rounded up to 256, plus t*N*h*4 (the fp32 partials,
 *     each rounded up to 256) only when a reducing mode takes the unfused path, i.e. when
 *     (N/t) % 128 != 0; with (N/t) % 128 == 0 the row GEMM is fused with its reduction and keeps the
 *     partials on chip. Requests needing more than the array return TP_ENOSPACE before any launch
 *     (sizes are bounded before they are multiplied, so huge N, h or F cannot wrap the check).
 *   - In TP_OUT_PARTIALS mode the partials are written to out[] (t fp32 [N, h] buffers).
 *   - All calls share the array and it keeps the last call's contents; every call overwrites all
 *     the scratch it reads, so nothing needs clearing. Calls that overlap on the GPU race on it.
 *   - The first call on a device resolves the array's address (it may load the module); make it
 *     before any stream capture.
 *   - No cudaMalloc, cudaFree or allocating library routine is called.
 * ------------------------------------------------------------------------------------------------ */
#define TP_MLP_NOALLOC_SCRATCH_BYTES (32u << 20)
tp_status tp_mlp_fwd_noalloc(const uint16_t* x, int64_t N, int64_t h, int64_t F, int t, tp_act act,
                             const uint16_t* w_in, const uint16_t* w_down, tp_reduce mode, float* const* out,
                             void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TP_H_ */
