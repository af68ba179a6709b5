/*
 * dlrm_mlp.h -- C ABI of the DLRMv1 MLP layers around the sparse stage, on
 * B200 tensor cores (tcgen05).
 *
 * The pages (luminal compare main...vanilla-pytorch, matmul2d.rs) fuse each
 * DLRMv1 MLP layer into one matmul kernel with the bias and the activation in
 * its store path:
 *   - linear_bias / linear_bias_relu / linear_bias_sigmoid:
 *         Y = act(A W^T + bias), A (M, K), W (N, K) row-major (the nn.Linear
 *         weight layout, "transpose_b"), bias (N,), act in {none, ReLU,
 *         sigmoid} applied to acc + bias (Activation enum doc comment);
 *   - linear_bias_split_a and its ReLU/Sigmoid forms: A's columns 0..K_lo-1
 *     come from A_lo and K_lo..K-1 from A_hi, so the top MLP's first layer
 *     reads [dense | interaction] without building the concatenation
 *     (a_split field doc comment).
 * The bottom MLP turns the dense features into the (B, D) `dense` input of
 * the interaction; the top MLP's first layer takes [dense | z] with the split
 * form, and the last layer is the CTR head (sigmoid).
 *
 * Precision: the pages' matmul multiplies f32 activations with f32 or
 * bf16-stored weights on CUDA cores. dlrm_linear_f32a keeps that arithmetic
 * on the tensor cores: each f32 activation is three exact bf16 planes, every
 * product is exact, and the sum is accumulated in f32 (in TMEM); bias and
 * activation are applied in f32. dlrm_linear_bf16 is the cheaper variant with
 * bf16 activations (one plane): A and W bf16, products exact, f32
 * accumulation. A layer's output can be written as f32, as bf16
 * (round-to-nearest-even) or as three planes for the next layer.
 *
 * Conventions are those of dlrm_sparse.h: "dev" pointers are device pointers
 * on the current device, the caller owns every buffer, nothing is allocated,
 * calls are asynchronous on `stream` and capturable into CUDA graphs, a
 * negative return is a dlrm_status_t and host-side checks run before anything
 * is launched. bf16 values travel as uint16_t bit patterns.
 */
#ifndef DLRM_MLP_H
#define DLRM_MLP_H

#include <stdint.h>

#include "dlrm_sparse.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Activation of a layer, applied to acc + bias (matmul2d.rs, Activation). */
typedef enum {
    DLRM_ACT_NONE = 0,
    DLRM_ACT_RELU = 1,    /* max(x, 0) */
    DLRM_ACT_SIGMOID = 2  /* 1 / (1 + exp(-x)) */
} dlrm_act_t;

/*
 * dlrm_linear_bf16 -- one MLP layer Y = act([A_lo | A_hi] W^T + bias).
 *   a_lo     dev (M, lda_lo) bf16 rows; columns [0, k_lo) are used. Required.
 *   a_hi     dev (M, lda_hi) bf16 rows; columns [0, k_hi) are used. NULL and
 *            k_hi = 0 for a plain layer.
 *   w        dev (N, ldw) bf16 rows; columns [0, k_lo + k_hi) are used.
 *   bias     dev (N,) f32, or NULL for no bias.
 *   act      dlrm_act_t.
 *   y_f32    dev (M, ldy_f32) f32 rows of the result, or NULL.
 *   y_bf16   dev (M, ldy_bf16) bf16 rows of the result, or NULL. At least one
 *            of y_f32, y_bf16 is given.
 *   status_dev dev int32, or NULL: DLRM_FLAG_TIMEOUT is OR-ed in if a bounded
 *            wait of the kernel ran out (the results are then not valid).
 * Requirements (DLRM_ERR_SHAPE / DLRM_ERR_ALIGN / DLRM_ERR_ARG otherwise):
 *   M >= 1, N >= 1, k_lo >= 1, k_hi >= 0, all of M, N, K < 2^31;
 *   lda_lo >= k_lo, lda_hi >= k_hi, ldw >= k_lo + k_hi, ldy_* >= N;
 *   lda_lo, lda_hi, ldw multiples of 8 (16-byte rows for the TMA loads) and
 *   a_lo, a_hi, w 16-byte aligned; k_lo a multiple of 8 when k_hi > 0;
 *   bias and y_f32 4-byte aligned, y_bf16 2-byte aligned.
 * Columns past k of A and W rows are never read; rows and columns of Y past
 * (M, N) are never written.
 */
DLRM_API int dlrm_linear_bf16(const uint16_t* a_lo, int64_t lda_lo, int64_t k_lo,
                              const uint16_t* a_hi, int64_t lda_hi, int64_t k_hi,
                              const uint16_t* w, int64_t ldw, const float* bias, int64_t M,
                              int64_t N, int act, float* y_f32, int64_t ldy_f32,
                              uint16_t* y_bf16, int64_t ldy_bf16, int32_t* status_dev,
                              dlrm_stream_t stream);

/*
 * dlrm_linear_f32a -- one MLP layer with f32 activations, the pages' own
 * mixed-precision linear (matmul2d.rs: A F32 (M, K) times weights BF16 or F32
 * (N, K), result F32, with the bias / ReLU / sigmoid epilogue and the split-A
 * form): Y = act([A_lo | A_hi] W^T + bias).
 *
 * Each f32 activation travels as three bf16 "planes" whose sum is the value
 * exactly (x = p0 + p1 + p2: p0 keeps x's top 8 significant bits, p1 the next
 * 8 of the remainder, p2 the rest; dlrm_split_f32_bf16x3 writes them, and a
 * layer can write its own output that way for the next one). The tensor
 * cores multiply bf16 exactly, so the layer sums the exact products
 * p_i * w for all three planes in f32 (in TMEM): the only error is that f32
 * accumulation, |Y - exact| <= (3K + 2) * 2^-23 * (sum_k |a_k w_k| + |bias|)
 * before the activation. f32 weights are given as three planes too
 * (w_planes = 3, split once with dlrm_split_f32_bf16x3); then the six
 * products p_i * q_j with i + j < 3 are summed, which leaves out terms below
 * 2^-20 * |a_k w_k| and adds that to the bound (6K accumulated products).
 *   a_lo      dev bf16, three planes of (M, lda_lo) rows, splane_lo elements
 *             apart; columns [0, k_lo) are used. Required.
 *   a_hi      dev bf16, three planes of (M, lda_hi) rows, splane_hi apart;
 *             columns [0, k_hi). NULL and k_hi = 0 for a plain layer.
 *   w         dev bf16 (N, ldw) rows: the weights (w_planes = 1), or three
 *             planes splane_w elements apart (w_planes = 3, f32 weights).
 *   bias, act as for dlrm_linear_bf16.
 *   y_f32     dev (M, ldy_f32) f32 result, or NULL.
 *   y_planes  dev bf16, three planes of (M, ldy_planes) rows splane_y apart:
 *             the exact split of the f32 result (the next layer's input), or
 *             NULL. At least one of y_f32, y_planes is given.
 *   status_dev as for dlrm_linear_bf16.
 * Requirements: those of dlrm_linear_bf16, plus plane strides that are
 * multiples of 8 elements and hold a whole plane (splane_lo >= (M-1)*lda_lo +
 * k_lo, and so on; DLRM_ERR_SHAPE / DLRM_ERR_ALIGN), w_planes 1 or 3
 * (DLRM_ERR_ARG). Tiny values below about 2^-110 may lose their last plane to
 * the tensor cores' handling of subnormal bf16 inputs.
 */
DLRM_API int dlrm_linear_f32a(const uint16_t* a_lo, int64_t lda_lo, int64_t splane_lo,
                              int64_t k_lo, const uint16_t* a_hi, int64_t lda_hi,
                              int64_t splane_hi, int64_t k_hi, const uint16_t* w, int64_t ldw,
                              int64_t splane_w, int w_planes, const float* bias, int64_t M,
                              int64_t N, int act, float* y_f32, int64_t ldy_f32,
                              uint16_t* y_planes, int64_t ldy_planes, int64_t splane_y,
                              int32_t* status_dev, dlrm_stream_t stream);

/*
 * dlrm_split_f32_bf16x3 -- the exact three-plane split of an f32 matrix:
 * for r < rows, c < cols, y[p*splane + r*ldy + c] (p = 0, 1, 2) are the bf16
 * bit patterns p0, p1, p2 with x[r][c] = p0 + p1 + p2 exactly (p0: x with the
 * low 16 bits of its encoding cleared; p1: the same of x - p0; p2: the rest).
 * x dev f32 (rows, ldx), y dev bf16; ldx, ldy >= cols, splane >= (rows-1)*ldy
 * + cols; x 4-byte and y 2-byte aligned.
 */
DLRM_API int dlrm_split_f32_bf16x3(const float* x, int64_t ldx, int64_t rows, int64_t cols,
                                   uint16_t* y, int64_t ldy, int64_t splane,
                                   dlrm_stream_t stream);

/*
 * dlrm_f32_to_bf16 -- y[r][c] = bf16 round-to-nearest-even of x[r][c] for
 * r < rows, c < cols (dev, row pitches ldx and ldy in elements, ldx, ldy >=
 * cols). Feeds f32 tensors (the dense features, the interaction z) to the
 * bf16 layers. x 4-byte and y 2-byte aligned.
 */
DLRM_API int dlrm_f32_to_bf16(const float* x, int64_t ldx, int64_t rows, int64_t cols,
                              uint16_t* y, int64_t ldy, dlrm_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DLRM_MLP_H */
