// dl_kernels.cuh -- the DeltaLog kernels for sm_100a (dl_step.cuh,
// dl_merge.cuh, dl_eager.cuh; shared pieces in dl_common.cuh and dl_q8.cuh).
//
// Notation ("DeltaLog: Deferred Materialization of Recurrent States for Linear
// Attention Decoding", Abstract): each head keeps a dense base S_b (fp32, or
// int8 codes with one fp32 scale per row -- the base quantized once per
// window, "LeapQuant" Abstract -- d_v x d_k, row = value index) and a
// bounded log of f < L compact entries
// (u_i, k_i, g_i), g_i = log of the decay accumulated since the base was
// merged (a scalar for GDN, a d_k vector for KDA and RWKV6).  The dense state
// the model sees is
//     S = S_b Diag(e^{g}) + sum_i u_i (k_i o e^{g - g_i})^T,
// g being the newest accumulated log-decay.  Keeping log-decay and forming
// only differences g - g_i <= 0 keeps every factor in (0, 1], so long runs of
// strong decay (RWKV6) cannot overflow or lose the ratio to underflow.
//
// Kernels (one CTA per (sequence, head), blockIdx.x = b*H + h):
//   dl_step_kernel   : decode step. Streams S_b into shared memory with bulk
//                      copies (TMA), forms S_b k-hat and S_b q-hat with one
//                      pass over the tile, adds the log correction from the
//                      log entries staged in shared memory, writes o_t and
//                      appends (u_t, k_t, g_t).  With FUSED, a head whose
//                      append would fill the log writes the merged base
//                      instead (it already holds S_b and the whole log).
//   dl_merge_kernel  : folds a log into the base (or into a separate output
//                      for materialize) -- a rank-f update of the tile.  An
//                      int8 base is requantized row by row as it is written.
//   dl_eager_kernel  : the dense read-modify-write step eager decoding does.
#pragma once

#include "dl_step.cuh"
#include "dl_merge.cuh"
#include "dl_eager.cuh"
