// kernels.cuh -- the sm_100a kernels of the decode-attention hot path.
//
//  * gqa_partition_bf16_kernel<D, NT>: one CTA owns one (sequence b, KV head g,
//    key chunk c) tile. A producer warp streams the chunk's K/V rows of head g
//    through a ring of shared-memory stages with TMA (2-D tiled loads, 128-byte
//    swizzle, no multicast); four consumer warps each take 16 keys of every
//    stage and, for ALL heads_per_kv query heads of the group at once, compute
//    the logits S^T = K Q^T and the value sum O^T += V^T P^T on the tensor cores
//    (mma.sync m16n8k16, bf16 in, fp32 accumulate), with the online softmax
//    (running max m, partition l) in fp32 registers. K/V rows are read from HBM
//    once per group and broadcast to its query heads (cortiq_engine
//    NystromState: every Q head of a group reads the same K/V rows; needle_core
//    attn.rs: broadcast, not repeat-copy).
//  * gqa_partition_f32_kernel<D, HMAX>: the fp32 K/V variant on CUDA cores
//    (fp32 FMA keeps the fp32 tolerance; no tensor-core format is exact here).
//  * The CTA that completes the last split of a (sequence, KV head) segment
//    merges the segment's partial states and the carry and writes the output
//    (ticket counter per segment), so one launch does the whole call.
//  * gqa_merge_kernel<D>: the standalone merge of caller-held states and a
//    carry (USearch linear algebra, DenseAttendConfig::carry: partial-softmax
//    rescaling), optional state out, optional out = acc / l.
//  * gqa_partition_coded_kernel<D, HMAX, MW>: the same tiles over a
//    dictionary-coded cache (qualiaDB KvDictionary read path): logits by table
//    lookup, value weights summed in fixed point with 32-bit shared atomics.
//  * gqa_topk_to_bias_kernel: index rows -> additive bias (metrale
//    glm5next_dsa_ref, topk_to_mask).
//
// The pieces live in tile.cuh (shared tile logic, partial states, fused
// merge), partition_bf16.cuh, partition_f32.cuh, merge.cuh, coded.cuh and
// topk.cuh; this header gathers them.
//
// Inside the partition kernels logits are kept in base 2 (scale * log2 e folded
// into one multiply) so that exp2 is the only transcendental; every state that
// leaves a kernel stores m in natural-log units (the largest logit).
#pragma once

#include "tile.cuh"
#include "partition_bf16.cuh"
#include "partition_f32.cuh"
#include "merge.cuh"
#include "coded.cuh"
#include "topk.cuh"
