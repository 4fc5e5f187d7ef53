// Host interface of the whole-layer decode kernel (decode_fused.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

constexpr int kDecMaxT = 16;  // batches of at most this many tokens

// Whether moe_layer_forward runs `s` as one decode kernel: bf16, 1 <= T <=
// kDecMaxT, d in {256, 512, 1024, 2048}, inter % 64 == 0, and no GEMM tile
// shape or failure injection forced by the flags.
bool decode_fused_eligible(const moe_shape_t& s);

// Workspace the kernel needs: partial rows of d fp32 values, and the sync words.
size_t decode_partial_rows(const moe_shape_t& s);
size_t decode_sync_bytes();

// The layer forward of an eligible shape: zeroes `sync` and launches one
// kernel of `sms` CTAs on `st`.  idx, w ([T, K]), logits ([T, n_routed]),
// part ([decode_partial_rows, d]) and sync are workspace regions.
int launch_decode_fused(const moe_shape_t& s, const void* u, const void* E, const float* bias,
                        const void* W13, const void* W2, const void* W13_s, const void* W2_s,
                        void* h, int32_t* idx, float* w, float* logits, float* part, void* sync,
                        int32_t* status, int sms, cudaStream_t st);

// Router, dispatch and gather of a batch of at most 128 tokens in one
// launch (decode_front.cu): bf16, d in {256, 512, 1024, 2048}, the default
// router.  Writes idx, w, counts, offsets, perm, inv and xperm as
// moe_route + moe_dispatch + the gather would (logits up to fp32 summation
// order); logits ([T, n]) and sync are workspace scratch.
bool decode_front_eligible(const moe_shape_t& s);
size_t decode_front_sync_bytes();
int launch_decode_front(const moe_shape_t& s, const void* u, const void* E, const float* bias,
                        int32_t* idx, float* w, float* logits, int32_t* counts, int32_t* offsets,
                        int32_t* perm, int32_t* inv, void* xperm, void* sync, int32_t* status,
                        int sms, cudaStream_t st);

}  // namespace moe
