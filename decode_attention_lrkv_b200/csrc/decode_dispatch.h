// Decode dispatch, shared by lrkv_decode_attn, lrkv_append_decode_attn and
// lrkv_decode_attn_noalloc.  The kernels are instantiated in their own
// translation units (decode_g*.cu, decode_simple.cu) so the library builds in
// parallel; this header only declares their launchers.
#pragma once

#include <cuda_runtime.h>

#include "decode_params.cuh"

namespace lrkv {

// Whether the streaming (tensor-core) kernel covers these sizes: the rank
// pairs it is instantiated for, any number of query heads per kv head.
bool stream_decode_supported(const lrkv_dims& D);

// The tensor-core streaming kernel for the shapes it is instantiated for (1
// or 2 query heads per kv head in one launch, more in launches of 4 heads,
// each streaming the cache), the CUDA-core kernel for every other valid
// shape.  p.k_new set: the fused append + decode, which only the streaming
// kernel has (its first launch appends).
lrkv_status launch_decode(const DecodeParams& p, cudaStream_t s);

// Per query-group launchers of the streaming kernel (*done = false: no
// instantiation for these ranks), and the CUDA-core kernel for any group.
lrkv_status launch_stream_g1(const DecodeParams& p, dim3 grid, cudaStream_t s, bool* done);
lrkv_status launch_stream_g2(const DecodeParams& p, dim3 grid, cudaStream_t s, bool* done);
lrkv_status launch_stream_g4(const DecodeParams& p, dim3 grid, cudaStream_t s, bool* done);
lrkv_status launch_simple_any(const DecodeParams& p, dim3 grid, cudaStream_t s);

}  // namespace lrkv
