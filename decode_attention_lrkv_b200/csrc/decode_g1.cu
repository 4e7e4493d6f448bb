// The streaming decode kernel for 1 query head(s) per kv head, every rank pair.
#include "decode_dispatch.h"
#include "decode_launch.cuh"

namespace lrkv {

lrkv_status launch_stream_g1(const DecodeParams& p, dim3 grid, cudaStream_t s, bool* done) {
  return launch_stream_g<1>(p, grid, s, done);
}

}  // namespace lrkv
