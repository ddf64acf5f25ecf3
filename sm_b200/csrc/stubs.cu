// Registry hooks for the tuned implementations; replaced as they are added.
#include "kvq_internal.cuh"

namespace kvq {

const AttendImpl* chunk_attend_impl() { return nullptr; }
}  // namespace kvq
