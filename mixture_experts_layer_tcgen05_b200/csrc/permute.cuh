// Shared by the permutation kernels and the forward that chooses between them.
#pragma once

namespace moe {

// Routed rows (T*k) up to which the permutation and the row gather run as one
// launch (permute_gather_small_kernel); larger batches take the chunked path.
constexpr int kSmallPermRows = 1024;

}  // namespace moe
