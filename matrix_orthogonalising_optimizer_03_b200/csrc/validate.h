// Host-side argument validation shared by the C entry points of libmuon.
#pragma once
#include "muon.h"

namespace muon {

// Host validation of a Newton-Schulz-only matrix list and its hyper-parameters
// (null pointers, enums, flags, eps, shapes, leading dimensions, dtypes, alignment,
// aliasing). Makes no CUDA call. Every Newton-Schulz entry point uses it, so the
// same arguments get the same status from each of them.
muon_status_t validate_ns(const muon_ns_matrix_t* mats, int n, const muon_hparams_t* hp);

}  // namespace muon
