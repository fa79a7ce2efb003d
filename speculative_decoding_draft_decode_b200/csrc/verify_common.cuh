// verify_common.cuh — pieces shared by the verify kernels: the state the
// rejection pass hands to the resample pass, the row statistics kept or
// exchanged for the draft statistics and the vocabulary-sharded path, and
// the programmatic-launch controls.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace specdec {

// Per-request state handed from the rejection statistics pass to the
// resample pass.
struct RejState {
    int32_t h;       // accepted drafts
    int32_t valid;   // 0: the request's target distribution is undefined
    float M;         // max logit of row h
    float pad;
    double Z;        // sum exp((l - M)/T) of row h
    int64_t row;     // logit row h, which is also the output slot of the drawn token
    int64_t qrow;    // q row h when a draft was rejected (residual), else -1 (bonus from p)
    int64_t pad2;
};

// Row statistics of the softmax pass, kept for every row when the draft
// statistics are requested: M = max logit, Z = sum exp((l - M) / T).
struct RowStat {
    float M;
    float pad;
    double Z;
};

// Vocabulary-sharded rejection: one row's statistics over one shard's
// columns, exchanged between the ranks: the max logit and sum exp((l - M)/T)
// of the shard, and, when the shard holds the row's draft token, its logit
// and q value.
struct ShardRowStat {
    float M;
    float l_draft;
    float q_draft;
    int32_t owned;  // 1: this shard holds the draft token of the row
    double S;
    double pad;
};

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start while the previous kernel of the stream finishes;
// griddepcontrol.wait blocks until that kernel has completed and its memory
// is visible, so every global access comes after it.  launch_dependents lets
// the next such kernel start its own launch early.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

}  // namespace specdec
