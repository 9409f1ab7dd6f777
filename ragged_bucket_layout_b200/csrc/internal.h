// Internal declarations shared by the planner (planner.cpp) and the device
// runtime (dbuf.cu).  Not part of the C-ABI.
#pragma once

#include <cstdint>
#include <string>
#include <vector>

#include "dbuf.h"

struct dbuf_plan_s {
    int32_t n = 0, m = 1;
    int64_t align = 16;
    int64_t slice = 0, bucket = 0, padding = 0, n_blocks = 0;
    std::vector<int64_t> rows, cols, k;  // caller order
    std::vector<int64_t> tile_cols;      // caller order; 0 = whole rows (see dbuf_tensor_desc)
    std::vector<int64_t> offset;         // caller order
    std::vector<int32_t> by_offset;      // tensor ids in bucket order
};

namespace dbuf_detail {

// Thread-local error message of the C-ABI.
void set_error(const std::string& msg);
dbuf_status fail(dbuf_status st, const std::string& msg);

// Tensor count and device of a dbuf (for the Muon state in muon.cu).
int32_t tensors_of(const dbuf_t* db);
int device_of(const dbuf_t* db);

}  // namespace dbuf_detail

// Return DBUF_ECUDA with the CUDA error text from a C-ABI function (CUDA
// sources only).
#define CUDA_TRY(call, what)                                                                            \
    do {                                                                                                \
        cudaError_t e_ = (call);                                                                        \
        if (e_ != cudaSuccess)                                                                          \
            return dbuf_detail::fail(DBUF_ECUDA, std::string(what) + ": " + cudaGetErrorString(e_));    \
    } while (0)
