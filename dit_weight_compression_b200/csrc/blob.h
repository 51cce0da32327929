// blob.h -- the library-owned blob object behind the opaque ep_blob handle, and the per-thread
// error message helpers shared by the host API (api.cpp) and the GPU API (decode.cu).
#pragma once

#include <cuda_runtime_api.h>

#include <mutex>
#include <string>
#include <vector>

#include "entropack.h"
#include "format.h"

namespace ep {

constexpr int kMaxDevices = 64;
constexpr int kMaxHostChunks = 8;   // host-output path: most chunks one call is split into

// Device-side state of one blob on one GPU.
struct DeviceCopy {
    uint8_t* blob = nullptr;        // copy of the serialised bytes (decode reads this)
    uint8_t* tables[6] = {};        // decode tables expanded from the blob's frequency tables, one
                                    // block per table layout (10, 12, 13, 14, 11, 15), each made on first use
    uint32_t* status = nullptr;     // sticky error bits written by the decode kernel
    uint8_t* stage_blob = nullptr;  // host-output path: per-call upload target
    uint8_t* stage_out = nullptr;   // host-output path: decode target before the D2H copy
    size_t stage_out_bytes = 0;
    float* stage_sigma = nullptr;   // host-output path of the row-scaled FP8 container: row scales
    cudaEvent_t chunk_done[kMaxHostChunks] = {};  // host-output path: chunk i decoded
};

int set_error(int code, const std::string& msg);
int set_error_static(int code, const char* msg);  // msg must be a string literal; no allocation
void clear_error();

}  // namespace ep

struct ep_blob {
    std::vector<uint8_t> bytes;
    ep::BlobLayout layout;
    std::mutex mu;                  // guards lazy device set-up
    ep::DeviceCopy dev[ep::kMaxDevices];
    bool host_pinned = false;
};
