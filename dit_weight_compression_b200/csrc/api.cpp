// api.cpp -- host-side entry points of the C ABI: compression, blob bytes, header fields,
// actual_bpp and the per-thread error message.  The GPU entry points live in decode.cu.
#include <cmath>
#include <cstring>
#include <new>

#include <cuda_runtime.h>

#include "blob.h"

namespace ep {

static thread_local std::string g_error;
static thread_local const char* g_static_error = nullptr;  // set by paths that must not allocate

int set_error(int code, const std::string& msg) {
    g_static_error = nullptr;
    g_error = msg;
    return code;
}
int set_error_static(int code, const char* msg) {
    g_static_error = msg;
    return code;
}
void clear_error() {
    g_static_error = nullptr;
    g_error.clear();
}

}  // namespace ep

using namespace ep;

extern "C" const char* ep_last_error(void) { return g_static_error ? g_static_error : g_error.c_str(); }

extern "C" int ep_compress_ex(const ep_tensor* in, double target_bpp, const ep_options* opt, ep_blob** out) {
    clear_error();
    if (!in || !out) return set_error(EP_ERR_ARG, "ep_compress: NULL argument");
    *out = nullptr;
    int es = dtype_bytes(in->dtype);
    if (es == 0) return set_error(EP_ERR_DTYPE, "ep_compress: unsupported dtype");
    if (in->rows <= 0 || in->cols <= 0) return set_error(EP_ERR_SHAPE, "ep_compress: empty tensor");
    if (!in->data) return set_error(EP_ERR_ARG, "ep_compress: NULL data");
    if (in->row_stride < in->cols) return set_error(EP_ERR_ARG, "ep_compress: row_stride < cols");
    // the documented range of target rates: finite, 0.001 to 11 bits per element
    if (!std::isfinite(target_bpp) || target_bpp < kTargetMin || target_bpp > kTargetMax)
        return set_error(EP_ERR_RANGE, "ep_compress: target_bpp must be finite and in [0.001, 11]");

    EncodeOptions o;
    bool host_encoder = false;
    if (opt) {
        if (opt->steps_per_tile < 0 || opt->steps_per_tile > 1024 || opt->num_threads < 0 ||
            !(opt->scale >= 0.0) || !std::isfinite(opt->scale) || (opt->prob_bits != 0 && !prob_bits_ok(opt->prob_bits)))
            return set_error(EP_ERR_ARG, "ep_compress: bad options");
        o.steps_per_tile = opt->steps_per_tile;
        o.threads = opt->num_threads;
        o.scale = opt->scale;
        o.rd_refine = opt->rd_refine != 0;
        o.prob_bits = opt->prob_bits ? opt->prob_bits : kProbBitsDefault;
        host_encoder = opt->host_encoder != 0;
    }
    // A device tensor is encoded on its GPU (same bytes), unless the refinement or the caller asks
    // for the host encoder; then it is copied to the host first.
    const bool on_gpu = in->device >= 0 && !o.rd_refine && !host_encoder;
    std::vector<uint8_t> host_copy;
    const void* src = in->data;
    int64_t stride = in->row_stride;
    if (in->device >= 0 && !on_gpu) {
        size_t row_bytes = size_t(in->cols) * es;
        try {
            host_copy.resize(row_bytes * size_t(in->rows));
        } catch (const std::bad_alloc&) {
            return set_error(EP_ERR_OOM, "ep_compress: host copy of the input");
        }
        int prev = 0;
        cudaGetDevice(&prev);
        cudaError_t e = cudaSetDevice(in->device);
        if (e == cudaSuccess)
            e = cudaMemcpy2D(host_copy.data(), row_bytes, in->data, size_t(in->row_stride) * es, row_bytes,
                             size_t(in->rows), cudaMemcpyDeviceToHost);
        cudaSetDevice(prev);
        if (e != cudaSuccess) return set_error(EP_ERR_CUDA, std::string("ep_compress: ") + cudaGetErrorString(e));
        src = host_copy.data();
        stride = in->cols;
    }

    ep_blob* b = new (std::nothrow) ep_blob();
    if (!b) return set_error(EP_ERR_OOM, "ep_compress: blob");
    std::string why;
    int rc;
    try {
        const EncodeInput ei{src, in->dtype, in->rows, in->cols, stride};
        if (on_gpu) {
            int prev = 0;
            cudaGetDevice(&prev);
            if (cudaSetDevice(in->device) != cudaSuccess) {
                delete b;
                return set_error(EP_ERR_ARG, "ep_compress: cannot use the tensor's device");
            }
            rc = encode_gpu(ei, target_bpp, o, b->bytes, why);
            cudaSetDevice(prev);
        } else {
            rc = encode(ei, target_bpp, o, b->bytes, why);
        }
    } catch (const std::bad_alloc&) {
        delete b;
        return set_error(EP_ERR_OOM, "ep_compress: out of host memory");
    }
    if (rc != 0) {
        delete b;
        const int code = rc == -4 ? EP_ERR_RANGE : rc == -6 ? EP_ERR_CUDA : rc == -7 ? EP_ERR_OOM : EP_ERR_SHAPE;
        return set_error(code, "ep_compress: " + why);
    }
    if (!parse_blob(b->bytes.data(), b->bytes.size(), b->layout, why)) {
        delete b;
        return set_error(EP_ERR_CORRUPT, "ep_compress produced an invalid blob: " + why);
    }
    *out = b;
    return EP_OK;
}

extern "C" int ep_compress(const ep_tensor* in, double target_bpp, ep_blob** out) {
    return ep_compress_ex(in, target_bpp, nullptr, out);
}

extern "C" double ep_actual_bpp(const ep_blob* b) {
    if (!b) return -1.0;
    return 8.0 * double(b->bytes.size()) / (double(b->layout.rows) * double(b->layout.cols));
}

extern "C" int ep_get_info(const ep_blob* b, ep_blob_info* info) {
    clear_error();
    if (!b || !info) return set_error(EP_ERR_ARG, "ep_get_info: NULL argument");
    const BlobLayout& L = b->layout;
    info->rows = L.rows;
    info->cols = L.cols;
    info->dtype = L.dtype;
    info->steps_per_tile = int(L.steps);
    info->n_tiles = L.n_tiles;
    info->n_vectors = L.n_vectors;
    info->scale = L.scale;
    info->bytes = b->bytes.size();
    info->prob_bits = L.prob_bits;
    return EP_OK;
}

extern "C" int ep_blob_to_bytes(const ep_blob* b, const uint8_t** data, size_t* n) {
    clear_error();
    if (!b || !data || !n) return set_error(EP_ERR_ARG, "ep_blob_to_bytes: NULL argument");
    *data = b->bytes.data();
    *n = b->bytes.size();
    return EP_OK;
}

extern "C" int ep_blob_from_bytes(const uint8_t* data, size_t n, ep_blob** out) {
    clear_error();
    if (!data || !out) return set_error(EP_ERR_ARG, "ep_blob_from_bytes: NULL argument");
    *out = nullptr;
    ep_blob* b = new (std::nothrow) ep_blob();
    if (!b) return set_error(EP_ERR_OOM, "ep_blob_from_bytes");
    try {
        b->bytes.assign(data, data + n);
    } catch (const std::bad_alloc&) {
        delete b;
        return set_error(EP_ERR_OOM, "ep_blob_from_bytes");
    }
    std::string why;
    if (!parse_blob(b->bytes.data(), n, b->layout, why)) {
        delete b;
        return set_error(EP_ERR_CORRUPT, "not a valid blob: " + why);
    }
    *out = b;
    return EP_OK;
}
