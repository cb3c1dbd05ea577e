// glq_handles.h -- the opaque handle types of the C ABI (include/glq.h):
// what a codebook and a layer own on the host and on the device.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include <vector>

#include "../../include/glq.h"
#include "glq_codebook_host.h"
#include "glq_internal.h"

struct glq_codebook_s {
    std::vector<uint16_t> host;  // fp16 bits (256-entry tables)
    int entries = 0;
    int device = 0;
    uint16_t *d_fp16 = nullptr;  // [entries][8]
    bool folded = false;
    glq::FoldedTable fold;
    uint32_t *d_table = nullptr;  // table_words words
    int table_words = 0;          // nb rounded up to a multiple of 4
};

struct glq_layer_s {
    int64_t m = 0, n = 0, m_pad = 0, n_pad = 0;
    int bpw = 0, RT = 0, KC = 0, G = 0;
    int device = 0, num_sms = 0;
    glq_codebook primary = nullptr, residual = nullptr;
    float ws = 0.f, rs = 0.f;
    uint4 *d_idx1 = nullptr;
    void *d_idx2 = nullptr;
    size_t idx1_bytes = 0, idx2_bytes = 0;
    uint32_t *d_sin = nullptr, *d_sout = nullptr;
    uint16_t *d_r8 = nullptr;  // 3 bpw residual table, columns 2,3,6,7 x 16
    glq_blocks bn{}, bm{};
    unsigned *d_err = nullptr;
    // GEMV work split
    int bands = 0, splits = 0, cps = 0, grid = 0;
    // workspace
    int64_t cap_rows = 0;  // rows of xr / info
    int64_t last_B = 0;    // batch of the last decode slice (glq_gemv_replay)
    __half *d_xr = nullptr;
    glq_rowinfo *d_info = nullptr;
    float *d_part = nullptr;
    size_t device_bytes = 0;
};

