// entro_internal.h -- library-internal types shared by the host encoder and
// the CUDA launch code.  Not part of the C ABI.
#pragma once
#include <stdint.h>

#include <vector>

#include "blob_format.h"

namespace entro {

struct Blob {
    std::vector<uint8_t> bytes;  // serialized blob
    BlobHeader header{};
    uint8_t lengths[256]{};
    uint64_t max_chunk_words = 0;  // lanes: longest lane (words); single: most words one chunk spans
    uint64_t coded_bits = 0;
    int finalize_info();  // parse + validate bytes, fill the fields above
};

int code_lengths(const int64_t *hist, int nsym, int max_len, uint8_t *len);
void canonical_codes(const uint8_t *len, uint32_t *code);

}  // namespace entro
