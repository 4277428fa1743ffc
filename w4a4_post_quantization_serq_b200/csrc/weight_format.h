// Host-side helpers of the prepared-weight checkpoint (serq_weight_save /
// serq_weight_load / serq_weight_file_*): the canonical sizes of each part,
// the E8M0 scale-atom <-> row-major conversion, the file header and its
// checksum. Plain C++; no CUDA.
//
// The artefact SERQ produces offline is the permuted, folded and quantized
// linear (reading notes Stage 3, gist.science/zh 2.3: the permutation and
// 1/s are merged into the weights ahead of time, so they cost nothing at run
// time). A checkpoint stores exactly that artefact in its canonical host form:
//   perm int32[K], s fp32[K], inv_s fp32[K], wq u8[N][K/2],
//   w_scale (INT4 weights fp32[N]; MXFP4 E8M0 u8[N][K/32]), rq u8[N][rp/2],
//   r_scale (INT4 weights fp32[N]; MXFP4 E8M0 u8[N][rp/32])
// in that order after a 64-byte header. Multi-byte fields are little-endian
// (the byte order of every host this library builds for).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cstring>

namespace serq {
namespace wfmt {

constexpr char kMagic[8] = {'S', 'E', 'R', 'Q', 'W', 'G', 'T', '\0'};
constexpr uint32_t kVersion = 1;
constexpr size_t kHeaderBytes = 64;

struct Header {            // the first 64 bytes of a checkpoint file
    char magic[8];
    uint32_t version;
    int32_t fmt, K, N, r, rp;
    uint64_t payload_bytes;
    uint64_t checksum;     // FNV-1a 64 over the payload bytes
    uint8_t reserved[16];
};
static_assert(sizeof(Header) == kHeaderBytes, "checkpoint header must be 64 bytes");

// Byte sizes of the canonical parts (fmt 0 = INT4, 1 = MXFP4, 2 = W4A8: INT4 weights).
struct Sizes {
    size_t perm, s, inv_s, wq, w_scale, rq, r_scale;
    size_t total() const { return perm + s + inv_s + wq + w_scale + rq + r_scale; }
};

inline Sizes canonical_sizes(int fmt, int K, int N, int rp) {
    Sizes z;
    z.perm = 4u * static_cast<size_t>(K);
    z.s = z.perm;
    z.inv_s = z.perm;
    z.wq = static_cast<size_t>(N) * (K / 2);
    z.rq = static_cast<size_t>(N) * (rp / 2);
    if (fmt != 1) {
        z.w_scale = 4u * static_cast<size_t>(N);
        z.r_scale = 4u * static_cast<size_t>(N);
    } else {
        z.w_scale = static_cast<size_t>(N) * (K / 32);
        z.r_scale = static_cast<size_t>(N) * (rp / 32);
    }
    return z;
}

inline uint64_t fnv1a64(const uint8_t* p, size_t n, uint64_t h = 1469598103934665603ull) {
    for (size_t i = 0; i < n; ++i) {
        h ^= p[i];
        h *= 1099511628211ull;
    }
    return h;
}

// Offset of E8M0 byte (row, block) in the scale-atom layout of a tensor with
// `nblk` blocks per row: atoms of 128 rows x 4 blocks (512 B), the layout the
// block-scaled tensor cores read.
inline size_t atom_offset(int row, int block, int nblk) {
    const size_t atoms_k = static_cast<size_t>((nblk + 3) / 4);
    return ((static_cast<size_t>(row / 128) * atoms_k + block / 4) * 512) + static_cast<size_t>(row % 32) * 16 +
           static_cast<size_t>((row % 128) / 32) * 4 + static_cast<size_t>(block % 4);
}

inline size_t atom_bytes(int rows, int nblk) {
    return static_cast<size_t>((rows + 127) / 128) * static_cast<size_t>((nblk + 3) / 4) * 512u;
}

// atoms (atom_bytes(rows, nblk)) -> row-major [rows][nblk]
inline void atoms_to_rows(const uint8_t* atoms, int rows, int nblk, uint8_t* dst) {
    for (int r = 0; r < rows; ++r)
        for (int b = 0; b < nblk; ++b) dst[static_cast<size_t>(r) * nblk + b] = atoms[atom_offset(r, b, nblk)];
}

// row-major [rows][nblk] -> atoms; bytes of padding rows / blocks are zero
inline void rows_to_atoms(const uint8_t* src, int rows, int nblk, uint8_t* atoms) {
    std::memset(atoms, 0, atom_bytes(rows, nblk));
    for (int r = 0; r < rows; ++r)
        for (int b = 0; b < nblk; ++b) atoms[atom_offset(r, b, nblk)] = src[static_cast<size_t>(r) * nblk + b];
}

}  // namespace wfmt
}  // namespace serq
