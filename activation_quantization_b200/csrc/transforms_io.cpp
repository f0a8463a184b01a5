// Checkpointing of calibrated transforms (host).
//
// WUSH news article, paragraph 6: the transforms are computed once from
// calibration moments, every block gets its own matrices and each of them costs
// extra storage (sharing among similar blocks reduces it).  These calls keep the
// calibration output so that inference can load it instead of recomputing.
//
// File layout (little-endian):
//   bytes  0..7   magic "WUSHTRF1"
//   u32           version (1)
//   u32           block size b
//   u32           transform kind (wush_transform)
//   u32           element type of the matrices (0 = fp32, the only one)
//   u32           moment normalisation the transforms were calibrated with
//                 (0 unknown, 1 means: Sigma_X / n_calib, Sigma_W / d_out)
//   u32           1 if a block -> transform index follows, else 0
//   i64           n_t, the number of transforms stored
//   i64           n_blocks, the number of d_in blocks they serve (n_t when no index)
//   f32 [n_t*b*b] T_X, then f32 [n_t*b*b] T_W, row-major per block
//   i32 [n_blocks] index (only when flagged)
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "wush.h"

namespace {

constexpr char kMagic[8] = {'W', 'U', 'S', 'H', 'T', 'R', 'F', '1'};
constexpr uint32_t kVersion = 1;

struct Header {
  char magic[8];
  uint32_t version, block, kind, dtype, sigma_norm, has_index;
  int64_t n_t, n_blocks;
};
static_assert(sizeof(Header) == 48, "packed header");

constexpr uint32_t kDtypeF32 = 0;

bool valid_shape(int block, int kind, int sigma_norm, int64_t n_t, int64_t n_blocks, bool has_index) {
  if (block < 2 || block > 256 || (block & (block - 1))) return false;
  if (kind < WUSH_T_IDENTITY || kind > WUSH_T_WUSH_DIAG) return false;
  if (sigma_norm < WUSH_NORM_UNKNOWN || sigma_norm > WUSH_NORM_MEAN) return false;
  if (n_t < 1 || n_blocks < 1 || n_t > (int64_t(1) << 32) || n_blocks > (int64_t(1) << 32)) return false;
  return has_index || n_t == n_blocks;
}

// Reads and checks the header, then checks that the file is exactly as long as the
// header says (so that a caller can size its buffers from the header safely), and
// leaves f positioned at the start of the body.
int read_header(FILE* f, Header* h) {
  if (std::fread(h, sizeof(Header), 1, f) != 1) return WUSH_ERR_IO;
  if (std::memcmp(h->magic, kMagic, 8) != 0 || h->version != kVersion || h->dtype != kDtypeF32)
    return WUSH_ERR_INVALID_ARG;
  if (h->has_index > 1 || !valid_shape(static_cast<int>(h->block), static_cast<int>(h->kind),
                                       static_cast<int>(h->sigma_norm), h->n_t, h->n_blocks, h->has_index != 0))
    return WUSH_ERR_INVALID_ARG;
  // at most 48 + 8 * 2^32 * 2^16 + 4 * 2^32 bytes: no overflow in 64 bits
  const int64_t want = static_cast<int64_t>(sizeof(Header)) + 8 * h->n_t * h->block * h->block +
                       (h->has_index ? 4 * h->n_blocks : 0);
  if (std::fseek(f, 0, SEEK_END) != 0) return WUSH_ERR_IO;
  const long have = std::ftell(f);
  if (have < 0 || std::fseek(f, static_cast<long>(sizeof(Header)), SEEK_SET) != 0) return WUSH_ERR_IO;
  return static_cast<int64_t>(have) == want ? WUSH_OK : WUSH_ERR_INVALID_ARG;
}

}  // namespace

extern "C" int wush_save_transforms(const char* path, int block, int kind, int sigma_norm, int64_t n_t,
                                    const float* t_x, const float* t_w, const int32_t* index, int64_t n_blocks) {
  if (!path || !t_x || !t_w) return WUSH_ERR_INVALID_ARG;
  const bool has_index = index != nullptr;
  if (!has_index) n_blocks = n_t;
  if (!valid_shape(block, kind, sigma_norm, n_t, n_blocks, has_index)) return WUSH_ERR_INVALID_ARG;
  if (has_index)
    for (int64_t j = 0; j < n_blocks; ++j)
      if (index[j] < 0 || index[j] >= n_t) return WUSH_ERR_INVALID_ARG;
  FILE* f = std::fopen(path, "wb");
  if (!f) return WUSH_ERR_IO;
  Header h;
  std::memcpy(h.magic, kMagic, 8);
  h.version = kVersion;
  h.block = static_cast<uint32_t>(block);
  h.kind = static_cast<uint32_t>(kind);
  h.dtype = kDtypeF32;
  h.sigma_norm = static_cast<uint32_t>(sigma_norm);
  h.has_index = has_index ? 1u : 0u;
  h.n_t = n_t;
  h.n_blocks = n_blocks;
  const size_t nt = static_cast<size_t>(n_t) * block * block;
  bool ok = std::fwrite(&h, sizeof(h), 1, f) == 1 && std::fwrite(t_x, sizeof(float), nt, f) == nt &&
            std::fwrite(t_w, sizeof(float), nt, f) == nt;
  if (ok && has_index)
    ok = std::fwrite(index, sizeof(int32_t), static_cast<size_t>(n_blocks), f) == static_cast<size_t>(n_blocks);
  ok = (std::fclose(f) == 0) && ok;
  return ok ? WUSH_OK : WUSH_ERR_IO;
}

extern "C" int wush_transforms_file_info(const char* path, int* block, int* kind, int* sigma_norm, int64_t* n_t,
                                         int64_t* n_blocks, int* has_index) {
  if (!path || !block || !kind || !sigma_norm || !n_t || !n_blocks || !has_index) return WUSH_ERR_INVALID_ARG;
  FILE* f = std::fopen(path, "rb");
  if (!f) return WUSH_ERR_IO;
  Header h;
  const int st = read_header(f, &h);
  std::fclose(f);
  if (st != WUSH_OK) return st;
  *block = static_cast<int>(h.block);
  *kind = static_cast<int>(h.kind);
  *sigma_norm = static_cast<int>(h.sigma_norm);
  *n_t = h.n_t;
  *n_blocks = h.n_blocks;
  *has_index = static_cast<int>(h.has_index);
  return WUSH_OK;
}

extern "C" int wush_load_transforms(const char* path, float* t_x, float* t_w, int64_t capacity_floats,
                                    int32_t* index, int64_t index_capacity) {
  if (!path || !t_x || !t_w) return WUSH_ERR_INVALID_ARG;
  FILE* f = std::fopen(path, "rb");
  if (!f) return WUSH_ERR_IO;
  Header h;
  int st = read_header(f, &h);
  const size_t nt = st == WUSH_OK ? static_cast<size_t>(h.n_t) * h.block * h.block : 0;
  if (st == WUSH_OK && static_cast<int64_t>(nt) > capacity_floats) st = WUSH_ERR_BUFFER_TOO_SMALL;
  if (st == WUSH_OK && h.has_index && (!index || h.n_blocks > index_capacity)) st = WUSH_ERR_BUFFER_TOO_SMALL;
  if (st == WUSH_OK) {
    bool ok = std::fread(t_x, sizeof(float), nt, f) == nt && std::fread(t_w, sizeof(float), nt, f) == nt;
    if (ok && h.has_index) {
      ok = std::fread(index, sizeof(int32_t), static_cast<size_t>(h.n_blocks), f) == static_cast<size_t>(h.n_blocks);
      for (int64_t j = 0; ok && j < h.n_blocks; ++j) ok = index[j] >= 0 && index[j] < h.n_t;
    }
    // nothing may follow the declared contents
    if (ok) ok = std::fgetc(f) == EOF;
    st = ok ? WUSH_OK : WUSH_ERR_INVALID_ARG;
  }
  std::fclose(f);
  return st;
}
