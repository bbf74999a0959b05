// Frozen kv-block lists on disk.
//
// "LoSA: Near-Lossless Sparse Attention for Training-Free Video Diffusion Acceleration",
// Abstract: the block indices selected at the calibration step are frozen and reused by
// every later step.  They are the method's only state, so a run that stops after the
// calibration can resume with the same lists from this file instead of calibrating again.
//
// Host code only.  File layout (little-endian):
//   [0, 8)    magic "BSALISTS"
//   [8, 12)   format version (1)
//   [12, 16)  header bytes (80)
//   [16, 60)  the bsa_shape the lists were selected for (11 int32)
//   [60, 64)  the retained-mass threshold (float32; informational)
//   [64, 72)  rows R (int64)
//   [72, 80)  entries nnz (int64)
//   [80, ...) row_ptr int32 [R + 1], then col_idx int32 [nnz]
//   last 8    FNV-1a 64-bit hash of every byte before it
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/bsattn.h"

namespace bsa {
bsa_status check_attention_shape(const bsa_shape* s);  // api.cu
}

namespace {

constexpr char kMagic[8] = {'B', 'S', 'A', 'L', 'I', 'S', 'T', 'S'};
constexpr uint32_t kVersion = 1;
constexpr uint32_t kHeaderBytes = 80;

// FNV-1a, 64-bit ("Fowler-Noll-Vo hash", offset basis and prime as published).
struct Fnv1a {
  uint64_t h = 1469598103934665603ull;
  void add(const void* p, size_t n) {
    const uint8_t* b = static_cast<const uint8_t*>(p);
    for (size_t i = 0; i < n; ++i) {
      h ^= b[i];
      h *= 1099511628211ull;
    }
  }
};

// The attention entry points' own shape check (every list file holds lists they accept).
bool shape_ok(const bsa_shape* s) { return bsa::check_attention_shape(s) == BSA_OK; }

long long rows_of(const bsa_shape* s) {
  return 1LL * s->batch * s->heads * (1LL * s->Tp * s->Hp * s->Wp / s->q_block);
}

long long kv_blocks_of(const bsa_shape* s) { return 1LL * s->Tp * s->Hp * s->Wp / 64; }

// The lists a selection produces: row_ptr from 0, non-decreasing, at most n_kb per row;
// each row's indices strictly ascending inside [0, n_kb).
bool lists_ok(long long rows, long long n_kb, const int32_t* row_ptr, const int32_t* col_idx) {
  if (row_ptr[0] != 0) return false;
  for (long long r = 0; r < rows; ++r) {
    const long long b = row_ptr[r], e = row_ptr[r + 1];
    if (e < b || e - b > n_kb) return false;
    for (long long i = b; i < e; ++i) {
      if (col_idx[i] < 0 || col_idx[i] >= n_kb) return false;
      if (i > b && col_idx[i] <= col_idx[i - 1]) return false;
    }
  }
  return true;
}

struct Header {
  bsa_shape shape;
  float threshold;
  int64_t rows, nnz;
};

void put_header(uint8_t* h, const Header& hd) {
  std::memcpy(h, kMagic, 8);
  std::memcpy(h + 8, &kVersion, 4);
  std::memcpy(h + 12, &kHeaderBytes, 4);
  std::memcpy(h + 16, &hd.shape, 44);
  std::memcpy(h + 60, &hd.threshold, 4);
  std::memcpy(h + 64, &hd.rows, 8);
  std::memcpy(h + 72, &hd.nnz, 8);
}

// Reads and checks the header; leaves the file positioned at row_ptr.
bsa_status get_header(FILE* f, Header* hd, Fnv1a* hash) {
  uint8_t h[kHeaderBytes];
  if (std::fread(h, 1, kHeaderBytes, f) != kHeaderBytes) return BSA_ERR_IO;
  uint32_t version = 0, hbytes = 0;
  std::memcpy(&version, h + 8, 4);
  std::memcpy(&hbytes, h + 12, 4);
  if (std::memcmp(h, kMagic, 8) != 0 || version != kVersion || hbytes != kHeaderBytes)
    return BSA_ERR_IO;
  std::memcpy(&hd->shape, h + 16, 44);
  std::memcpy(&hd->threshold, h + 60, 4);
  std::memcpy(&hd->rows, h + 64, 8);
  std::memcpy(&hd->nnz, h + 72, 8);
  if (!shape_ok(&hd->shape) || hd->rows != rows_of(&hd->shape) || hd->nnz < 0 ||
      hd->nnz > hd->rows * kv_blocks_of(&hd->shape))
    return BSA_ERR_IO;
  if (hash) hash->add(h, kHeaderBytes);
  return BSA_OK;
}

bool same_shape(const bsa_shape* a, const bsa_shape* b) {
  return std::memcmp(a, b, sizeof(bsa_shape)) == 0;
}

}  // namespace

extern "C" {

bsa_status bsa_lists_save(const char* path, const bsa_shape* shape, float threshold,
                          const int32_t* row_ptr, const int32_t* col_idx) {
  if (path == nullptr || shape == nullptr || row_ptr == nullptr) return BSA_ERR_INVALID_ARG;
  if (!shape_ok(shape)) return BSA_ERR_UNSUPPORTED;
  const long long rows = rows_of(shape), n_kb = kv_blocks_of(shape);
  const long long nnz = row_ptr[rows];
  if (nnz > 0 && col_idx == nullptr) return BSA_ERR_INVALID_ARG;
  if (nnz < 0 || nnz > rows * n_kb || !lists_ok(rows, n_kb, row_ptr, col_idx))
    return BSA_ERR_INVALID_ARG;
  Header hd;
  hd.shape = *shape;
  hd.threshold = threshold;
  hd.rows = rows;
  hd.nnz = nnz;
  uint8_t h[kHeaderBytes];
  put_header(h, hd);
  Fnv1a hash;
  hash.add(h, kHeaderBytes);
  hash.add(row_ptr, static_cast<size_t>(rows + 1) * 4);
  if (nnz > 0) hash.add(col_idx, static_cast<size_t>(nnz) * 4);
  // written under a temporary name and renamed, so a reader never sees half a file
  const std::string tmp = std::string(path) + ".tmp";
  FILE* f = std::fopen(tmp.c_str(), "wb");
  if (f == nullptr) return BSA_ERR_IO;
  bool ok = std::fwrite(h, 1, kHeaderBytes, f) == kHeaderBytes;
  ok = ok && std::fwrite(row_ptr, 4, static_cast<size_t>(rows + 1), f) == static_cast<size_t>(rows + 1);
  if (nnz > 0) ok = ok && std::fwrite(col_idx, 4, static_cast<size_t>(nnz), f) == static_cast<size_t>(nnz);
  ok = ok && std::fwrite(&hash.h, 8, 1, f) == 1;
  ok = (std::fclose(f) == 0) && ok;
  if (!ok || std::rename(tmp.c_str(), path) != 0) {
    std::remove(tmp.c_str());
    return BSA_ERR_IO;
  }
  return BSA_OK;
}

bsa_status bsa_lists_read_header(const char* path, bsa_shape* shape, float* threshold,
                                 int64_t* nnz) {
  if (path == nullptr) return BSA_ERR_INVALID_ARG;
  FILE* f = std::fopen(path, "rb");
  if (f == nullptr) return BSA_ERR_IO;
  Header hd;
  const bsa_status st = get_header(f, &hd, nullptr);
  std::fclose(f);
  if (st != BSA_OK) return st;
  if (shape) *shape = hd.shape;
  if (threshold) *threshold = hd.threshold;
  if (nnz) *nnz = hd.nnz;
  return BSA_OK;
}

bsa_status bsa_lists_load(const char* path, const bsa_shape* shape, float* threshold,
                          int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity) {
  if (path == nullptr || shape == nullptr || row_ptr == nullptr || col_capacity < 0)
    return BSA_ERR_INVALID_ARG;
  if (!shape_ok(shape)) return BSA_ERR_UNSUPPORTED;
  FILE* f = std::fopen(path, "rb");
  if (f == nullptr) return BSA_ERR_IO;
  Fnv1a hash;
  Header hd;
  bsa_status st = get_header(f, &hd, &hash);
  if (st == BSA_OK && !same_shape(&hd.shape, shape)) st = BSA_ERR_INVALID_ARG;
  if (st == BSA_OK && hd.nnz > col_capacity) st = BSA_ERR_CAPACITY;
  if (st == BSA_OK && hd.nnz > 0 && col_idx == nullptr) st = BSA_ERR_INVALID_ARG;
  // read into host staging first: the caller's buffers are written only for a good file
  std::vector<int32_t> rp, ci;
  uint64_t stored = 0;
  if (st == BSA_OK) {
    rp.resize(static_cast<size_t>(hd.rows + 1));
    ci.resize(static_cast<size_t>(hd.nnz));
    bool ok = std::fread(rp.data(), 4, rp.size(), f) == rp.size();
    ok = ok && (ci.empty() || std::fread(ci.data(), 4, ci.size(), f) == ci.size());
    ok = ok && std::fread(&stored, 8, 1, f) == 1;
    uint8_t extra;
    ok = ok && std::fread(&extra, 1, 1, f) == 0;  // nothing after the hash
    if (!ok) st = BSA_ERR_IO;
  }
  std::fclose(f);
  if (st != BSA_OK) return st;
  hash.add(rp.data(), rp.size() * 4);
  if (!ci.empty()) hash.add(ci.data(), ci.size() * 4);
  if (hash.h != stored || rp[hd.rows] != hd.nnz ||
      !lists_ok(hd.rows, kv_blocks_of(shape), rp.data(), ci.data()))
    return BSA_ERR_IO;
  std::memcpy(row_ptr, rp.data(), rp.size() * 4);
  if (!ci.empty()) std::memcpy(col_idx, ci.data(), ci.size() * 4);
  if (threshold) *threshold = hd.threshold;
  return BSA_OK;
}

}  // extern "C"
