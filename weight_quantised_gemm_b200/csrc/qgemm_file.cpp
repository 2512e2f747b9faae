// At-rest file format of a packed weight: the stored, still-quantised form of
// the weights (stable-diffusion.rs README, introduction, keeps weights packed
// when stored) written to and read from disk. Host-only; plain stdio.
//
// Layout, little-endian:
//   bytes 0-7    magic "QGEMMW01"
//   int32 x 4    N, K, bits, group
//   uint64 x 3   packed_bytes, scales_bytes, biases_bytes (as qgemm_pack_sizes)
//   the packed codes, then the fp16 scales, then the fp16 biases (if any)

#include <cstdio>
#include <cstring>

#include "qgemm.h"
#include "qgemm_internal.h"

namespace {

constexpr char kMagic[8] = {'Q', 'G', 'E', 'M', 'M', 'W', '0', '1'};

struct Header {
  char magic[8];
  int32_t N, K, bits, group;
  uint64_t packed_bytes, scales_bytes, biases_bytes;
};
static_assert(sizeof(Header) == 48, "header layout");

struct File {
  FILE* f;
  explicit File(FILE* fp) : f(fp) {}
  ~File() {
    if (f) std::fclose(f);
  }
};

int read_header(FILE* f, const char* path, Header* h) {
  if (std::fread(h, sizeof(Header), 1, f) != 1)
    return qg::fail(QGEMM_ERR_INVALID_ARG, "%s: too short for a qgemm weight header", path);
  if (std::memcmp(h->magic, kMagic, sizeof kMagic))
    return qg::fail(QGEMM_ERR_INVALID_ARG, "%s: not a qgemm weight file", path);
  size_t pb, sb, bb;
  const int st = qgemm_pack_sizes(h->N, h->K, h->bits, h->group, &pb, &sb, &bb);
  if (st != QGEMM_OK) return st;
  if (pb != h->packed_bytes || sb != h->scales_bytes || bb != h->biases_bytes)
    return qg::fail(QGEMM_ERR_INVALID_ARG, "%s: array sizes do not match N=%d K=%d bits=%d", path, h->N, h->K,
                    h->bits);
  // The file holds exactly the header and the three arrays: a short or
  // overlong file is refused here, before a caller sizes buffers from the
  // header or any array byte is copied out.
  if (std::fseek(f, 0, SEEK_END) != 0) return qg::fail(QGEMM_ERR_INVALID_ARG, "%s: cannot seek", path);
  const long end = std::ftell(f);
  if (end < 0 || std::fseek(f, static_cast<long>(sizeof(Header)), SEEK_SET) != 0)
    return qg::fail(QGEMM_ERR_INVALID_ARG, "%s: cannot seek", path);
  const unsigned long long want = sizeof(Header) + static_cast<unsigned long long>(pb) + sb + bb;
  if (static_cast<unsigned long long>(end) != want)
    return qg::fail(QGEMM_ERR_INVALID_ARG, "%s: %ld bytes, the header describes %llu", path, end, want);
  return QGEMM_OK;
}

}  // namespace

extern "C" int qgemm_save(const char* path, int32_t N, int32_t K, int32_t bits, int32_t group, const void* packed,
                          const void* scales, const void* biases) {
  if (!path) return qg::fail(QGEMM_ERR_INVALID_ARG, "null path");
  size_t pb, sb, bb;
  int st = qgemm_pack_sizes(N, K, bits, group, &pb, &sb, &bb);
  if (st != QGEMM_OK) return st;
  if (!packed || !scales || (bb && !biases)) return qg::fail(QGEMM_ERR_INVALID_ARG, "null buffer passed to qgemm_save");
  File file(std::fopen(path, "wb"));
  if (!file.f) return qg::fail(QGEMM_ERR_INVALID_ARG, "%s: cannot open for writing", path);
  Header h;
  std::memcpy(h.magic, kMagic, sizeof kMagic);
  h.N = N;
  h.K = K;
  h.bits = bits;
  h.group = group;
  h.packed_bytes = pb;
  h.scales_bytes = sb;
  h.biases_bytes = bb;
  if (std::fwrite(&h, sizeof h, 1, file.f) != 1 || std::fwrite(packed, 1, pb, file.f) != pb ||
      std::fwrite(scales, 1, sb, file.f) != sb || (bb && std::fwrite(biases, 1, bb, file.f) != bb))
    return qg::fail(QGEMM_ERR_INVALID_ARG, "%s: write failed", path);
  return QGEMM_OK;
}

extern "C" int qgemm_load_header(const char* path, int32_t* N, int32_t* K, int32_t* bits, int32_t* group) {
  if (!path || !N || !K || !bits || !group) return qg::fail(QGEMM_ERR_INVALID_ARG, "null argument");
  File file(std::fopen(path, "rb"));
  if (!file.f) return qg::fail(QGEMM_ERR_INVALID_ARG, "%s: cannot open for reading", path);
  Header h;
  const int st = read_header(file.f, path, &h);
  if (st != QGEMM_OK) return st;
  *N = h.N;
  *K = h.K;
  *bits = h.bits;
  *group = h.group;
  return QGEMM_OK;
}

extern "C" int qgemm_load(const char* path, void* packed, void* scales, void* biases) {
  if (!path || !packed || !scales) return qg::fail(QGEMM_ERR_INVALID_ARG, "null argument");
  File file(std::fopen(path, "rb"));
  if (!file.f) return qg::fail(QGEMM_ERR_INVALID_ARG, "%s: cannot open for reading", path);
  Header h;
  int st = read_header(file.f, path, &h);
  if (st != QGEMM_OK) return st;
  if (h.biases_bytes && !biases) return qg::fail(QGEMM_ERR_INVALID_ARG, "%s: the format has biases", path);
  if (std::fread(packed, 1, h.packed_bytes, file.f) != h.packed_bytes ||
      std::fread(scales, 1, h.scales_bytes, file.f) != h.scales_bytes ||
      (h.biases_bytes && std::fread(biases, 1, h.biases_bytes, file.f) != h.biases_bytes))
    return qg::fail(QGEMM_ERR_INVALID_ARG, "%s: truncated", path);
  if (std::fgetc(file.f) != EOF) return qg::fail(QGEMM_ERR_INVALID_ARG, "%s: trailing bytes after the arrays", path);
  return QGEMM_OK;
}
