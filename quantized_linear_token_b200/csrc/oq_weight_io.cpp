// Prepared weights on disk: the codes and row norms that oq_weight_prepare
// writes (offline in the method: hotpaper.ai abstract, the rotation folded
// into the weight rows), saved with the layer settings they belong to so
// that a later process can load them into a layer built the same way and
// skip the preparation.
//
// File layout, little-endian:
//   offset  0  magic "OQWTS\0\0\0"                      8 bytes
//           8  format version (1)                       u32
//          12  d_in, d_out, a_bits, w_bits, flags       5 x i32
//          32  seed                                      u64
//          40  codebook hash                             u64 (FNV-1a 64 over the
//              bit patterns of both codebooks' levels and thresholds)
//          48  words per weight row (d_in w_bits / 32)   i64
//          56  r[d_out]                                  f32
//              Wcodes[d_out][words per row]              u32
// A load checks every header field against the layer (an INT4 weight-only
// layer has no codebooks and hashes to 0).
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "oq_internal.h"

namespace oq {
namespace {

constexpr char kMagic[8] = {'O', 'Q', 'W', 'T', 'S', 0, 0, 0};
constexpr uint32_t kVersion = 1;

struct Header {
  char magic[8];
  uint32_t version;
  int32_t d_in, d_out, a_bits, w_bits, flags;
  uint64_t seed;
  uint64_t cb_hash;
  int64_t words_per_row;
};
static_assert(sizeof(Header) == 56, "header layout");

uint64_t fnv1a(uint64_t h, const void* p, size_t n) {
  const unsigned char* b = static_cast<const unsigned char*>(p);
  for (size_t i = 0; i < n; ++i) {
    h ^= b[i];
    h *= 0x100000001B3ull;
  }
  return h;
}

uint64_t codebook_hash(const oq_layer* L) {
  if (L->int4_only) return 0;
  uint64_t h = 0xCBF29CE484222325ull;
  const oq_codebook* cbs[2] = {&L->cb_a, &L->cb_w};
  for (const oq_codebook* cb : cbs) {
    const int n = 1 << cb->bits;
    h = fnv1a(h, cb->levels, sizeof(double) * (size_t)n);
    h = fnv1a(h, cb->thresholds, sizeof(double) * (size_t)(n - 1));
  }
  return h;
}

Header header_of(const oq_layer* L) {
  Header h;
  std::memset(&h, 0, sizeof(h));
  std::memcpy(h.magic, kMagic, 8);
  h.version = kVersion;
  h.d_in = L->d_in;
  h.d_out = L->d_out;
  h.a_bits = L->a_bits;
  h.w_bits = L->w_bits;
  h.flags = L->flags;
  h.seed = L->seed;
  h.cb_hash = codebook_hash(L);
  h.words_per_row = (int64_t)L->d_in * L->w_bits / 32;
  return h;
}

oq_status fail(oq_status st, const std::string& msg) {
  set_error(msg);
  return st;
}

struct File {
  FILE* f = nullptr;
  ~File() {
    if (f) std::fclose(f);
  }
};

}  // namespace
}  // namespace oq

using namespace oq;

extern "C" {

oq_status oq_weight_save(const oq_layer* L, const uint32_t* Wcodes, const float* r, const char* path) {
  if (!L || !Wcodes || !r || !path) return fail(OQ_ERR_INVALID_ARG, "oq_weight_save: null argument");
  const Header h = header_of(L);
  std::vector<float> rh((size_t)L->d_out);
  std::vector<uint32_t> ch((size_t)L->d_out * (size_t)h.words_per_row);
  cudaError_t e = cudaMemcpy(rh.data(), r, rh.size() * sizeof(float), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(ch.data(), Wcodes, ch.size() * sizeof(uint32_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(OQ_ERR_CUDA, std::string("oq_weight_save: copy from the device: ") +
                                                     cudaGetErrorString(e));
  const std::string tmp = std::string(path) + ".tmp";
  File out;
  out.f = std::fopen(tmp.c_str(), "wb");
  if (!out.f) return fail(OQ_ERR_INVALID_ARG, std::string("oq_weight_save: cannot open ") + tmp);
  bool ok = std::fwrite(&h, sizeof(h), 1, out.f) == 1 && std::fwrite(rh.data(), sizeof(float), rh.size(), out.f) == rh.size() &&
            std::fwrite(ch.data(), sizeof(uint32_t), ch.size(), out.f) == ch.size();
  ok = (std::fclose(out.f) == 0) && ok;
  out.f = nullptr;
  if (!ok || std::rename(tmp.c_str(), path) != 0) {
    std::remove(tmp.c_str());
    return fail(OQ_ERR_INVALID_ARG, std::string("oq_weight_save: cannot write ") + path);
  }
  return OQ_OK;
}

oq_status oq_weight_load(const oq_layer* L, const char* path, uint32_t* Wcodes, float* r) {
  if (!L || !path) return fail(OQ_ERR_INVALID_ARG, "oq_weight_load: null argument");
  File in;
  in.f = std::fopen(path, "rb");
  if (!in.f) return fail(OQ_ERR_INVALID_ARG, std::string("oq_weight_load: cannot open ") + path);
  Header h;
  if (std::fread(&h, sizeof(h), 1, in.f) != 1 || std::memcmp(h.magic, kMagic, 8) != 0)
    return fail(OQ_ERR_INVALID_ARG, "oq_weight_load: not a prepared-weight file");
  if (h.version != kVersion) return fail(OQ_ERR_UNSUPPORTED, "oq_weight_load: unknown format version");
  const Header want = header_of(L);
  if (h.d_in != want.d_in || h.d_out != want.d_out || h.a_bits != want.a_bits || h.w_bits != want.w_bits ||
      h.flags != want.flags || h.seed != want.seed || h.words_per_row != want.words_per_row)
    return fail(OQ_ERR_INVALID_ARG, "oq_weight_load: the file was prepared for another layer (shape, bits, flags "
                                    "or seed differ)");
  if (h.cb_hash != want.cb_hash)
    return fail(OQ_ERR_INVALID_ARG, "oq_weight_load: the file's codebooks differ from the layer's");
  if (!Wcodes || !r) return fail(OQ_ERR_INVALID_ARG, "oq_weight_load: null Wcodes or r");
  std::vector<float> rh((size_t)h.d_out);
  std::vector<uint32_t> ch((size_t)h.d_out * (size_t)h.words_per_row);
  if (std::fread(rh.data(), sizeof(float), rh.size(), in.f) != rh.size() ||
      std::fread(ch.data(), sizeof(uint32_t), ch.size(), in.f) != ch.size())
    return fail(OQ_ERR_INVALID_ARG, "oq_weight_load: the file is truncated");
  if (std::fgetc(in.f) != EOF) return fail(OQ_ERR_INVALID_ARG, "oq_weight_load: trailing bytes after the weights");
  cudaError_t e = cudaMemcpy(r, rh.data(), rh.size() * sizeof(float), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(Wcodes, ch.data(), ch.size() * sizeof(uint32_t), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return fail(OQ_ERR_CUDA, std::string("oq_weight_load: copy to the device: ") +
                                                     cudaGetErrorString(e));
  return OQ_OK;
}

}  // extern "C"
