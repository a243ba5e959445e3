// Context checkpoints: a suspended context's host spans and metadata in one file, resumed
// without recomputation ("Context beyond VRAM", "What I built": a checkpointed context
// lifecycle).  Host code only.  Layout and refusal rules are stated in include/akv.h.
#include <cerrno>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "akv_internal.cuh"

namespace {

constexpr char kMagic[8] = {'A', 'K', 'V', 'C', 'K', 'P', 'T', '1'};
constexpr uint32_t kVersion = 1;
constexpr int kMaxCount = 1 << 20;

// CRC-32 of IEEE 802.3: reflected polynomial 0xEDB88320, initial value and final XOR
// 0xFFFFFFFF, one table lookup per byte.
struct Crc32 {
  uint32_t table[256];
  Crc32() {
    for (uint32_t n = 0; n < 256; ++n) {
      uint32_t c = n;
      for (int k = 0; k < 8; ++k) c = (c & 1u) ? 0xEDB88320u ^ (c >> 1) : c >> 1;
      table[n] = c;
    }
  }
  uint32_t update(uint32_t crc, const uint8_t* p, size_t n) const {
    for (size_t i = 0; i < n; ++i) crc = table[(crc ^ p[i]) & 0xFFu] ^ (crc >> 8);
    return crc;
  }
};

const Crc32& crc32() {
  static const Crc32 c;
  return c;
}

uint32_t crc_of(const void* p, uint64_t n) {
  return crc32().update(0xFFFFFFFFu, static_cast<const uint8_t*>(p), (size_t)n) ^ 0xFFFFFFFFu;
}

akv_status io_error(const char* what, const char* path) {
  char buf[600];
  std::snprintf(buf, sizeof(buf), "checkpoint %s %s: %s", what, path, std::strerror(errno));
  return akv::set_error(AKV_ERR_INVALID, buf);
}

akv_status refuse(const char* what, const char* path) {
  char buf[600];
  std::snprintf(buf, sizeof(buf), "checkpoint %s refused: %s", path, what);
  return akv::set_error(AKV_ERR_INVALID, buf);
}

struct Header {
  char magic[8];
  uint32_t version, n_meta, n_spans, zero;
};
struct SpanEntry {
  uint64_t bytes;
  uint32_t crc, zero;
};

// Reads the header, meta and span table of an open checkpoint file.
akv_status read_head(std::FILE* f, const char* path, Header& h, std::vector<uint64_t>& meta,
                     std::vector<SpanEntry>& spans) {
  if (std::fread(&h, sizeof(h), 1, f) != 1) return refuse("short header", path);
  if (std::memcmp(h.magic, kMagic, 8) != 0) return refuse("not a checkpoint (magic)", path);
  if (h.version != kVersion) return refuse("unknown version", path);
  if (h.n_meta > (uint32_t)kMaxCount || h.n_spans > (uint32_t)kMaxCount || h.zero != 0)
    return refuse("corrupt header", path);
  meta.resize(h.n_meta);
  spans.resize(h.n_spans);
  if (h.n_meta && std::fread(meta.data(), sizeof(uint64_t), h.n_meta, f) != h.n_meta)
    return refuse("short meta", path);
  if (h.n_spans && std::fread(spans.data(), sizeof(SpanEntry), h.n_spans, f) != h.n_spans)
    return refuse("short span table", path);
  for (const SpanEntry& e : spans)
    if (e.zero != 0) return refuse("corrupt span table", path);
  return AKV_OK;
}

}  // namespace

extern "C" {

akv_status akv_checkpoint_write(const char* path, const uint64_t* meta, int n_meta, const void* const* spans,
                                const uint64_t* span_bytes, int n_spans) {
  if (!path || !*path) return akv::set_error(AKV_ERR_INVALID, "checkpoint path is empty");
  if (n_meta < 0 || n_spans < 0 || n_meta > kMaxCount || n_spans > kMaxCount)
    return akv::set_error(AKV_ERR_INVALID, "checkpoint counts out of range");
  if ((n_meta && !meta) || (n_spans && (!spans || !span_bytes)))
    return akv::set_error(AKV_ERR_INVALID, "checkpoint arrays are null");
  for (int i = 0; i < n_spans; ++i)
    if (span_bytes[i] && !spans[i]) return akv::set_error(AKV_ERR_INVALID, "checkpoint span pointer is null");
  std::vector<SpanEntry> table(n_spans);
  for (int i = 0; i < n_spans; ++i) table[i] = SpanEntry{span_bytes[i], crc_of(spans[i], span_bytes[i]), 0};
  const std::string tmp = std::string(path) + ".tmp";
  std::FILE* f = std::fopen(tmp.c_str(), "wb");
  if (!f) return io_error("open", tmp.c_str());
  Header h;
  std::memcpy(h.magic, kMagic, 8);
  h.version = kVersion;
  h.n_meta = (uint32_t)n_meta;
  h.n_spans = (uint32_t)n_spans;
  h.zero = 0;
  bool good = std::fwrite(&h, sizeof(h), 1, f) == 1;
  good = good && (!n_meta || std::fwrite(meta, sizeof(uint64_t), n_meta, f) == (size_t)n_meta);
  good = good && (!n_spans || std::fwrite(table.data(), sizeof(SpanEntry), n_spans, f) == (size_t)n_spans);
  for (int i = 0; good && i < n_spans; ++i)
    good = !span_bytes[i] || std::fwrite(spans[i], 1, span_bytes[i], f) == span_bytes[i];
  good = (std::fflush(f) == 0) && good;
  if (std::fclose(f) != 0) good = false;
  if (!good) {
    akv_status s = io_error("write", tmp.c_str());
    std::remove(tmp.c_str());
    return s;
  }
  if (std::rename(tmp.c_str(), path) != 0) {
    akv_status s = io_error("rename onto", path);
    std::remove(tmp.c_str());
    return s;
  }
  return akv::set_error(AKV_OK, "");
}

akv_status akv_checkpoint_info(const char* path, uint64_t* meta, int* n_meta, uint64_t* span_bytes, int* n_spans) {
  if (!path || !n_meta || !n_spans) return akv::set_error(AKV_ERR_INVALID, "checkpoint info: null argument");
  if (*n_meta < 0 || *n_spans < 0) return akv::set_error(AKV_ERR_INVALID, "checkpoint info: negative capacity");
  std::FILE* f = std::fopen(path, "rb");
  if (!f) return io_error("open", path);
  Header h;
  std::vector<uint64_t> m;
  std::vector<SpanEntry> t;
  akv_status s = read_head(f, path, h, m, t);
  std::fclose(f);
  if (s != AKV_OK) return s;
  for (int i = 0; i < *n_meta && i < (int)h.n_meta; ++i) meta[i] = m[i];
  for (int i = 0; i < *n_spans && i < (int)h.n_spans; ++i) span_bytes[i] = t[i].bytes;
  *n_meta = (int)h.n_meta;
  *n_spans = (int)h.n_spans;
  return akv::set_error(AKV_OK, "");
}

akv_status akv_checkpoint_read(const char* path, void* const* spans, const uint64_t* span_bytes, int n_spans) {
  if (!path || n_spans < 0 || (n_spans && (!spans || !span_bytes)))
    return akv::set_error(AKV_ERR_INVALID, "checkpoint read: null or negative argument");
  std::FILE* f = std::fopen(path, "rb");
  if (!f) return io_error("open", path);
  Header h;
  std::vector<uint64_t> m;
  std::vector<SpanEntry> t;
  akv_status s = read_head(f, path, h, m, t);
  if (s == AKV_OK && (int)h.n_spans != n_spans) s = refuse("span count differs from the caller's", path);
  for (int i = 0; s == AKV_OK && i < n_spans; ++i) {
    if (t[i].bytes != span_bytes[i]) s = refuse("span size differs from the caller's buffer", path);
    else if (span_bytes[i] && !spans[i]) s = akv::set_error(AKV_ERR_INVALID, "checkpoint read: null buffer");
    else if (span_bytes[i] && std::fread(spans[i], 1, span_bytes[i], f) != span_bytes[i]) s = refuse("truncated", path);
    else if (crc_of(spans[i], span_bytes[i]) != t[i].crc) s = refuse("CRC-32 mismatch", path);
  }
  if (s == AKV_OK && std::fgetc(f) != EOF) s = refuse("trailing bytes", path);
  std::fclose(f);
  return s == AKV_OK ? akv::set_error(AKV_OK, "") : s;
}

}  // extern "C"
