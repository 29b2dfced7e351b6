// The int8 container as a file: the one stored artifact from which every
// width is served ("Matryoshka Quantization" explainer page, section 3.2: only
// the int8 model is kept; lower widths are sliced from it). Host-side I/O on
// host buffers; the caller moves device data.
//
// Layout, little-endian:
//   bytes 0..3    "MQC8"
//   bytes 4..7    format version (1)
//   bytes 8..15   N (int64), output channels
//   bytes 16..23  K (int64), input features
//   then          q, N*K uint8, row-major
//   then          alpha, N fp32
//   then          zero, N fp32
//   last 4 bytes  CRC-32 (IEEE 802.3 polynomial, reflected, 0xEDB88320) of all
//                 bytes before it
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <string>

#include <unistd.h>

#include "../../include/mq.h"
#include "mq_internal.h"

namespace mq {
namespace {

constexpr char kMagic[4] = {'M', 'Q', 'C', '8'};
constexpr uint32_t kVersion = 1;
constexpr int64_t kHeaderBytes = 24;

static_assert(sizeof(float) == 4, "fp32 layout");

// CRC-32 (reflected, polynomial 0xEDB88320), table built on first use.
struct Crc32 {
  uint32_t table[256];
  Crc32() {
    for (uint32_t i = 0; i < 256; ++i) {
      uint32_t c = i;
      for (int k = 0; k < 8; ++k) c = (c & 1u) ? (0xEDB88320u ^ (c >> 1)) : (c >> 1);
      table[i] = c;
    }
  }
  uint32_t update(uint32_t crc, const void* data, size_t n) const {
    const uint8_t* p = static_cast<const uint8_t*>(data);
    crc = ~crc;
    for (size_t i = 0; i < n; ++i) crc = table[(crc ^ p[i]) & 0xFFu] ^ (crc >> 8);
    return ~crc;
  }
};
const Crc32& crc_table() {
  static const Crc32 t;
  return t;
}

bool host_little_endian() {
  const uint32_t one = 1;
  uint8_t b;
  std::memcpy(&b, &one, 1);
  return b == 1;
}

struct File {
  std::FILE* f = nullptr;
  File(const char* path, const char* mode) : f(std::fopen(path, mode)) {}
  ~File() {
    if (f) std::fclose(f);
  }
};

}  // namespace

// Writes the whole file under a temporary name beside `path` (path.tmp.<pid>),
// closes it, and only then renames it over `path`: a reader sees the old file
// or the complete new one, never a partial write, and a failed save leaves
// `path` as it was.
int container_save(const char* path, const uint8_t* q, const float* alpha, const float* zero, int64_t N,
                   int64_t K, char* why, size_t why_len) {
  if (!host_little_endian()) { std::snprintf(why, why_len, "big-endian hosts are not supported"); return 1; }
  const std::string tmp = std::string(path) + ".tmp." + std::to_string(static_cast<long long>(getpid()));
  std::FILE* f = std::fopen(tmp.c_str(), "wb");
  if (!f) { std::snprintf(why, why_len, "cannot open %s for writing", tmp.c_str()); return 1; }
  const Crc32& T = crc_table();
  uint8_t header[kHeaderBytes];
  std::memcpy(header, kMagic, 4);
  std::memcpy(header + 4, &kVersion, 4);
  std::memcpy(header + 8, &N, 8);
  std::memcpy(header + 16, &K, 8);
  uint32_t crc = T.update(0, header, sizeof(header));
  bool ok = std::fwrite(header, 1, sizeof(header), f) == sizeof(header);
  const size_t nq = static_cast<size_t>(N) * static_cast<size_t>(K);
  ok = ok && std::fwrite(q, 1, nq, f) == nq;
  crc = T.update(crc, q, nq);
  ok = ok && std::fwrite(alpha, 4, static_cast<size_t>(N), f) == static_cast<size_t>(N);
  crc = T.update(crc, alpha, 4 * static_cast<size_t>(N));
  ok = ok && std::fwrite(zero, 4, static_cast<size_t>(N), f) == static_cast<size_t>(N);
  crc = T.update(crc, zero, 4 * static_cast<size_t>(N));
  ok = ok && std::fwrite(&crc, 4, 1, f) == 1;
  ok = ok && std::fflush(f) == 0;
  ok = (std::fclose(f) == 0) && ok;  // fclose reports errors of buffered writes too
  if (!ok) {
    std::remove(tmp.c_str());
    std::snprintf(why, why_len, "write to %s failed", tmp.c_str());
    return 1;
  }
  if (std::rename(tmp.c_str(), path) != 0) {
    std::remove(tmp.c_str());
    std::snprintf(why, why_len, "cannot rename %s to %s", tmp.c_str(), path);
    return 1;
  }
  return 0;
}

int container_info(const char* path, int64_t* N, int64_t* K, char* why, size_t why_len) {
  File fh(path, "rb");
  if (!fh.f) { std::snprintf(why, why_len, "cannot open %s", path); return 1; }
  uint8_t header[kHeaderBytes];
  if (std::fread(header, 1, sizeof(header), fh.f) != sizeof(header)) {
    std::snprintf(why, why_len, "%s: truncated header", path);
    return 1;
  }
  uint32_t version = 0;
  std::memcpy(&version, header + 4, 4);
  if (std::memcmp(header, kMagic, 4) != 0 || version != kVersion) {
    std::snprintf(why, why_len, "%s: not an int8 container file of version %u", path, kVersion);
    return 1;
  }
  std::memcpy(N, header + 8, 8);
  std::memcpy(K, header + 16, 8);
  if (*N < 1 || *K < 1 || *N > (int64_t(1) << 40) / *K) {
    std::snprintf(why, why_len, "%s: implausible shape", path);
    return 1;
  }
  return 0;
}

int container_load(const char* path, uint8_t* q, float* alpha, float* zero, int64_t N, int64_t K, char* why,
                   size_t why_len) {
  int64_t fn = 0, fk = 0;
  if (container_info(path, &fn, &fk, why, why_len) != 0) return 1;
  if (fn != N || fk != K) {
    std::snprintf(why, why_len, "%s holds %lld x %lld, not %lld x %lld", path, (long long)fn, (long long)fk,
                  (long long)N, (long long)K);
    return 2;
  }
  File fh(path, "rb");
  if (!fh.f) { std::snprintf(why, why_len, "cannot open %s", path); return 1; }
  const Crc32& T = crc_table();
  uint8_t header[kHeaderBytes];
  bool ok = std::fread(header, 1, sizeof(header), fh.f) == sizeof(header);
  uint32_t crc = T.update(0, header, sizeof(header));
  const size_t nq = static_cast<size_t>(N) * static_cast<size_t>(K);
  ok = ok && std::fread(q, 1, nq, fh.f) == nq;
  ok = ok && std::fread(alpha, 4, static_cast<size_t>(N), fh.f) == static_cast<size_t>(N);
  ok = ok && std::fread(zero, 4, static_cast<size_t>(N), fh.f) == static_cast<size_t>(N);
  uint32_t stored = 0;
  ok = ok && std::fread(&stored, 4, 1, fh.f) == 1;
  if (!ok) { std::snprintf(why, why_len, "%s: truncated", path); return 1; }
  uint8_t extra;
  if (std::fread(&extra, 1, 1, fh.f) != 0) { std::snprintf(why, why_len, "%s: trailing bytes", path); return 1; }
  crc = T.update(crc, q, nq);
  crc = T.update(crc, alpha, 4 * static_cast<size_t>(N));
  crc = T.update(crc, zero, 4 * static_cast<size_t>(N));
  if (crc != stored) { std::snprintf(why, why_len, "%s: checksum mismatch (corrupt file)", path); return 1; }
  return 0;
}

}  // namespace mq
