// mobi_ckpt.cu — many-in-one checkpoints of packed MoBiSlice layers (host code).
//
// One file keeps every slice of every layer once ([ja] §2.1: a single
// decomposition serves all precisions; [en] §3: many-in-one storage, fetching
// only the slices a precision needs). Codes and scale/zero words are stored
// slice-major exactly as mobi_pack writes them, so a load at k slices reads a
// prefix of each block and lands as a packed array with S = k. The format is
// stated in include/mobi.h.
//
// Device loads stream the file through two pinned staging buffers: while one
// buffer's host-to-device copy runs on the caller's stream the next chunk is
// read into the other, and each slice's CRC-32C is updated as its bytes pass.
#include <cuda_runtime.h>
#include <fcntl.h>
#include <sys/stat.h>
#include <unistd.h>

#include <cerrno>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/mobi.h"
#include "mobi_host.h"

namespace mobi {
namespace ckpt {

constexpr char kMagic[8] = {'M', 'O', 'B', 'I', 'C', 'K', 'P', 'T'};
constexpr uint32_t kVersion = 1;
constexpr size_t kHeaderBytes = 64;
constexpr size_t kEntryBytes = 192;
constexpr size_t kNameBytes = 96;
constexpr uint64_t kAlign = 4096;
constexpr size_t kStageBytes = size_t(16) << 20;  // per pinned staging buffer

constexpr int64_t kMaxCkptDim = int64_t(1) << 28;  // largest N or K of a stored tensor (as the GEMM)

struct Entry {
  char name[kNameBytes];
  int64_t N, K;
  int32_t G, S;
  uint64_t codes_off, codes_slice;
  uint64_t sz_off, sz_slice;
  uint32_t crc_codes[kMaxSlices], crc_sz[kMaxSlices];
};
static_assert(sizeof(Entry) <= kEntryBytes, "table entry fits its 192 bytes");

// ---- CRC-32C (Castagnoli), reflected polynomial 0x82F63B78 ------------------------------
//
// Hardware crc32 instructions on x86-64 with SSE4.2 (eight bytes per step),
// else a byte-wise table built from the polynomial.
[[maybe_unused]] static uint32_t g_table[256];
[[maybe_unused]] static bool g_table_ready = false;

[[maybe_unused]] static void build_table() {
  for (uint32_t i = 0; i < 256; ++i) {
    uint32_t c = i;
    for (int k = 0; k < 8; ++k) c = (c & 1u) ? (c >> 1) ^ 0x82F63B78u : c >> 1;
    g_table[i] = c;
  }
  g_table_ready = true;
}

static uint32_t crc_update(uint32_t state, const uint8_t* p, size_t n) {
#if defined(__x86_64__) && defined(__SSE4_2__)
  uint64_t c = state;
  while (n >= 8) {
    uint64_t v;
    memcpy(&v, p, 8);
    c = __builtin_ia32_crc32di(c, v);
    p += 8;
    n -= 8;
  }
  uint32_t c32 = (uint32_t)c;
  while (n--) c32 = __builtin_ia32_crc32qi(c32, *p++);
  return c32;
#else
  if (!g_table_ready) build_table();
  while (n--) state = g_table[(state ^ *p++) & 0xFFu] ^ (state >> 8);
  return state;
#endif
}

// ---- files ------------------------------------------------------------------------------

static bool pwrite_all(int fd, const void* buf, size_t n, uint64_t off) {
  const uint8_t* p = static_cast<const uint8_t*>(buf);
  while (n > 0) {
    const ssize_t w = pwrite(fd, p, n, (off_t)off);
    if (w < 0 && errno == EINTR) continue;
    if (w <= 0) return false;
    p += w;
    n -= (size_t)w;
    off += (uint64_t)w;
  }
  return true;
}

static bool pread_all(int fd, void* buf, size_t n, uint64_t off) {
  uint8_t* p = static_cast<uint8_t*>(buf);
  while (n > 0) {
    const ssize_t r = pread(fd, p, n, (off_t)off);
    if (r < 0 && errno == EINTR) continue;
    if (r <= 0) return false;
    p += r;
    n -= (size_t)r;
    off += (uint64_t)r;
  }
  return true;
}

static uint64_t align_up(uint64_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

// Pinned staging buffers (lazily allocated; a reader or a save owns its pair).
struct Staging {
  void* buf[2] = {nullptr, nullptr};
  cudaEvent_t done[2] = {nullptr, nullptr};
  bool ready = false;
  cudaError_t init() {
    if (ready) return cudaSuccess;
    for (int i = 0; i < 2; ++i) {
      cudaError_t e = cudaHostAlloc(&buf[i], kStageBytes, cudaHostAllocDefault);
      if (e != cudaSuccess) return note_error("cudaHostAlloc (checkpoint staging)", e);
      e = cudaEventCreateWithFlags(&done[i], cudaEventDisableTiming);
      if (e != cudaSuccess) return note_error("cudaEventCreate (checkpoint staging)", e);
    }
    ready = true;
    return cudaSuccess;
  }
  ~Staging() {
    for (int i = 0; i < 2; ++i) {
      if (done[i]) cudaEventDestroy(done[i]);
      if (buf[i]) cudaFreeHost(buf[i]);
    }
  }
};

}  // namespace ckpt
}  // namespace mobi

struct mobi_ckpt {
  int fd = -1;
  std::string path;
  std::vector<mobi::ckpt::Entry> entries;
  mobi::ckpt::Staging staging;
  int64_t bytes_read = 0;
};

using namespace mobi;
using namespace mobi::ckpt;

namespace {

mobi_status io_error(const char* what, const std::string& path) {
  char msg[512];
  snprintf(msg, sizeof msg, "%s: %s (%s)", what, path.c_str(), errno ? strerror(errno) : "format");
  note_message(msg);
  return MOBI_ERR_IO;
}

bool valid_tensor(const mobi_ckpt_tensor& t) {
  if (!t.name || !t.codes || !t.sz) return false;
  const size_t len = strnlen(t.name, kNameBytes);
  if (len == 0 || len >= kNameBytes) return false;
  if (t.N <= 0 || t.K <= 0 || t.G <= 0 || t.K % t.G != 0 || t.K % 16 != 0) return false;
  if (t.S < 1 || t.S > kMaxSlices) return false;
  return true;
}

// Copy `n` bytes of one block (host or device memory) to the file at `off`,
// updating `crc`. Device blocks go through the pinned staging buffers.
mobi_status write_block(int fd, const void* src, uint64_t n, uint64_t off, bool host, Staging& st, cudaStream_t s,
                        uint32_t* crc, const std::string& path) {
  uint32_t c = 0xFFFFFFFFu;
  const uint8_t* p = static_cast<const uint8_t*>(src);
  for (uint64_t done = 0; done < n;) {
    const size_t len = (size_t)(n - done < kStageBytes ? n - done : kStageBytes);
    const uint8_t* chunk = p + done;
    if (!host) {
      cudaError_t e = cudaMemcpyAsync(st.buf[0], chunk, len, cudaMemcpyDeviceToHost, s);
      if (e == cudaSuccess) e = cudaStreamSynchronize(s);
      if (e != cudaSuccess) {
        note_error("checkpoint device-to-host copy", e);
        return MOBI_ERR_CUDA;
      }
      chunk = static_cast<const uint8_t*>(st.buf[0]);
    }
    c = crc_update(c, chunk, len);
    if (!pwrite_all(fd, chunk, len, off + done)) return io_error("write failed", path);
    done += len;
  }
  *crc = c ^ 0xFFFFFFFFu;
  return MOBI_OK;
}

}  // namespace

extern "C" {

uint32_t mobi_crc32c(uint32_t crc, const void* data, size_t n) {
  if (!data || n == 0) return crc;
  return crc_update(crc ^ 0xFFFFFFFFu, static_cast<const uint8_t*>(data), n) ^ 0xFFFFFFFFu;
}

mobi_status mobi_ckpt_save(const char* path, const mobi_ckpt_tensor* tensors, int count, int host_ptrs,
                           void* stream) {
  if (!path || !tensors || count < 1) return MOBI_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    if (!valid_tensor(tensors[i])) return MOBI_ERR_INVALID_ARG;
    for (int j = 0; j < i; ++j)
      if (strcmp(tensors[i].name, tensors[j].name) == 0) return MOBI_ERR_INVALID_ARG;
  }
  // Layout: header, table, then each tensor's codes and sz blocks on 4 KB boundaries.
  std::vector<Entry> entries((size_t)count);
  uint64_t off = align_up(kHeaderBytes + (uint64_t)count * kEntryBytes);
  for (int i = 0; i < count; ++i) {
    const mobi_ckpt_tensor& t = tensors[i];
    Entry& e = entries[(size_t)i];
    memset(&e, 0, sizeof e);
    strncpy(e.name, t.name, kNameBytes - 1);
    e.N = t.N;
    e.K = t.K;
    e.G = t.G;
    e.S = t.S;
    e.codes_slice = (uint64_t)t.N * (uint64_t)t.K / 4;
    e.sz_slice = (uint64_t)(t.K / t.G) * (uint64_t)t.N * 4;
    e.codes_off = off;
    off = align_up(off + e.codes_slice * (uint64_t)t.S);
    e.sz_off = off;
    off = align_up(off + e.sz_slice * (uint64_t)t.S);
  }
  const std::string final_path(path);
  const std::string tmp = final_path + ".tmp" + std::to_string((long)getpid());
  const int fd = open(tmp.c_str(), O_WRONLY | O_CREAT | O_TRUNC, 0644);
  if (fd < 0) return io_error("cannot create", tmp);
  Staging st;
  mobi_status status = MOBI_OK;
  if (!host_ptrs && st.init() != cudaSuccess) status = MOBI_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int i = 0; i < count && status == MOBI_OK; ++i) {
    const mobi_ckpt_tensor& t = tensors[i];
    Entry& e = entries[(size_t)i];
    for (int sl = 0; sl < t.S && status == MOBI_OK; ++sl) {
      status = write_block(fd, reinterpret_cast<const uint8_t*>(t.codes) + e.codes_slice * sl, e.codes_slice,
                           e.codes_off + e.codes_slice * sl, host_ptrs != 0, st, s, &e.crc_codes[sl], tmp);
      if (status == MOBI_OK)
        status = write_block(fd, reinterpret_cast<const uint8_t*>(t.sz) + e.sz_slice * sl, e.sz_slice,
                             e.sz_off + e.sz_slice * sl, host_ptrs != 0, st, s, &e.crc_sz[sl], tmp);
    }
  }
  if (status == MOBI_OK) {
    std::vector<uint8_t> table((size_t)count * kEntryBytes, 0);
    for (int i = 0; i < count; ++i) memcpy(table.data() + (size_t)i * kEntryBytes, &entries[(size_t)i], sizeof(Entry));
    uint8_t hdr[kHeaderBytes] = {0};
    memcpy(hdr, kMagic, 8);
    const uint32_t ver = kVersion, cnt = (uint32_t)count;
    const uint64_t toff = kHeaderBytes, tbytes = table.size();
    const uint32_t tcrc = mobi_crc32c(0, table.data(), table.size());
    memcpy(hdr + 8, &ver, 4);
    memcpy(hdr + 12, &cnt, 4);
    memcpy(hdr + 16, &toff, 8);
    memcpy(hdr + 24, &tbytes, 8);
    memcpy(hdr + 32, &tcrc, 4);
    if (!pwrite_all(fd, table.data(), table.size(), toff) || !pwrite_all(fd, hdr, kHeaderBytes, 0) ||
        ftruncate(fd, (off_t)off) != 0 || fsync(fd) != 0)
      status = io_error("write failed", tmp);
  }
  if (close(fd) != 0 && status == MOBI_OK) status = io_error("close failed", tmp);
  if (status == MOBI_OK && rename(tmp.c_str(), final_path.c_str()) != 0) status = io_error("rename failed", tmp);
  if (status != MOBI_OK) unlink(tmp.c_str());
  return status;
}

mobi_status mobi_ckpt_open(const char* path, mobi_ckpt** out) {
  if (!path || !out) return MOBI_ERR_INVALID_ARG;
  *out = nullptr;
  errno = 0;
  const int fd = open(path, O_RDONLY);
  if (fd < 0) return io_error("cannot open", path);
  auto fail = [&](const char* what) {
    const mobi_status st = io_error(what, path);
    close(fd);
    return st;
  };
  struct stat sb;
  if (fstat(fd, &sb) != 0) return fail("stat failed");
  const uint64_t fsize = (uint64_t)sb.st_size;
  uint8_t hdr[kHeaderBytes];
  errno = 0;
  if (fsize < kHeaderBytes || !pread_all(fd, hdr, kHeaderBytes, 0)) return fail("truncated header");
  if (memcmp(hdr, kMagic, 8) != 0) return fail("not a MoBiQuant checkpoint");
  uint32_t ver, cnt, tcrc;
  uint64_t toff, tbytes;
  memcpy(&ver, hdr + 8, 4);
  memcpy(&cnt, hdr + 12, 4);
  memcpy(&toff, hdr + 16, 8);
  memcpy(&tbytes, hdr + 24, 8);
  memcpy(&tcrc, hdr + 32, 4);
  if (ver != kVersion) return fail("unsupported checkpoint version");
  if (cnt == 0 || cnt > (1u << 20) || tbytes != (uint64_t)cnt * kEntryBytes || toff < kHeaderBytes ||
      toff > fsize || tbytes > fsize - toff)
    return fail("corrupt table header");
  std::vector<uint8_t> table((size_t)tbytes);
  if (!pread_all(fd, table.data(), table.size(), toff)) return fail("truncated table");
  if (mobi_crc32c(0, table.data(), table.size()) != tcrc) return fail("table checksum mismatch");
  mobi_ckpt* c = new mobi_ckpt();
  c->fd = fd;
  c->path = path;
  c->entries.resize(cnt);
  for (uint32_t i = 0; i < cnt; ++i) {
    Entry& e = c->entries[i];
    memcpy(&e, table.data() + (size_t)i * kEntryBytes, sizeof(Entry));
    e.name[kNameBytes - 1] = 0;
    // Sizes bounded as for the GEMM (N, K <= 2^28), so the products below stay
    // under 2^59; offsets are compared by subtraction, so nothing can wrap.
    const bool dims_ok = e.N > 0 && e.K > 0 && e.N <= kMaxCkptDim && e.K <= kMaxCkptDim && e.G > 0 &&
                         e.K % e.G == 0 && e.S >= 1 && e.S <= kMaxSlices;
    const bool ok = dims_ok && e.codes_slice == (uint64_t)e.N * (uint64_t)e.K / 4 &&
                    e.sz_slice == (uint64_t)(e.K / e.G) * (uint64_t)e.N * 4 && e.codes_off <= fsize &&
                    e.codes_slice * (uint64_t)e.S <= fsize - e.codes_off && e.sz_off <= fsize &&
                    e.sz_slice * (uint64_t)e.S <= fsize - e.sz_off;
    if (!ok) {
      delete c;
      return fail("corrupt table entry");
    }
  }
  *out = c;
  return MOBI_OK;
}

int mobi_ckpt_count(const mobi_ckpt* c) { return c ? (int)c->entries.size() : -1; }

int mobi_ckpt_find(const mobi_ckpt* c, const char* name) {
  if (!c || !name) return -1;
  for (size_t i = 0; i < c->entries.size(); ++i)
    if (strncmp(c->entries[i].name, name, kNameBytes) == 0) return (int)i;
  return -1;
}

mobi_status mobi_ckpt_info(const mobi_ckpt* c, int index, const char** name, int64_t* N, int64_t* K, int* G,
                           int* S) {
  if (!c || index < 0 || index >= (int)c->entries.size()) return MOBI_ERR_INVALID_ARG;
  const Entry& e = c->entries[(size_t)index];
  if (name) *name = e.name;
  if (N) *N = e.N;
  if (K) *K = e.K;
  if (G) *G = e.G;
  if (S) *S = e.S;
  return MOBI_OK;
}

int64_t mobi_ckpt_bytes_read(const mobi_ckpt* c) { return c ? c->bytes_read : -1; }

mobi_status mobi_ckpt_load(mobi_ckpt* c, int index, int slices, uint32_t* codes, uint32_t* sz, int host_ptrs,
                           int verify, void* stream) {
  if (!c || index < 0 || index >= (int)c->entries.size() || !codes || !sz) return MOBI_ERR_INVALID_ARG;
  const Entry& e = c->entries[(size_t)index];
  if (slices < 1 || slices > e.S) return MOBI_ERR_INVALID_ARG;
  if (!host_ptrs && c->staging.init() != cudaSuccess) return MOBI_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  struct Block {
    uint64_t off, n;
    uint8_t* dst;
    uint32_t crc;
  };
  std::vector<Block> blocks;
  for (int sl = 0; sl < slices; ++sl)
    blocks.push_back({e.codes_off + e.codes_slice * sl, e.codes_slice,
                      reinterpret_cast<uint8_t*>(codes) + e.codes_slice * sl, e.crc_codes[sl]});
  for (int sl = 0; sl < slices; ++sl)
    blocks.push_back({e.sz_off + e.sz_slice * sl, e.sz_slice, reinterpret_cast<uint8_t*>(sz) + e.sz_slice * sl,
                      e.crc_sz[sl]});
  int cur = 0;  // staging buffer for the next chunk
  bool pending[2] = {false, false};
  for (const Block& b : blocks) {
    uint32_t crc = 0xFFFFFFFFu;
    for (uint64_t done = 0; done < b.n;) {
      const size_t len = (size_t)(b.n - done < kStageBytes ? b.n - done : kStageBytes);
      uint8_t* dst = b.dst + done;
      uint8_t* buf = host_ptrs ? dst : static_cast<uint8_t*>(c->staging.buf[cur]);
      if (!host_ptrs && pending[cur]) {  // the copy out of this buffer must have finished
        const cudaError_t ce = cudaEventSynchronize(c->staging.done[cur]);
        if (ce != cudaSuccess) {
          note_error("checkpoint staging wait", ce);
          return MOBI_ERR_CUDA;
        }
        pending[cur] = false;
      }
      errno = 0;
      if (!pread_all(c->fd, buf, len, b.off + done)) {
        if (!host_ptrs) cudaStreamSynchronize(s);
        return io_error("truncated data block", c->path);
      }
      c->bytes_read += (int64_t)len;
      if (verify) crc = crc_update(crc, buf, len);
      if (!host_ptrs) {
        cudaError_t ce = cudaMemcpyAsync(dst, buf, len, cudaMemcpyHostToDevice, s);
        if (ce == cudaSuccess) ce = cudaEventRecord(c->staging.done[cur], s);
        if (ce != cudaSuccess) {
          note_error("checkpoint host-to-device copy", ce);
          cudaStreamSynchronize(s);
          return MOBI_ERR_CUDA;
        }
        pending[cur] = true;
        cur ^= 1;
      }
      done += len;
    }
    if (verify && (crc ^ 0xFFFFFFFFu) != b.crc) {
      if (!host_ptrs) cudaStreamSynchronize(s);
      errno = 0;
      return io_error("data checksum mismatch", c->path);
    }
  }
  if (!host_ptrs) {
    const cudaError_t ce = cudaStreamSynchronize(s);
    if (ce != cudaSuccess) {
      note_error("checkpoint copy", ce);
      return MOBI_ERR_CUDA;
    }
  }
  return MOBI_OK;
}

void mobi_ckpt_close(mobi_ckpt* c) {
  if (!c) return;
  if (c->fd >= 0) close(c->fd);
  delete c;
}

}  // extern "C"
