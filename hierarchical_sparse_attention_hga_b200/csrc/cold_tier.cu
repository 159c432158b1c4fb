// Cold tier (HGA technical summary, "Architettura della Memoria": the whole K/V
// history may live in host RAM or on NVMe; only the routed groups reach VRAM).
//
// File layout: K then V, each [units][n_alloc][D] bf16 rows, so a group's 16
// rows, a chunk and any window run are contiguous byte ranges.  Reads and writes
// are positioned (pread / pwrite) and split over a pool of host threads by
// (sequence, KV head) unit; each thread issues its units' requests back to back,
// so the drive sees up to `threads` requests in flight.
#include "cold_tier.h"

#include <fcntl.h>
#include <sys/stat.h>
#include <unistd.h>

#include <algorithm>
#include <atomic>
#include <cerrno>
#include <cstring>
#include <system_error>
#include <thread>
#include <vector>

namespace hga {
namespace {

// Full positioned read / write of `bytes` at `off` (retrying short transfers).
std::string full_io(int fd, void* buf, int64_t bytes, int64_t off, bool write) {
  char* p = static_cast<char*>(buf);
  while (bytes > 0) {
    const ssize_t n = write ? ::pwrite(fd, p, static_cast<size_t>(bytes), off)
                            : ::pread(fd, p, static_cast<size_t>(bytes), off);
    if (n < 0) {
      if (errno == EINTR) continue;
      return std::string(write ? "pwrite" : "pread") + ": " + std::strerror(errno);
    }
    if (n == 0) return "unexpected end of file";
    p += n;
    off += n;
    bytes -= n;
  }
  return "";
}

// Runs fn(u) for u in [0, units) on up to `threads` threads (the calling one
// included; if the system refuses a thread, the ones started share the units);
// the first error wins.
template <typename Fn>
std::string parallel_units(int64_t units, int threads, Fn fn) {
  const int nt = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(threads, units)));
  std::atomic<int64_t> next{0};
  std::vector<std::string> errs(nt);
  auto work = [&](int w) {
    for (int64_t u = next++; u < units; u = next++) {
      std::string e = fn(u);
      if (!e.empty()) {
        errs[w] = e;
        next = units;  // stop handing out units
        return;
      }
    }
  };
  std::vector<std::thread> pool;
  try {
    for (int w = 1; w < nt; ++w) pool.emplace_back(work, w);
  } catch (const std::system_error&) {
  }
  work(0);
  for (auto& t : pool) t.join();
  for (auto& e : errs)
    if (!e.empty()) return e;
  return "";
}

}  // namespace

std::string cold_open(const char* path, int64_t units, int64_t n_alloc, int64_t row_bytes,
                      bool create, ColdStore* out) {
  const int fd = ::open(path, O_RDWR | O_CLOEXEC | (create ? O_CREAT : 0), 0644);
  if (fd < 0) return std::string("open ") + path + ": " + std::strerror(errno);
  const int64_t need = 2 * units * n_alloc * row_bytes;
  struct stat st;
  if (::fstat(fd, &st) != 0) {
    const std::string e = std::string("fstat: ") + std::strerror(errno);
    ::close(fd);
    return e;
  }
  if (st.st_size < need) {
    if (!create) {
      ::close(fd);
      return "the file holds " + std::to_string(st.st_size) + " bytes, the history " +
             std::to_string(need);
    }
    if (::ftruncate(fd, need) != 0) {
      const std::string e = std::string("ftruncate: ") + std::strerror(errno);
      ::close(fd);
      return e;
    }
  }
  out->fd = fd;
  out->units = units;
  out->n_alloc = n_alloc;
  out->row_bytes = row_bytes;
  return "";
}

void cold_close(ColdStore* s) {
  if (s->fd >= 0) ::close(s->fd);
  s->fd = -1;
}

std::string cold_write(const ColdStore& s, const void* k, const void* v, int64_t t0, int64_t t1,
                       int threads) {
  const int64_t half = s.units * s.n_alloc * s.row_bytes;
  return parallel_units(s.units, threads, [&](int64_t u) -> std::string {
    const int64_t off = (u * s.n_alloc + t0) * s.row_bytes, bytes = (t1 - t0) * s.row_bytes;
    std::string e = full_io(s.fd, const_cast<char*>(static_cast<const char*>(k)) + off, bytes,
                            off, true);
    if (e.empty())
      e = full_io(s.fd, const_cast<char*>(static_cast<const char*>(v)) + off, bytes, half + off,
                  true);
    return e;
  });
}

std::string cold_stage(const ColdStore& s, const LayerParams& p, const int64_t* pos,
                       const int2* plan, const int32_t* n_plan, int mode, void* staging,
                       int threads) {
  const int64_t half = s.units * s.n_alloc * s.row_bytes;
  const int64_t unit_bytes = cold_stage_unit_bytes(p);
  const int64_t group_bytes = static_cast<int64_t>(p.g) * s.row_bytes;
  const int64_t wr = window_row_capacity(p);
  return parallel_units(s.units, threads, [&](int64_t u) -> std::string {
    char* sg = static_cast<char*>(staging) + u * unit_bytes;
    char* sw = sg + 2 * static_cast<int64_t>(p.kg) * group_bytes;
    const int64_t base = u * s.n_alloc * s.row_bytes;
    const int m = std::min(n_plan[u], p.kg);
    for (int r = 0; r < m; ++r) {
      const int64_t gid = plan[u * p.kg + r].x;
      if (gid < 0 || (gid + 1) * p.g > s.n_alloc) return "a missed group outside the history";
      const int64_t off = base + gid * group_bytes;
      std::string e = full_io(s.fd, sg + r * group_bytes, group_bytes, off, false);
      if (e.empty())
        e = full_io(s.fd, sg + (p.kg + r) * group_bytes, group_bytes, half + off, false);
      if (!e.empty()) return e;
    }
    const int64_t pb = pos[u / p.Hkv];
    if (pb < 0 || pb >= s.n_alloc) return "a position outside the history";
    const int64_t nw = window_row_count(p, pb, mode);
    for (int64_t i = 0; i < nw;) {  // contiguous runs of window tokens, one read each
      const int64_t t = window_row_token(p, pb, mode, i);
      int64_t n = 1;
      while (i + n < nw && window_row_token(p, pb, mode, i + n) == t + n) ++n;
      const int64_t off = base + t * s.row_bytes;
      std::string e = full_io(s.fd, sw + i * s.row_bytes, n * s.row_bytes, off, false);
      if (e.empty())
        e = full_io(s.fd, sw + (wr + i) * s.row_bytes, n * s.row_bytes, half + off, false);
      if (!e.empty()) return e;
      i += n;
    }
    return "";
  });
}

}  // namespace hga
