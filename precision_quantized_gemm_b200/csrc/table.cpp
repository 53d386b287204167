// table.cpp — the ahead-of-time per-shape configuration table and dispatch.
//
// "Helion in the vLLM backend" (third and fifth paragraphs): the autotuner
// picks a variant and config per input shape, and the picks are kept in
// configuration files maintained per model.  This file holds those entries
// keyed by (format, M, N, K) and answers lookups on the host without any
// device work (so dispatch is legal during CUDA-graph capture).  A lookup
// that misses the exact M uses the smallest tuned M' >= M of the same
// (format, N, K): tokens are bucketed upwards, as the M buckets of
// FlashInfer PR 3948 ("M bucketing by floor(log2 M)") share one tactic.
//
// File format (text, one entry per line):
//   qgemm-table 2
//   device <name with spaces replaced by _> sms <count>
//   <fmt> <M> <N> <K> <split_k> <swap_ab> <tile_n> <stages> <reduce_mode 0..2> <variant> <rows> <us>
// Version 1 files (no variant and rows columns: the tile kernel) still load.
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <fstream>
#include <map>
#include <sstream>
#include <string>
#include <tuple>

#include "../../include/qgemm.h"

// Name (spaces as '_') and SM count of the current device; false without one.
bool qg_current_device(char* name, size_t cap, int* sms);

namespace {

struct Entry {
  qg_config cfg;
  double us;
};
using Key = std::tuple<int, int, int, int>;  // fmt, N, K, M  (M last: range lookups)

struct Table {
  std::map<Key, Entry> entries;
  std::string device = "unknown";
  int sms = 0;
};

constexpr const char* kMagic = "qgemm-table";
constexpr int kVersion = 2;

bool valid_cfg_fields(const qg_config& c) {
  if (c.reserved != 0 || c.variant < 0 || c.variant > 3) return false;
  if (c.variant == 3)
    return c.split_k == 1 && c.swap_ab == 0 && (c.tile_n == 128 || c.tile_n == 256) && c.stages >= 2 &&
           c.stages <= 12 && c.reduce_mode == 0 && c.rows == 0;
  if (c.variant == 2)
    return c.split_k == 1 && c.swap_ab == 0 && (c.tile_n == 128 || c.tile_n == 256) && c.stages >= 2 &&
           c.stages <= 12 && c.reduce_mode == 0 && c.rows == 0;
  if (c.variant == 1)
    return c.split_k == 1 && c.swap_ab == 1 && (c.tile_n == 8 || c.tile_n == 16 || c.tile_n == 32) && c.stages >= 2 &&
           c.stages <= 64 && c.reduce_mode == 0 && (c.rows == 8 || c.rows == 16 || c.rows == 32 || c.rows == 64);
  return c.split_k >= 1 && c.split_k <= 256 && (c.swap_ab == 0 || c.swap_ab == 1) &&
         c.tile_n >= 16 && c.tile_n <= 256 && c.stages >= 2 && c.stages <= 12 &&
         c.reduce_mode >= 0 && c.reduce_mode <= 2 && c.rows == 0;
}

}  // namespace

extern "C" {

qg_status qgemm_table_create(void** table) {
  if (!table) return QG_ERR_INVALID_ARG;
  *table = new Table();
  return QG_OK;
}

void qgemm_table_free(void* table) { delete static_cast<Table*>(table); }

int qgemm_table_size(const void* table) {
  return table ? (int)static_cast<const Table*>(table)->entries.size() : 0;
}

qg_status qgemm_table_put(void* table, qg_format f, int M, int N, int K, const qg_config* cfg,
                          double us) {
  if (!table || !cfg || M <= 0 || N <= 0 || K <= 0 || (int)f < 0 || (int)f > 3)
    return QG_ERR_INVALID_ARG;
  if (!valid_cfg_fields(*cfg)) return QG_ERR_INVALID_ARG;
  Entry e;
  e.cfg = *cfg;
  e.us = us;
  static_cast<Table*>(table)->entries[Key((int)f, N, K, M)] = e;
  return QG_OK;
}

qg_status qgemm_table_save(const void* table, const char* path) {
  if (!table || !path) return QG_ERR_INVALID_ARG;
  const Table* t = static_cast<const Table*>(table);
  std::ofstream out(path);
  if (!out) return QG_ERR_TABLE_IO;
  std::string dev = t->device;
  std::replace(dev.begin(), dev.end(), ' ', '_');
  out << kMagic << " " << kVersion << "\n";
  out << "device " << dev << " sms " << t->sms << "\n";
  for (const auto& kv : t->entries) {
    int f, N, K, M;
    std::tie(f, N, K, M) = kv.first;
    const qg_config& c = kv.second.cfg;
    char line[256];
    std::snprintf(line, sizeof(line), "%d %d %d %d %d %d %d %d %d %d %d %.4f\n", f, M, N, K, c.split_k,
                  c.swap_ab, c.tile_n, c.stages, c.reduce_mode, c.variant, c.rows, kv.second.us);
    out << line;
  }
  return out.good() ? QG_OK : QG_ERR_TABLE_IO;
}

qg_status qgemm_table_load(const char* path, void** table) {
  if (!path || !table) return QG_ERR_INVALID_ARG;
  std::ifstream in(path);
  if (!in) return QG_ERR_TABLE_IO;
  std::string magic;
  int version = 0;
  if (!(in >> magic >> version) || magic != kMagic || version < 1 || version > kVersion) return QG_ERR_TABLE_IO;
  std::string tag, dev, tag2;
  int sms = 0;
  if (!(in >> tag >> dev >> tag2 >> sms) || tag != "device" || tag2 != "sms") return QG_ERR_TABLE_IO;
  Table* t = new Table();
  t->device = dev;
  t->sms = sms;
  std::string line;
  std::getline(in, line);  // rest of the header line
  while (std::getline(in, line)) {
    if (line.empty() || line[0] == '#') continue;
    std::istringstream ls(line);
    int f, M, N, K;
    qg_config c = {};
    double us = 0;
    bool good = static_cast<bool>(ls >> f >> M >> N >> K >> c.split_k >> c.swap_ab >> c.tile_n >> c.stages >>
                                  c.reduce_mode);
    if (good && version >= 2) good = static_cast<bool>(ls >> c.variant >> c.rows);
    if (good) good = static_cast<bool>(ls >> us);
    if (!good || f < 0 || f > 3 || M <= 0 || N <= 0 || K <= 0 || !valid_cfg_fields(c)) {
      delete t;
      return QG_ERR_TABLE_IO;
    }
    t->entries[Key(f, N, K, M)] = Entry{c, us};
  }
  *table = t;
  return QG_OK;
}

qg_status qgemm_dispatch(const void* table, qg_format f, int M, int N, int K, qg_config* out,
                         int* hit) {
  if (!out || !hit || M <= 0 || N <= 0 || K <= 0 || (int)f < 0 || (int)f > 3) return QG_ERR_INVALID_ARG;
  if (table) {
    const Table* t = static_cast<const Table*>(table);
    // identity gate: a table tuned on another device (name or SM count) is
    // not used; the scored default stands in (hit = -1)
    if (t->sms > 0 && t->device != "unknown") {
      char name[256];
      int sms = 0;
      if (qg_current_device(name, sizeof(name), &sms) && (sms != t->sms || t->device != name)) {
        *hit = -1;
        return qgemm_default_config(f, M, N, K, out);
      }
    }
    auto it = t->entries.lower_bound(Key((int)f, N, K, M));
    if (it != t->entries.end()) {
      int ef, eN, eK, eM;
      std::tie(ef, eN, eK, eM) = it->first;
      if (ef == (int)f && eN == N && eK == K) {
        *out = it->second.cfg;
        *hit = (eM == M) ? 1 : 2;
        return QG_OK;
      }
    }
  }
  *hit = 0;
  return qgemm_default_config(f, M, N, K, out);
}

}  // extern "C"

// Used by the tuner to stamp the table with the device it was tuned on
// (spaces in the name become '_', as in the file).
void qg_table_set_device(void* table, const char* name, int sms) {
  Table* t = static_cast<Table*>(table);
  t->device = name ? name : "unknown";
  std::replace(t->device.begin(), t->device.end(), ' ', '_');
  t->sms = sms;
}

// Entries in key order, for the validation gate; and their removal.
int qg_table_entry(const void* table, int i, int* f, int* M, int* N, int* K, qg_config* cfg) {
  const Table* t = static_cast<const Table*>(table);
  if (i < 0 || i >= (int)t->entries.size()) return 0;
  auto it = t->entries.begin();
  std::advance(it, i);
  std::tie(*f, *N, *K, *M) = it->first;
  *cfg = it->second.cfg;
  return 1;
}
void qg_table_erase(void* table, int f, int M, int N, int K) {
  static_cast<Table*>(table)->entries.erase(Key(f, N, K, M));
}
