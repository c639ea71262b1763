// Host-side stream helpers used by the API translation unit.
#pragma once
#include <cstdint>
#include <string>
#include <vector>

#include "stagq.h"

namespace stagq {

struct HostStreamBuffers {
  std::vector<uint8_t> planes, pair_idx;
  std::vector<int32_t> row_ptr;
  std::vector<uint16_t> col, val;
  stagq_host_stream view{};
};

int check_shape(int64_t out, int64_t in, int64_t group, int n_planes);
int validate_stream(const stagq_host_stream* s);
int read_stream_file(const char* path, HostStreamBuffers* buf);
void set_error(const std::string& msg);

}  // namespace stagq
