#!/usr/bin/env bash
# Build libtq4_1s.so for sm_100a (B200).  Usage: build.sh [output.so]
set -euo pipefail
HERE="$(cd "$(dirname "${BASH_SOURCE[0]}")" && pwd)"
ROOT="$(cd "$HERE/../.." && pwd)"
OUT="${1:-$HERE/../libtq4_1s.so}"
NVCC="${NVCC:-nvcc}"
"$NVCC" -std=c++17 -O3 -lineinfo -rdc=true -shared -Xcompiler -fPIC -Xcompiler -fvisibility=hidden \
  -gencode arch=compute_100a,code=sm_100a \
  -I"$ROOT/include" -I"$HERE" \
  "$HERE/tq4_api.cu" "$HERE/tq4_kernels.cu" "$HERE/tq4_streamk.cu" "$HERE/tq4_decode.cu" "$HERE/tq4_gemm.cu" "$HERE/tq4_static.cu" \
  -o "$OUT" ${TQ_EXTRA_NVCC_FLAGS:-}
