// Included after the kernel source's headers: the runtime calls it makes become host operations.
#pragma once
#define cudaFuncSetAttribute(...) cudaSuccess
#define cudaMemsetAsync(p, v, n, s) (memset((p), (v), (n)), cudaSuccess)
#define cudaGetLastError() cudaSuccess
#define cudaGetDevice(p) (*(p) = 0, cudaSuccess)
#define cudaDeviceGetAttribute(p, attr, dev) (*(p) = 148, cudaSuccess)
