"""One step of a chunked-prefill batch shaped like the long mixed config but
with 8192-token prefixes (4 chunks of 512 causal rows + 2 short decode rows,
32q/8kv heads, D 128, bs 16, bf16), through the C ABI -- small enough for a
full ncu capture of the chunk kernel.  Run on a GPU: python tests/chunk_profile_case.py
"""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import torch  # noqa: E402

import workloads  # noqa: E402
from gpu_harness import device_inputs, gpu_step  # noqa: E402
from paged_kv_cache_388_b200 import _lib  # noqa: E402
from paged_kv_cache_388_b200.batch import build_batch  # noqa: E402


def main():
    wl = workloads.mixed_workload("chunk_mixed_8k", 4242, 2, 1000, 2000, 4, 8192, 512, 32, 8, 128, 16,
                                  "bf16")
    vals = workloads.values(wl)
    batch = build_batch(wl)
    d = device_inputs(wl, vals, batch)
    for _ in range(2):
        gpu_step(_lib, wl, batch, d)
    torch.cuda.synchronize()
    assert _lib.pa_get_device_error() == 0
    print("ok", wl.name)


if __name__ == "__main__":
    main()
