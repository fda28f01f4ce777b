"""Byte and FLOP counts bench.py divides by (host logic, CPU): the backward's
bytes at the DeepSeek-V3 shape counted by hand, and the writes of the
write-aware roofline."""
import numpy as np

import bench
import moe_inputs as mi


def test_backward_bytes_and_writes_deepseek_v3():
    w = mi.WORKLOADS["deepseek_v3"]
    kept = np.full(w.E_r, 128)                       # every expert touched, T*K rows
    flops, nbytes = bench.train_work(w, kept)
    mat = 7168 * 2048 * 2                            # one bf16 expert matrix
    weights_read = 256 * 3 * mat + 3 * mat           # routed + shared
    grads_written = 256 * 3 * mat + 3 * mat
    assert nbytes == weights_read + grads_written + 3 * 4096 * 7168 * 2 + 256 * 7168 * 4
    assert bench.train_writes(w) == grads_written + 4096 * 7168 * 2 + 256 * 7168 * 4
    # dA, dX and the three weight gradients: 2 * 3 * 2 FLOPs per (row, d, f) of each GEMM pair
    assert flops == 12 * 7168 * (2048 * 4096 * 8 + 2048 * 4096) + 4 * 4096 * 256 * 7168
