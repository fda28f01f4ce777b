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


def test_gateup_bytes_follow_the_roofline_definition():
    """The dominant kernel's bytes at the DeepSeek-V3 shape: the gate and up
    weights of the 256 touched experts and of the shared expert plus h read
    once; the permuted rows and SwiGLU products only in the implementation
    bytes."""
    w = mi.WORKLOADS["deepseek_v3"]
    kept = np.full(w.E_r, 128)
    flops, nbytes = bench.gateup_work(w, kept)
    mat = 7168 * 2048 * 2
    assert nbytes == 256 * 2 * mat + 2 * mat + 4096 * 7168 * 2      # 15.15 GB
    assert abs(nbytes - 15.15e9) < 0.01e9
    assert flops == 4 * 7168 * 2048 * (4096 * 8 + 4096)
    impl = bench.gateup_impl_bytes(w, kept)
    rows = 4096 * 8
    assert impl == 2 * (257 * 2 * 7168 * 2048 + (rows + 4096) * 7168 + (rows + 4096) * 2048)
    # an expert with no kept row costs nothing
    kept[:10] = 0
    assert bench.gateup_work(w, kept)[1] == nbytes - 10 * 2 * mat
    # down: W_down of the touched experts and the shared one, y written once
    d_flops, d_bytes = bench.down_work(w, np.full(w.E_r, 128))
    assert d_bytes == 257 * mat + 4096 * 7168 * 2
    # the layer: all three matrices, fp32 centroids, h in and y out
    l_flops, l_bytes = bench.layer_work(w, np.full(w.E_r, 128))
    assert l_bytes == 257 * 3 * mat + 256 * 7168 * 4 + 2 * 4096 * 7168 * 2


def test_e4m3_bytes_count_codes_and_row_scales():
    w = mi.WORKLOADS["deepseek_v3_e4m3"]
    kept = np.full(w.E_r, 128)
    _, nbytes = bench.gateup_work(w, kept)
    assert nbytes == 257 * 2 * (7168 * 2048 + 4 * 2048) + 4096 * 7168 * 2
