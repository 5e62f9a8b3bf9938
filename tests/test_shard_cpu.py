"""CPU checks of the head split (hybrid_softmax_linear_b200.shard): the partition of the
heads, the input slices, and, on world-size-2 gloo process groups, that each rank's
partial layer (the float64 oracle on its heads) summed across ranks is the whole layer's
output."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from hybrid_softmax_linear_b200 import shard, synth
from oracle import vdn_oracle as vo


def test_head_range_partitions_the_heads():
    for heads in (1, 2, 5, 8, 40, 41):
        for world in range(1, min(heads, 9) + 1):
            ranges = [shard.head_range(heads, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == heads
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [h1 - h0 for h0, h1 in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        shard.head_range(3, 4, 0)


def test_slices_are_the_heads_columns():
    s = synth.Shape(5, 3, 2, 2, 4, 8)
    inp = synth.make_inputs(s, "f32", seed=3, with_beta=True)
    part = shard.slice_inputs(inp, 4, 8, 1, 3)
    np.testing.assert_array_equal(part["q"], inp["q"][:, 1:3])
    np.testing.assert_array_equal(part["w_gate_l"], inp["w_gate_l"][1:3])
    np.testing.assert_array_equal(part["beta"], inp["beta"][:, 1:3])
    np.testing.assert_array_equal(part["w_os"], inp["w_os"][:, 8:24])
    assert part["w_ol"].shape == (32, 16) and part["w_ol"].flags["C_CONTIGUOUS"]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, shape, linear, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        s = synth.Shape(*shape)
        inp = synth.make_inputs(s, "f32", seed=17, with_beta=(linear == "delta"))
        inp = {n: a.astype(np.float64) for n, a in inp.items()}
        h0, h1 = shard.head_range(s.heads, world, rank)
        part = shard.slice_inputs(inp, s.heads, s.head_dim, h0, h1)
        y_r = vo.layer(part, s.frames, s.tokens_per_frame, s.chunk_frames, linear=linear)["y"]
        y = shard.reduce_partials(torch.from_numpy(np.ascontiguousarray(y_r)))
        np.save(os.path.join(out_dir, f"y{rank}.npy"), y.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("linear", ["elu1", "delta"])
def test_gloo_head_split_sums_to_the_whole_layer(tmp_path, linear):
    shape = (13, 6, 3, 4, 4, 8)        # 4 heads over 2 ranks
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), shape, linear, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    s = synth.Shape(*shape)
    inp = synth.make_inputs(s, "f32", seed=17, with_beta=(linear == "delta"))
    inp = {n: a.astype(np.float64) for n, a in inp.items()}
    ref = vo.layer(inp, s.frames, s.tokens_per_frame, s.chunk_frames, linear=linear)["y"]
    for r in range(world):
        np.testing.assert_allclose(np.load(tmp_path / f"y{r}.npy"), ref, rtol=1e-12, atol=1e-13)
