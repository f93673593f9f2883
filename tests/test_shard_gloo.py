"""Multi-rank host logic on CPU: two gloo ranks split a batch by sequence, each
projects its shard with the oracle, and the gathered shards equal the whole batch
(no data-path collective: the all_gather only collects results to check). For
data-parallel training, each rank's backward of its shard, summed over ranks by
allreduce_gradients, equals the backward of the whole batch."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads as W
from oracle import projector as O
from oracle import backward as B
from vision_language_projector_b200.shard import allreduce_gradients, plan_shard, sequence_block


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case():
    wl = W.Workload("shard_case", 120, 6, 2, 8, 12, 6, True, False, True, 1, 2, 3, 160, (5, 5), None, False)
    hw = W.grid_hw(wl)
    crop = W.spatial_crop(wl)
    rows = O.image_rows(hw, wl.k, crop)
    ids = W.input_ids(wl, rows)
    feats = W.features(wl, hw)
    w = W.weights(wl)
    table = W.embed_table(wl)
    emb = O.bf16_bits_to_f64(W.prefill_embeds(wl, ids, table))
    emb[np.isnan(emb)] = 0.0
    return wl, hw, crop, rows, ids, feats, w, emb


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl, hw, crop, rows, ids, feats, w, emb = _case()
        per_seq = wl.n_images // wl.B
        image_seq = [i // per_seq for i in range(wl.n_images)]
        sh = plan_shard(image_seq, [wl.views_per_image] * wl.n_images, hw, wl.B, wl.S, world, rank)
        mine = O.forward(feats[sh.patches], hw[sh.views], crop[sh.images], wl.k, O.params_f64(w), ids[sh.ids],
                         W.IMAGE_TOKEN_ID, emb[sh.ids])
        parts = [None] * world
        dist.all_gather_object(parts, (sh.ids.start, sh.ids.stop, mine))
        if rank == 0:
            out.put([(a, b, m.tolist()) for a, b, m in parts])
    finally:
        dist.destroy_process_group()


def test_sequence_blocks_partition():
    for n in (1, 7, 16, 33):
        for world in (1, 2, 3, 8):
            blocks = [sequence_block(n, world, r) for r in range(world)]
            assert blocks[0].start == 0 and blocks[-1].stop == n
            assert all(a.stop == b.start for a, b in zip(blocks, blocks[1:]))
            sizes = [b.stop - b.start for b in blocks]
            assert max(sizes) - min(sizes) <= 1


def test_two_gloo_ranks_reassemble_the_batch():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    parts = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl, hw, crop, rows, ids, feats, w, emb = _case()
    whole = O.forward(feats, hw, crop, wl.k, O.params_f64(w), ids, W.IMAGE_TOKEN_ID, emb)
    got = np.zeros_like(whole)
    covered = np.zeros(len(whole), bool)
    for a, b, m in parts:
        got[a:b] = np.array(m)
        assert not covered[a:b].any()
        covered[a:b] = True
    assert covered.all()
    np.testing.assert_array_equal(got, whole)


def _grad_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl, hw, crop, rows, ids, feats, w, emb = _case()
        per_seq = wl.n_images // wl.B
        image_seq = [i // per_seq for i in range(wl.n_images)]
        sh = plan_shard(image_seq, [wl.views_per_image] * wl.n_images, hw, wl.B, wl.S, world, rank)
        d_out = O.bf16_bits_to_f64(W.grad_out(wl, len(ids)))
        params = O.params_f64(w)
        params["mid"] = [(np.ones((wl.N1, wl.N1)) * 0.01, np.zeros(wl.N1))]       # depth 3
        g = B.backward(feats[sh.patches], hw[sh.views], crop[sh.images], wl.k, params, ids[sh.ids],
                       W.IMAGE_TOKEN_ID, d_out[sh.ids])
        mine = {k: torch.from_numpy(g[k]) for k in ("W1", "b1", "W2", "b2", "gamma", "beta", "newline", "sep")}
        mine["W_mid"] = [torch.from_numpy(g["mid"][0][0])]
        mine["b_mid"] = [torch.from_numpy(g["mid"][0][1])]
        # the shard's own feature gradient: a different size on every rank, not summed
        mine["features"] = torch.from_numpy(g["features"]).clone()
        allreduce_gradients(mine)
        assert torch.equal(mine.pop("features"), torch.from_numpy(g["features"]))
        if rank == 0:
            out.put({k: ([t.numpy().tolist() for t in v] if isinstance(v, list) else v.numpy().tolist())
                     for k, v in mine.items()})
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_sum_to_the_batch_gradient():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_grad_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl, hw, crop, rows, ids, feats, w, emb = _case()
    params = O.params_f64(w)
    params["mid"] = [(np.ones((wl.N1, wl.N1)) * 0.01, np.zeros(wl.N1))]
    want = B.backward(feats, hw, crop, wl.k, params, ids, W.IMAGE_TOKEN_ID,
                      O.bf16_bits_to_f64(W.grad_out(wl, len(ids))))
    for k in ("W1", "b1", "W2", "b2", "gamma", "beta", "newline", "sep"):
        np.testing.assert_allclose(np.array(got[k]), want[k], rtol=1e-12, atol=1e-12, err_msg=k)
    np.testing.assert_allclose(np.array(got["W_mid"][0]), want["mid"][0][0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(np.array(got["b_mid"][0]), want["mid"][0][1], rtol=1e-12, atol=1e-12)
