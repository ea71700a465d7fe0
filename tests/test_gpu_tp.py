"""TP over the expert intermediate dimension I on one GPU: every rank's slice
is run in turn (moe_tp_shard, moe_layer_forward_partial) and moe_tp_reduce
sums the ranks' fp32 partial outputs in one kernel that reads all of them --
the single-GPU form of the reduction, whose parts on several GPUs are peer
mappings.  Checked against the oracle: the shards are exact copies of the
oracle's slices, every rank's partial matches the oracle's layer on that
slice, and the reduced output matches the oracle's unsplit layer (equal to
the sum of the slices by the oracle's own pin).  Routing is taken from the
logits the kernels computed, which must be identical on every rank."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import mixture_experts_layer_61_b200 as moe
import oracle
from helpers import OUT_TOL, cfg_for, host, rel_err, sample_tokens, small_shape

pytestmark = pytest.mark.gpu


def _run_tp(shape, T, n_ranks, seed, n_sample=None, check_rank=None, pad_mode=0, k=None, override=None):
    w = mi.make_weights(shape, seed, device="cuda")
    x = mi.make_x(shape, T, seed, device="cuda")
    cl = moe.tp_config(cfg_for(shape, T, pad_mode=pad_mode), n_ranks)
    kt = None if k is None else torch.from_numpy(np.asarray(k, np.int32)).cuda()
    ws = moe.alloc_workspace(moe.workspace_size(cl))
    parts, lgs = [], []
    for r in range(n_ranks):
        a13, a2 = moe.tp_shard(w["w13"], w["w2"], r, n_ranks)
        s13, s2 = moe.tp_shard(w["w13_sh"], w["w2_sh"], r, n_ranks) if shape.I_sh else (None, None)
        parts.append(moe.layer_forward_partial(cl, x, w["w_r"], a13, a2, ws, s13, s2, logits_override=override,
                                               k=kt))
        moe.check_status(ws)
        lgs.append(moe.layer_logits(cl, ws).clone())
        del a13, a2, s13, s2
    assert all(torch.equal(lgs[0], lg) for lg in lgs[1:])  # every rank routes identically
    out = moe.tp_reduce(parts, dtype=x.dtype)
    lg = lgs[0].cpu().numpy() if override is None else override.cpu().numpy()
    tok = sample_tokens(T, n_sample or T, seed)
    hx, h13, h2 = host(x), host(w["w13"]), host(w["w2"])
    sh = dict(w13_sh=host(w["w13_sh"]), w2_sh=host(w["w2_sh"])) if shape.I_sh else {}
    ref = oracle.moe_layer(hx, None, h13, h2, shape.K, shape.score_fn, shape.renorm, logits=lg, tokens=tok, k=k,
                           **sh)
    errs = {"out": rel_err(out.float().cpu().numpy()[tok], ref)}
    ranks = range(n_ranks) if check_rank is None else [check_rank]
    for r in ranks:
        o13, o2 = oracle.tp_shard(h13, h2, r, n_ranks)
        osh = {}
        if shape.I_sh:
            a, b = oracle.tp_shard(sh["w13_sh"], sh["w2_sh"], r, n_ranks)
            osh = dict(w13_sh=a, w2_sh=b)
        ref_r = oracle.moe_layer(hx, None, o13, o2, shape.K, shape.score_fn, shape.renorm, logits=lg, tokens=tok,
                                 k=k, **osh)
        errs[f"part{r}"] = rel_err(parts[r].cpu().numpy()[tok], ref_r)
    return errs


def test_tp_shard_is_the_oracle_slice():
    shape = small_shape(H=256, E=4, K=2, I=512)
    w = mi.make_weights(shape, 1, device="cuda", shared=False)
    for n, r in [(1, 0), (2, 1), (4, 2), (8, 7)]:
        a13, a2 = moe.tp_shard(w["w13"], w["w2"], r, n)
        o13, o2 = oracle.tp_shard(host(w["w13"]), host(w["w2"]), r, n)
        assert np.array_equal(host(a13), o13) and np.array_equal(host(a2), o2)
    d13, d2 = moe.tp_shard(w["w13"][1].contiguous(), w["w2"][1].contiguous(), 3, 4)  # one dense FFN
    o13, o2 = oracle.tp_shard(host(w["w13"])[1], host(w["w2"])[1], 3, 4)
    assert np.array_equal(host(d13), o13) and np.array_equal(host(d2), o2)


@pytest.mark.parametrize("n_ranks", [2, 4])
@pytest.mark.parametrize("T", [5, 96, 300])
def test_tp_small_layer_with_shared(n_ranks, T):
    shape = small_shape(H=512, E=16, K=4, I=768, I_sh=256)
    errs = _run_tp(shape, T, n_ranks, seed=T + n_ranks)
    assert max(errs.values()) < OUT_TOL, errs


@pytest.mark.parametrize("T", [24, 200])
def test_tp_dynamic_k_max_value_padding_and_supplied_logits(T):
    # per-token expert counts 0..K (0 = shared experts only), max-value padding,
    # skewed supplied logits: the same on every rank
    shape = small_shape(H=512, E=16, K=4, I=768, I_sh=256, score_fn=1)
    k = np.random.default_rng(T).integers(0, 5, T).astype(np.int32)
    lg = mi.zipf_gumbel_logits(16, T, 1.2, seed=T, device="cuda")
    errs = _run_tp(shape, T, 2, seed=T, pad_mode=1, k=k, override=lg)
    assert max(errs.values()) < OUT_TOL, errs


def test_tp_tiny_fp32():
    errs = _run_tp(mi.SHAPES["tiny"], 64, 2, seed=4)
    assert max(errs.values()) < OUT_TOL, errs


@pytest.mark.parametrize("name,T,n_ranks", [("mixtral", 32, 8), ("mixtral", 2048, 4), ("qwen2moe", 32, 8),
                                            ("deepseekv3", 32, 8)])
def test_tp_full_size_sampled(name, T, n_ranks):
    errs = _run_tp(mi.SHAPES[name], T, n_ranks, seed=7, n_sample=24, check_rank=n_ranks - 1)
    assert max(errs.values()) < OUT_TOL, errs
    torch.cuda.empty_cache()


def test_tp_one_rank_is_the_layer_bit_for_bit():
    # the unsplit partial rounded once is exactly what the layer's combine rounds
    shape = small_shape(H=512, E=16, K=4, I=768, I_sh=256)
    for T in (7, 200):
        x, w = mi.make_x(shape, T, 2, device="cuda"), mi.make_weights(shape, 2, device="cuda")
        cfg = cfg_for(shape, T)
        ws = moe.alloc_workspace(moe.workspace_size(cfg))
        ref = moe.layer_forward(cfg, x, w["w_r"], w["w13"], w["w2"], ws, w["w13_sh"], w["w2_sh"])
        tp = moe.tp_layer_forward(moe.tp_config(cfg, 1), x, w["w_r"], w["w13"], w["w2"], ws, w["w13_sh"],
                                  w["w2_sh"])
        torch.cuda.synchronize()
        assert torch.equal(tp, ref)


@pytest.mark.parametrize("n", [1, 3, 16])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_tp_reduce_is_the_rank_order_fp32_sum(n, dtype):
    g = torch.Generator().manual_seed(n)
    count = 4 * 1237
    host_parts = [torch.randn(count, generator=g) * (r + 1) for r in range(n)]
    acc = host_parts[0].numpy().copy()
    for p in host_parts[1:]:
        acc = (acc + p.numpy()).astype(np.float32)   # IEEE fp32 adds in rank order
    want = torch.from_numpy(acc).to(dtype)            # one round-to-nearest-even
    got = moe.tp_reduce([p.cuda() for p in host_parts], dtype=dtype).cpu()
    assert torch.equal(got, want)


def test_tp_argument_errors():
    a = torch.zeros(64, dtype=torch.float32, device="cuda")
    with pytest.raises(moe.MoeError):
        moe.tp_reduce([a] * 17)
    with pytest.raises(moe.MoeError):
        moe.tp_reduce([a[1:61]])                      # not 16-byte aligned
    w13 = torch.zeros(2, 2 * 24, 16, dtype=torch.bfloat16, device="cuda")
    w2 = torch.zeros(2, 16, 24, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError):
        moe.tp_shard(w13, w2, 0, 5)                   # 24 does not split over 5
    with pytest.raises(ValueError):
        moe.tp_config(moe.config(4, 16, 2, 1, 24), 5)


@pytest.mark.parametrize("n_ranks,n_chunks", [(2, 2), (2, 4), (4, 4), (1, 3)])
def test_tp_overlapped_down_chunks(n_ranks, n_chunks):
    # the all-reduce overlapped with the down projection: per rank the front
    # part, then the down projection + combine of each block of H / n_chunks
    # output features into its own fp32 part; the parts summed over the ranks
    # (here in rank order on one GPU, where an all-reduce would run) and placed
    # side by side are the layer; every rank's blocks side by side are its
    # slice's partial output.  T = 700 on 16 experts: 175 rows per expert, the
    # two-launch expert FFN (CTA-pair GEMMs) and the shared GEMM pair.
    shape = small_shape(H=768, E=16, K=4, I=768, I_sh=384)
    T, seed = 700, 41 + n_ranks + n_chunks
    w = mi.make_weights(shape, seed, device="cuda")
    x = mi.make_x(shape, T, seed, device="cuda")
    cl = moe.tp_config(cfg_for(shape, T), n_ranks)
    assert not moe.ffn_fused(cl)
    ws = moe.alloc_workspace(moe.workspace_size(cl))
    total = [torch.zeros((T, shape.H // n_chunks), dtype=torch.float32, device="cuda") for _ in range(n_chunks)]
    tok = sample_tokens(T, 128, seed)
    hx, h13, h2 = host(x), host(w["w13"]), host(w["w2"])
    hs13, hs2 = host(w["w13_sh"]), host(w["w2_sh"])
    lg = None
    for r in range(n_ranks):
        a13, a2 = moe.tp_shard(w["w13"], w["w2"], r, n_ranks)
        s13, s2 = moe.tp_shard(w["w13_sh"], w["w2_sh"], r, n_ranks)
        moe.layer_forward_partial_front(cl, x, w["w_r"], a13, ws, s13, s2)
        parts = [moe.layer_forward_partial_down(cl, a2, c, n_chunks, ws) for c in range(n_chunks)]
        moe.check_status(ws)
        if lg is None:
            lg = moe.layer_logits(cl, ws).cpu().numpy()
        full_r = torch.cat(parts, dim=1).cpu().numpy()
        o13, o2 = oracle.tp_shard(h13, h2, r, n_ranks)
        q13, q2 = oracle.tp_shard(hs13, hs2, r, n_ranks)
        ref_r = oracle.moe_layer(hx, None, o13, o2, shape.K, shape.score_fn, shape.renorm, logits=lg, tokens=tok,
                                 w13_sh=q13, w2_sh=q2)
        assert rel_err(full_r[tok], ref_r) < OUT_TOL
        for c in range(n_chunks):
            total[c] += parts[c]
    out = moe.tp_gather(total, torch.empty((T, shape.H), dtype=x.dtype, device="cuda"))
    torch.cuda.synchronize()
    ref = oracle.moe_layer(hx, None, h13, h2, shape.K, shape.score_fn, shape.renorm, logits=lg, tokens=tok,
                           w13_sh=hs13, w2_sh=hs2)
    assert rel_err(out.float().cpu().numpy()[tok], ref) < OUT_TOL


def test_tp_overlapped_one_rank_equals_the_layer():
    # the whole overlapped step on one rank (the all-reduce has nothing to sum)
    # against the unsplit layer: the same routing and the same numerics up to
    # the fp32 order of the down GEMM's split tiles
    shape = small_shape(H=512, E=8, K=2, I=1024, I_sh=512)
    T = 1200
    w = mi.make_weights(shape, 9, device="cuda")
    x = mi.make_x(shape, T, 9, device="cuda")
    cfg = cfg_for(shape, T)
    ws = moe.alloc_workspace(moe.workspace_size(cfg))
    ref = moe.layer_forward(cfg, x, w["w_r"], w["w13"], w["w2"], ws, w["w13_sh"], w["w2_sh"]).float()
    cl = moe.tp_config(cfg, 1)
    out = moe.tp_layer_forward_overlapped(cl, x, w["w_r"], w["w13"], w["w2"], ws, w["w13_sh"], w["w2_sh"],
                                          n_chunks=4)
    moe.check_status(ws)
    assert rel_err(out.float().cpu().numpy(), ref.cpu().numpy()) < 1e-2


def test_tp_down_chunk_arguments():
    shape = small_shape(H=512, E=8, K=2, I=512)
    cfg = cfg_for(shape, 1200)
    ws = moe.alloc_workspace(moe.workspace_size(cfg))
    w2 = torch.zeros((8, 512, 512), dtype=torch.bfloat16, device="cuda")
    for chunk, n in [(0, 3), (4, 4), (-1, 2), (0, 0)]:       # 512 / 3 not whole; chunk out of range
        with pytest.raises(moe.MoeError):
            moe.layer_forward_partial_down(cfg, w2, chunk, n, ws,
                                           torch.empty((1200, 128), dtype=torch.float32, device="cuda"))
    small = cfg_for(shape, 8)                                 # decode size: the fused expert FFN
    with pytest.raises(moe.MoeError):
        moe.layer_forward_partial_down(small, w2, 0, 2, moe.alloc_workspace(moe.workspace_size(small)),
                                       torch.empty((8, 256), dtype=torch.float32, device="cuda"))
