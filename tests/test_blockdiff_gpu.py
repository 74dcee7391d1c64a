"""Block-diffusion decoding as a library feature (bidirectional_mamba_ssd_b200.
blockdiff): the per-layer state cache, the one-launch commit of every layer
(ssd_prefix_state_layers) and a whole block captured as one CUDA graph and
replayed, checked against the fp64 oracle's own chain of states (every step's
output of every layer, and the cache after each block)."""
import numpy as np
import pytest
import torch

import oracle
import ssd_inputs as si
from paritylib import check
from ssd_inputs import to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssd():
    import bidirectional_mamba_ssd_b200 as m
    return m


def _layers_inputs(layers, batch, L, H, N, G, seed):
    """Per-layer forward-direction inputs stacked along a leading layer axis."""
    per = [si.bidir_inputs(batch, L, H, 64, N, G, "bf16", seed=seed + l, device="cuda") for l in range(layers)]
    return (torch.stack([p["x"] for p in per]).contiguous(), torch.stack([p["dt"][0] for p in per]).contiguous(),
            torch.stack([p["A"][0] for p in per]).contiguous(), torch.stack([p["B"][0] for p in per]).contiguous())


@pytest.mark.parametrize("shape", [(3, 2, 300, 32, 128, 32), (2, 1, 200, 4, 64, 2)],
                         ids=["one_launch_192_units", "per_layer_8_units"])
def test_prefix_state_layers(ssd, shape):
    layers, batch, L, H, N, G = shape
    x, dt, A, B = _layers_inputs(layers, batch, L, H, N, G, seed=50)
    g = torch.Generator(device="cuda").manual_seed(7)
    init = torch.randn(layers, batch, H, 64, N, generator=g, device="cuda") * 0.1
    out = ssd.ssd_prefix_state_layers(x, dt, A, B, init=init)
    torch.cuda.synchronize()
    assert ssd.ssd_get_device_status() == 0
    for l in range(layers):
        o = oracle.prefix_state(to_f64(x[l]), to_f64(dt[l]), to_f64(A[l]), to_f64(B[l]), init=to_f64(init[l]))
        check(to_f64(out[l]), o, torch.bfloat16, f"layer {l}", state=True)
    # in place (the commit form): out aliases init
    st = init.clone()
    ssd.ssd_prefix_state_layers(x, dt, A, B, init=st, out=st)
    torch.cuda.synchronize()
    assert torch.equal(st, out)


def test_block_graph_against_oracle(ssd):
    from bidirectional_mamba_ssd_b200.blockdiff import BlockDiffusionCache, BlockGraph
    layers, batch, H, N, G, T, steps, prefix = 2, 2, 8, 128, 8, 64, 3, 200
    cache = BlockDiffusionCache(layers, batch, H, 64, N, device="cuda")
    # prefill every layer's cache in one call
    px, pdt, pA, pB = _layers_inputs(layers, batch, prefix, H, N, G, seed=80)
    cache.prefill(px, pdt, pA, pB)
    torch.cuda.synchronize()
    chain = [oracle.prefix_state(to_f64(px[l]), to_f64(pdt[l]), to_f64(pA[l]), to_f64(pB[l])) for l in range(layers)]
    for l in range(layers):
        check(to_f64(cache.state[l]), chain[l], torch.bfloat16, f"prefill layer {l}", state=True)

    bg = BlockGraph(cache, steps, T, H, 64, N, G)
    # each layer's A, D (both directions) are fixed across blocks
    for l in range(layers):
        p = si.bidir_inputs(1, 1, H, 64, N, G, "bf16", seed=90 + l, device="cuda")
        bg.A[l].copy_(p["A"])
        bg.D[l].copy_(p["D"])
    bg.capture()
    for blk in range(2):
        ins = {}
        for s in range(steps):
            for l in range(layers):
                p = si.bidir_inputs(batch, T, H, 64, N, G, "bf16", seed=1000 * blk + 10 * s + l, device="cuda")
                for k in ("x", "dt", "B", "C"):
                    getattr(bg, k)[s, l].copy_(p[k])
                ins[s, l] = p
        bg.replay()
        torch.cuda.synchronize()
        assert ssd.ssd_get_device_status() == 0
        A64, D64 = to_f64(bg.A), to_f64(bg.D)
        for s in range(steps):
            for l in range(layers):
                p = ins[s, l]
                o = oracle.block_step(to_f64(p["x"]), to_f64(p["dt"]), A64[l], to_f64(p["B"]), to_f64(p["C"]),
                                      D64[l], chain[l])
                check(to_f64(bg.out[s, l]), o, torch.bfloat16, f"block {blk} step {s} layer {l}")
        for l in range(layers):
            p = ins[steps - 1, l]
            chain[l] = oracle.prefix_state(to_f64(p["x"]), to_f64(p["dt"][0]), A64[l, 0], to_f64(p["B"][0]),
                                           init=chain[l])
            check(to_f64(cache.state[l]), chain[l], torch.bfloat16, f"block {blk} commit layer {l}", state=True)
