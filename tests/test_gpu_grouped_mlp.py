"""Grouped SwiGLU MLP parity on the GPU (Transformer Engine "Mixture of
Experts", Grouped GEMM and Grouped MLP), through the C ABI, against the
oracle's per-expert loop. Shapes span several 128x256 tiles, ragged expert
blocks and empty experts."""
import numpy as np
import pytest
import torch

import oracle
import helpers
import workloads as wl
from helpers import assert_close, bits, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def grouped_case(T, H, I, E, k, seed, dead=(), skew=False):
    w = wl.WORKLOADS["tiny"].scaled(T=T, H=H, I=I, E=E, k=k, seed=seed, skew=skew,
                                     dead_experts=0)
    d = wl.make_inputs(w, "cuda")
    logits = d["logits"]
    for e in dead:
        logits[:, e] -= 1e4
    import routing_grouped_gemm_score_b200 as m
    r = m.moe_router_topk(logits, k)
    p = m.moe_permute(d["x"], r["topk_idx"], r["offsets"])
    return m, w, d, r, p


@pytest.mark.parametrize("tiles", ["single", "pair", "swap"])
@pytest.mark.parametrize("T,H,I,E,k,dead", [
    (64, 128, 256, 8, 2, ()),            # the tiny workload's shape
    (1000, 256, 384, 4, 2, (2,)),        # several M tiles per expert, a ragged tail, an empty expert
    (300, 512, 192, 8, 2, (0, 7)),       # I not a multiple of 128: half-empty SwiGLU tile
    (700, 320, 640, 16, 4, ()),          # H not a multiple of 256: ragged N tile in the down GEMM
    (1, 128, 128, 8, 2, ()),             # a single token
    (4500, 256, 256, 4, 2, (1,)),        # large expert blocks (the default picks pair tiles)
    (600, 200, 136, 8, 2, (5,)),         # H and I multiples of 8 only: partial 8-column chunks
    (300, 72, 40, 4, 2, ()),             # narrow rows: one partial K slice, a partial N block
])
def test_grouped_mlp_matches_expert_loop(T, H, I, E, k, dead, tiles, monkeypatch):
    helpers.force_kernels(gemm_tiles=tiles)
    m, w, d, r, p = grouped_case(T, H, I, E, k, seed=T + H + I, dead=dead)
    out = m.moe_grouped_mlp(p["x_perm"], r["offsets"], d["w_gate_up"], d["w_down"], save=True)
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    offs = r["offsets"].cpu().numpy()
    for e in dead:
        assert offs[e + 1] == offs[e]
    xp = bits(p["x_perm"])
    wgu, wd = bits(d["w_gate_up"]), bits(d["w_down"])
    y_ref = oracle.grouped_mlp(xp, offs, wgu, wd, round_bf16=True)
    assert_close(out["y_perm"], y_ref, "y_perm")
    # intermediates: g, u and h of every row
    for e in range(E):
        r0, r1 = offs[e], offs[e + 1]
        if r1 == r0:
            continue
        y, g, u, h = oracle.expert_mlp(xp[r0:r1], wgu[e], wd[e], round_bf16=True, want_intermediates=True)
        assert_close(out["gu"][r0:r1, :I], g, f"g of expert {e}")
        assert_close(out["gu"][r0:r1, I:], u, f"u of expert {e}")
        assert_close(out["h"][r0:r1], h, f"h of expert {e}")


def test_grouped_mlp_is_deterministic():
    m, w, d, r, p = grouped_case(512, 256, 256, 8, 2, seed=3)
    a = m.moe_grouped_mlp(p["x_perm"], r["offsets"], d["w_gate_up"], d["w_down"])["y_perm"]
    b = m.moe_grouped_mlp(p["x_perm"], r["offsets"], d["w_gate_up"], d["w_down"])["y_perm"]
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("tiles", ["auto", "swap"])
def test_rows_past_offsets_end_are_untouched(tiles):
    """offsets[E] < A: rows after the last expert block are not written."""
    import routing_grouped_gemm_score_b200 as m
    helpers.force_kernels(gemm_tiles=tiles)
    E, H, I = 4, 128, 128
    A = 300
    offsets = torch.tensor([0, 50, 50, 170, 200], dtype=torch.int32, device="cuda")
    g_ = torch.Generator(device="cuda").manual_seed(1)
    x = torch.randn((A, H), generator=g_, device="cuda").to(torch.bfloat16)
    wgu = (torch.randn((E, H, 2 * I), generator=g_, device="cuda") / H ** 0.5).to(torch.bfloat16)
    wd = (torch.randn((E, I, H), generator=g_, device="cuda") / I ** 0.5).to(torch.bfloat16)
    y = torch.full((A, H), 7.0, device="cuda").to(torch.bfloat16)
    ws = torch.empty(m.lib().moe_grouped_mlp_workspace_size(A, E, H, I), dtype=torch.uint8, device="cuda")
    rc = m.lib().moe_grouped_mlp(x.data_ptr(), A, offsets.data_ptr(), E, H, I, wgu.data_ptr(),
                                 wd.data_ptr(), y.data_ptr(), None, None, ws.data_ptr(), ws.numel(),
                                 torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert torch.all(y[200:].float() == 7.0)
    ref = oracle.grouped_mlp(bits(x), offsets.cpu().numpy(), bits(wgu), bits(wd))
    assert_close(y[:200], ref[:200], "y_perm")


TILE_EDGE_SIZES = [0, 1, 63, 64, 65, 127, 128, 129, 255, 256, 257, 270, 288, 289, 300, 385, 513, 544, 545]


def edge_case_inputs(sizes, H, I, seed):
    E = len(sizes)
    offs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    A = int(offs[-1])
    g_ = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn((A, H), generator=g_, device="cuda").to(torch.bfloat16)
    wgu = (torch.randn((E, H, 2 * I), generator=g_, device="cuda") / H ** 0.5).to(torch.bfloat16)
    wd = (torch.randn((E, I, H), generator=g_, device="cuda") / I ** 0.5).to(torch.bfloat16)
    scale = torch.rand((A,), generator=g_, device="cuda") + 0.5
    return offs, x, wgu, wd, scale


def test_tile_kinds_agree_bit_for_bit_on_tails():
    """Single-CTA, CTA-pair and swap-AB tiles give identical bits for y,
    [g | u] and h, with and without a row scale, on blocks whose last tile is
    short: each output element is the same fp32 sum over K in the same order,
    whichever tile holds it and whichever operand the weights are."""
    import routing_grouped_gemm_score_b200 as m
    offs, x, wgu, wd, scale = edge_case_inputs(TILE_EDGE_SIZES, 192, 320, 12)
    offs_t = torch.from_numpy(offs).cuda()
    for rs in (None, scale):
        outs = {}
        for tiles in ("single", "pair", "swap"):
            helpers.force_kernels(gemm_tiles=tiles)
            o = m.moe_grouped_mlp(x, offs_t, wgu, wd, save=True, row_scale=rs)
            torch.cuda.synchronize()
            outs[tiles] = {k: v.view(torch.int16).clone() for k, v in o.items()}
        assert m.moe_get_device_status() == 0
        for tiles in ("pair", "swap"):
            for key in ("y_perm", "gu", "h"):
                assert torch.equal(outs["single"][key], outs[tiles][key]), (tiles, key, rs is not None)


@pytest.mark.parametrize("tiles", ["single", "pair", "swap"])
def test_block_sizes_around_tile_edges(tiles, monkeypatch):
    """Expert blocks of 0 to 545 rows: every split of a block into 256-row
    pair tiles plus a last 128-row or 256-row pair tile (one CTA's 64 rows
    empty or not; a remainder of 1 to 33 rows: 257, 270, 288, 289, 513, 544,
    545), and into 128-row single tiles, with g, u and h checked as well as
    y."""
    import routing_grouped_gemm_score_b200 as m
    helpers.force_kernels(gemm_tiles=tiles)
    sizes = TILE_EDGE_SIZES
    E, H, I = len(sizes), 192, 320
    offs, x, wgu, wd, _ = edge_case_inputs(sizes, H, I, 11)
    out = m.moe_grouped_mlp(x, torch.from_numpy(offs).cuda(), wgu, wd, save=True)
    torch.cuda.synchronize()
    assert m.moe_get_device_status() == 0
    xb, wgub, wdb = bits(x), bits(wgu), bits(wd)
    assert_close(out["y_perm"], oracle.grouped_mlp(xb, offs, wgub, wdb, round_bf16=True), "y_perm")
    for e in range(E):
        r0, r1 = offs[e], offs[e + 1]
        if r1 == r0:
            continue
        y, g, u, h = oracle.expert_mlp(xb[r0:r1], wgub[e], wdb[e], round_bf16=True, want_intermediates=True)
        assert_close(out["gu"][r0:r1, :I], g, f"g of expert {e}")
        assert_close(out["gu"][r0:r1, I:], u, f"u of expert {e}")
        assert_close(out["h"][r0:r1], h, f"h of expert {e}")
