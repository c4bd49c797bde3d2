"""GPU parity and invariance of the MoE steps around the grouped GEMM (include/bi_moe.h):
routing, dispatch and gather bit-exact against the oracle, combine within the tolerance (and
bit-exact on exact inputs), and the whole layer T-invariant bitwise."""
import numpy as np
import pytest
import torch

import invariant_deterministic_gemm_bi_b200 as bg
import oracle
from oracle import moe as omoe
from invariant_deterministic_gemm_bi_b200 import inputs
from tests import parity

pytestmark = pytest.mark.gpu
DEV = "cuda"
E, TOPK = 64, 8


def gpu_route(logits, k=TOPK):
    T = logits.shape[0]
    ex = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    bg.bi_moe_route_topk(logits, k, ex, w)
    return ex, w


def gpu_dispatch(experts, n_exp=E):
    T, k = experts.shape
    off = torch.empty(n_exp + 1, dtype=torch.int32, device=DEV)
    tok = torch.full((T * k,), -1, dtype=torch.int32, device=DEV)
    ros = torch.full((T * k,), -1, dtype=torch.int32, device=DEV)
    bg.bi_moe_dispatch(experts, n_exp, off, tok, ros)
    return off, tok, ros


@pytest.mark.parametrize("T,kind", [(1, "gauss"), (1000, "gauss"), (513, "ties")])
def test_route_matches_oracle(T, kind):
    g = inputs.generator(9400 + T, "cpu")
    logits = torch.randn(T, E, generator=g, dtype=torch.float32)
    if kind == "ties":
        logits = torch.round(logits * 2) / 2          # few distinct values: many ties
    ex, w = gpu_route(logits.to(DEV))
    oex, ow = omoe.route_topk(logits.numpy(), TOPK)
    assert (ex.cpu().numpy() == oex).all(), "expert selection differs from the oracle"
    wg = w.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(wg - ow) <= 8e-6 * ow + 1e-12), float(np.max(np.abs(wg - ow) / ow))


# T * 8 pairs: up to 4096 the pass kernels, up to 16384 8-warp segments, above 32-warp segments
@pytest.mark.parametrize("T", [1, 7, 1024, 4096, 8192])
def test_dispatch_matches_oracle(T):
    g = inputs.generator(9500 + T, "cpu")
    experts = torch.randint(0, E, (T, TOPK), generator=g, dtype=torch.int32)
    off, tok, ros = gpu_dispatch(experts.to(DEV))
    ooff, otok, oros = omoe.dispatch(experts.numpy(), E)
    assert (off.cpu().numpy() == ooff).all()
    assert (tok.cpu().numpy() == otok).all()
    assert (ros.cpu().numpy() == oros).all()


@pytest.mark.parametrize("T", [1001, 3001])
def test_dispatch_with_ids_not_16_byte_aligned(T):
    # ids 4 bytes past a 16-byte boundary take the scalar loads, with 8 warps per expert block
    # (8008 pairs) and with 32 (24008 pairs); the grouping is the same
    g = inputs.generator(9550 + T, "cpu")
    experts = torch.randint(0, E, (T, TOPK), generator=g, dtype=torch.int32)
    buf = torch.empty(T * TOPK + 4, dtype=torch.int32, device=DEV)
    view = buf[1:1 + T * TOPK].view(T, TOPK)
    view.copy_(experts.to(DEV))
    assert view.data_ptr() % 16 == 4
    off, tok, ros = gpu_dispatch(view)
    ooff, otok, oros = omoe.dispatch(experts.numpy(), E)
    assert (off.cpu().numpy() == ooff).all()
    assert (tok.cpu().numpy() == otok).all()
    assert (ros.cpu().numpy() == oros).all()


def test_dispatch_leaves_out_of_range_ids():
    experts = torch.tensor([[0, 5], [64, 1], [3, 3]], dtype=torch.int32)
    off, tok, ros = gpu_dispatch(experts.to(DEV))
    ooff, otok, oros = omoe.dispatch(experts.numpy(), E)
    assert (off.cpu().numpy() == ooff).all() and int(off[-1]) == 5
    R = int(ooff[-1])
    assert (tok.cpu().numpy()[:R] == otok).all()
    assert (ros.cpu().numpy() == oros).all()       # -1 where the id was out of range


def test_gather_is_exact():
    T, K, R = 300, 7168, 2400
    X = inputs.bf16_gaussian((T, K), seed=9601, device=DEV)
    g = inputs.generator(9602, "cpu")
    tok = torch.randint(0, T, (R,), generator=g, dtype=torch.int32)
    A = torch.empty((R, K), dtype=torch.bfloat16, device=DEV)
    bg.bi_moe_gather_rows(X, tok.to(DEV), A)
    ref = omoe.gather_rows(inputs.to_numpy_bits(X), tok.numpy())
    assert (inputs.to_numpy_bits(A) == ref).all()


def _combine_inputs(T, N, seed, exact=False):
    R = T * TOPK
    g = inputs.generator(seed, "cpu")
    ros = torch.randperm(R, generator=g).to(torch.int32)
    if exact:
        C = inputs.bf16_integers((R, N), seed=seed + 1)
        w = torch.tensor([2.0 ** -j for j in range(TOPK)], dtype=torch.float32).repeat(T, 1)
    else:
        C = inputs.bf16_gaussian((R, N), seed=seed + 1)
        w = torch.rand(T, TOPK, generator=g, dtype=torch.float32) / TOPK
    return C, ros, w


@pytest.mark.parametrize("T,N,exact", [(1, 2048, False), (1000, 2048, False), (64, 2048, True)])
def test_combine_matches_oracle(T, N, exact):
    C, ros, w = _combine_inputs(T, N, 9700 + T, exact)
    Y = torch.empty((T, N), dtype=torch.bfloat16, device=DEV)
    bg.bi_moe_combine(C.to(DEV), ros.to(DEV), w.to(DEV), Y)
    yref, ybits = omoe.combine(inputs.to_numpy_bits(C), ros.numpy(), w.numpy())
    got = inputs.to_numpy_bits(Y)
    if exact:
        parity.assert_bits_equal_values(got, ybits, "exact combine")
    else:
        cv = oracle.bf16_to_f64(inputs.to_numpy_bits(C))
        scale = np.zeros((T, N))
        rows = ros.numpy().reshape(T, TOPK)
        for j in range(TOPK):
            scale += np.abs(w.numpy()[:, j:j + 1].astype(np.float64) * cv[rows[:, j]])
        err = np.abs(oracle.bf16_to_f64(got) - yref)
        assert np.all(err <= 2.0 ** -7 * np.abs(yref) + 2.0 ** -20 * scale + 1e-30)


def _moe_layer(tokens, logits, B, plan):
    """route -> dispatch -> gather -> grouped GEMM -> combine, all on the GPU."""
    T, K = tokens.shape
    N = B.shape[1]
    ex, w = gpu_route(logits)
    off, tok, ros = gpu_dispatch(ex)
    R = T * TOPK
    A = torch.empty((R, K), dtype=torch.bfloat16, device=DEV)
    bg.bi_moe_gather_rows(tokens, tok, A)
    C = torch.empty((R, N), dtype=torch.bfloat16, device=DEV)
    bg.bi_grouped_gemm_run(plan, A, B, C, off)
    Y = torch.empty((T, N), dtype=torch.bfloat16, device=DEV)
    bg.bi_moe_combine(C, ros, w, Y)
    bg.bi_gemm_sync_status(plan)
    return Y


def test_moe_layer_rows_invariant_to_t():
    N, K = 2048, 7168
    B = inputs.bf16_gaussian((E, N, K), seed=9801, std=K ** -0.5, device=DEV)
    plan = bg.bi_gemm_plan(N, K, bg.BI_DTYPE_BF16, E)
    g = inputs.generator(9802, "cpu")
    test_tok = inputs.bf16_gaussian((16, K), seed=9803, device=DEV)
    test_logits = torch.randn(16, E, generator=g, dtype=torch.float32).to(DEV)
    ref = torch.cat([_moe_layer(test_tok[i:i + 1].contiguous(), test_logits[i:i + 1].contiguous(), B, plan)
                     for i in range(16)]).view(torch.int16)
    rng = np.random.default_rng(9804)
    for T in [64, 1024]:
        toks = inputs.bf16_gaussian((T, K), seed=9805 + T, device=DEV)
        logits = torch.randn(T, E, generator=g, dtype=torch.float32).to(DEV)
        pos = torch.from_numpy(rng.choice(T, size=16, replace=False)).to(DEV)
        toks[pos] = test_tok
        logits[pos] = test_logits
        Y = _moe_layer(toks, logits, B, plan).view(torch.int16)
        bad = (Y[pos] != ref).any(dim=1)
        assert not bad.any(), f"T={T}: {int(bad.sum())} of 16 tokens differ from their T=1 output"
