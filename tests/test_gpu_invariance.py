"""GPU batch invariance, bitwise: a row computed alone (M = 1) must come out with exactly the same
bits inside every larger batch, at any position, under row permutations and among fresh random
co-batched rows ("DeepSeek不惜代价保住它！V4关键特性被挖出来了" (QbitAI), section
"什么是batch invariance").  Needs no oracle: the M = 1 result is the single correct bit pattern.
"""
import numpy as np
import pytest
import torch

import invariant_deterministic_gemm_bi_b200 as bg
from invariant_deterministic_gemm_bi_b200 import inputs
from tests import routing as routing_mod
from tests.gpu_util import kblock_major_scales

pytestmark = pytest.mark.gpu
DEV = "cuda"


class Dense:
    def __init__(self, B, dtype=bg.BI_DTYPE_BF16, scale_b=None):
        self.B = B
        self.N, self.K = B.shape
        self.plan = bg.bi_gemm_plan(self.N, self.K, dtype, 1)
        self.scale_b = scale_b

    def __call__(self, A, sa_mk=None):
        C = torch.empty((A.shape[0], self.N), dtype=torch.bfloat16, device=DEV)
        sa = kblock_major_scales(sa_mk) if sa_mk is not None else None
        bg.bi_gemm_run(self.plan, A, self.B, C, scale_a=sa, scale_b=self.scale_b)
        bg.bi_gemm_sync_status(self.plan)
        return C


def alone(f, rows, scales=None):
    """Each row computed on its own (M = 1)."""
    out = []
    for i in range(rows.shape[0]):
        out.append(f(rows[i:i + 1].contiguous(), None if scales is None else scales[i:i + 1]))
    return torch.cat(out).view(torch.int16)


def check_in_batch(f, test_rows, ref_bits, M, seed, fresh, scales=None, fresh_scales=None,
                   positions=None):
    """Put min(M, T) test rows at random (or given) positions among fresh rows; compare bits."""
    rng = np.random.default_rng(seed)
    T = test_rows.shape[0]
    k = min(M, T) if positions is None else len(positions)
    pick = rng.choice(T, size=k, replace=False)
    pos = rng.choice(M, size=k, replace=False) if positions is None else np.asarray(positions)[:k]
    batch = fresh(M).clone()
    batch[torch.from_numpy(pos).to(DEV)] = test_rows[torch.from_numpy(pick).to(DEV)]
    bscales = None
    if scales is not None:
        bscales = fresh_scales(M).clone()
        bscales[torch.from_numpy(pos).to(DEV)] = scales[torch.from_numpy(pick).to(DEV)]
    C = f(batch, bscales).view(torch.int16)
    got = C[torch.from_numpy(pos).to(DEV)]
    want = ref_bits[torch.from_numpy(pick).to(DEV)]
    bad = (got != want).any(dim=1)
    assert not bad.any(), f"M={M}: {int(bad.sum())} of {k} rows differ from their M=1 bits"


# ---------------------------------------------------------------------------------------------
# small shape: M in {1, 3, 8, 17, 64} under permutations (Gaussian and integer inputs)
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("kind", ["gaussian", "integer"])
def test_small_rows_invariant_under_batch_size_and_permutation(kind):
    gen = inputs.bf16_gaussian if kind == "gaussian" else inputs.bf16_integers
    B = gen((256, 512), seed=1001, device=DEV)
    f = Dense(B)
    test_rows = gen((16, 512), seed=1002, device=DEV)
    ref = alone(f, test_rows)
    for M in [1, 3, 8, 17, 64]:
        for trial in range(8):
            s = inputs.derived_seed(1000, M, trial)
            check_in_batch(f, test_rows, ref, M, s,
                           lambda m, s=s: gen((m, 512), seed=s, device=DEV))
    # a full permutation of one batch permutes its output rows bit for bit
    A = gen((64, 512), seed=1003, device=DEV)
    C = f(A).view(torch.int16)
    for trial in range(8):
        perm = torch.from_numpy(np.random.default_rng(trial).permutation(64)).to(DEV)
        assert torch.equal(f(A[perm].contiguous()).view(torch.int16), C[perm])


# ---------------------------------------------------------------------------------------------
# decode-shaped: N = 4096, K = 7168, M = 1 .. 256, fresh co-batched rows, first/last positions
# ---------------------------------------------------------------------------------------------

def test_decode_rows_invariant_across_m_sweep():
    N, K = 4096, 7168
    B = inputs.bf16_gaussian((N, K), seed=2001, std=K ** -0.5, device=DEV)
    f = Dense(B)
    test_rows = inputs.bf16_gaussian((32, K), seed=2002, device=DEV)
    ref = alone(f, test_rows)
    for M in [2, 4, 8, 16, 32, 64, 128, 256]:
        for trial in range(4):
            s = inputs.derived_seed(2000, M, trial)
            fresh = lambda m, s=s: inputs.bf16_gaussian((m, K), seed=s, device=DEV)
            check_in_batch(f, test_rows, ref, M, s, fresh)
        check_in_batch(f, test_rows, ref, M, M, fresh, positions=[0, M - 1])


def test_scheduling_forms_of_one_plan_agree_bitwise():
    # One 64x32 four-chain plan, ragged in N (the last 64-column lockstep pair is half outside N)
    # and in K (113 chunks: chain 0 has 29 chunks and chains 1-3 have 28, and the last group of
    # every form is short).  M = 1 takes the tiny-batch form (16 chunks per stage), M = 20 the
    # small-batch form (8), M = 64 the plan's own form (4), M = 100 (258 tiles > 148 SMs) the
    # two-tile and M = 300 (645 tiles) the four-tile lockstep form: a row's bits must not depend
    # on which of them ran it.
    N, K = 4128, 7232
    B = inputs.bf16_gaussian((N, K), seed=2101, std=K ** -0.5, device=DEV)
    f = Dense(B)
    info = bg.bi_gemm_plan_describe(f.plan)
    assert (info["block_m"], info["block_n"], info["k_order_id"]) == (64, 32, 3)
    test_rows = inputs.bf16_gaussian((24, K), seed=2102, device=DEV)
    ref = alone(f, test_rows)
    for M in [20, 64, 100, 300]:
        s = inputs.derived_seed(2100, M, 0)
        fresh = lambda m, s=s: inputs.bf16_gaussian((m, K), seed=s, device=DEV)
        check_in_batch(f, test_rows, ref, M, s, fresh)
        check_in_batch(f, test_rows, ref, M, M, fresh,
                       positions=sorted({q for q in (0, 63, 64, 127, 128, M - 1) if q < M}))


def adversarial_bf16(shape, kind, seed, device="cpu"):
    """bf16 operands built to expose any difference in how an instruction sums its K products:
    exponents spread over 2^-24..2^24 ("wide"), pairs that cancel to a few ulps ("cancel"), or a
    small background under 1 % large spikes ("spikes").  Drawn on `device`, returned on the GPU."""
    g = torch.Generator(device=device).manual_seed(seed)
    kw = dict(generator=g, device=device)
    if kind == "spikes":
        x = torch.randn(shape, **kw) * 2.0 ** -10
        mask = torch.rand(shape, **kw) < 0.01
        x = torch.where(mask, torch.randn(shape, **kw) * 2.0 ** 10, x)
        return x.to(torch.bfloat16).to(DEV)
    e = torch.randint(-24, 25, shape, **kw).float()
    sign = torch.randint(0, 2, shape, **kw).float() * 2 - 1
    x = sign * (1 + torch.rand(shape, **kw)) * torch.exp2(e)
    del e, sign
    if kind == "cancel":
        odd = x[..., 1::2]
        x[..., 1::2] = -x[..., 0::2][..., : odd.shape[-1]] * (
            1 + 2.0 ** -7 * torch.randint(-2, 3, odd.shape, **kw).float())
    return x.to(torch.bfloat16).to(DEV)


@pytest.mark.parametrize("kind", ["wide", "cancel", "spikes"])
def test_scheduling_forms_agree_bitwise_on_adversarial_inputs(kind):
    # The wide lockstep forms issue one 64 x 64 or 64 x 128 instruction where the plan's own form
    # issues 64 x 32 ones; the rows of every form must still carry the M = 1 bits, on inputs whose
    # sums depend on the order and width of each instruction's internal reduction.
    N, K = 4128, 7232
    B = adversarial_bf16((N, K), kind, 2201)
    f = Dense(B)
    test_rows = adversarial_bf16((16, K), kind, 2202)
    ref = alone(f, test_rows)
    for M in [8, 20, 64, 100, 300]:
        s = inputs.derived_seed(2200, M, 0)
        fresh = lambda m, s=s: adversarial_bf16((m, K), kind, s)
        check_in_batch(f, test_rows, ref, M, s, fresh,
                       positions=sorted({q for q in (0, 31, 63, 64, 127, 128, 255, M - 1) if q < M}))


# ---------------------------------------------------------------------------------------------
# prefill-shaped: both shapes, M in {1024, 4096, 16384}, plus the 1024-row subset test
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(7168, 2048), (2048, 7168)])
def test_prefill_rows_invariant_and_subsets(N, K):
    B = inputs.bf16_gaussian((N, K), seed=3001, std=K ** -0.5, device=DEV)
    f = Dense(B)
    test_rows = inputs.bf16_gaussian((256, K), seed=3002, device=DEV)
    ref = alone(f, test_rows)
    batches = {}
    for M in [1024, 4096, 16384]:
        s = inputs.derived_seed(3000, M)
        fresh = lambda m, s=s: inputs.bf16_gaussian((m, K), seed=s, device=DEV)
        check_in_batch(f, test_rows, ref, M, s, fresh)
        batches[M] = fresh(M)
    # a random 1024-row subset of the 16384-row batch, run as its own call
    big = batches[16384]
    Cbig = f(big).view(torch.int16)
    idx = torch.from_numpy(np.random.default_rng(7).choice(16384, 1024, replace=False)).to(DEV)
    Csub = f(big[idx].contiguous()).view(torch.int16)
    assert torch.equal(Csub, Cbig[idx])


# ---------------------------------------------------------------------------------------------
# FP8 block-scaled: M = 1 .. 4096, co-batched rows with different scales
# ---------------------------------------------------------------------------------------------

def test_fp8_rows_invariant_across_m_sweep():
    N = K = 7168
    KB = K // 128
    qb = inputs.e4m3_gaussian((N, K), seed=4001, device=DEV)
    sb = inputs.scales_log_uniform((N // 128, KB), seed=4002, device=DEV)
    f = Dense(qb, bg.BI_DTYPE_E4M3_BLOCKSCALED, scale_b=sb)
    test_rows = inputs.e4m3_gaussian((32, K), seed=4003, device=DEV)
    test_scales = inputs.scales_log_uniform((32, KB), seed=4004, device=DEV)
    ref = alone(f, test_rows, test_scales)
    for M in [2, 4, 8, 16, 32, 64, 128, 256, 512, 1024, 2048, 4096]:
        for trial in range(2):
            s = inputs.derived_seed(4000, M, trial)
            check_in_batch(f, test_rows, ref, M, s,
                           lambda m, s=s: inputs.e4m3_gaussian((m, K), seed=s, device=DEV),
                           scales=test_scales,
                           fresh_scales=lambda m, s=s: inputs.scales_log_uniform((m, KB), seed=s + 1,
                                                                                 device=DEV))


def e4m3_any_codes(shape, seed):
    """Uniformly random e4m3 codes over the whole format (subnormals to +-448, no NaN)."""
    g = torch.Generator().manual_seed(seed)
    c = torch.randint(0, 256, shape, generator=g, dtype=torch.int32)
    c = torch.where((c & 0x7F) == 0x7F, c - 1, c)   # 0x7F / 0xFF are NaN in e4m3fn
    return c.to(torch.uint8).view(torch.float8_e4m3fn).to(DEV)


def test_fp8_forms_agree_bitwise_on_full_range_codes():
    # The FP8 wide lockstep form issues one 128 x 128 x 32 instruction where the plan's form
    # issues 128 x 64 x 32 ones; with codes spread over the whole e4m3 range the products of one
    # instruction span ~2^34, so any difference in its internal alignment would show.
    N = K = 7168
    KB = K // 128
    qb = e4m3_any_codes((N, K), 4101)
    sb = inputs.scales_log_uniform((N // 128, KB), seed=4102, device=DEV)
    f = Dense(qb, bg.BI_DTYPE_E4M3_BLOCKSCALED, scale_b=sb)
    test_rows = e4m3_any_codes((8, K), 4103)
    test_scales = inputs.scales_log_uniform((8, KB), seed=4104, device=DEV)
    ref = alone(f, test_rows, test_scales)
    for M in [16, 256, 1024]:
        s = inputs.derived_seed(4100, M)
        check_in_batch(f, test_rows, ref, M, s, lambda m, s=s: e4m3_any_codes((m, K), s),
                       scales=test_scales,
                       fresh_scales=lambda m, s=s: inputs.scales_log_uniform((m, KB), seed=s + 1,
                                                                             device=DEV),
                       positions=[0, 127, 128, M - 1] if M > 128 else [0, M - 1])


# ---------------------------------------------------------------------------------------------
# grouped MoE: per (token, expert) rows invariant to T and to the other tokens of the expert
# ---------------------------------------------------------------------------------------------

def moe_outputs(plan, B, tokens, routing):
    A = tokens[routing.token_of_row.to(DEV)].contiguous()
    C = torch.empty((A.shape[0], B.shape[1]), dtype=torch.bfloat16, device=DEV)
    bg.bi_grouped_gemm_run(plan, A, B, C, routing.offsets.to(DEV))
    bg.bi_gemm_sync_status(plan)
    return C.view(torch.int16)


def pair_bits(C, routing):
    """{(token, expert): output bits} for a grouped result."""
    tok = routing.token_of_row.tolist()
    exp = routing.expert_of_row.tolist()
    return {(t, e): C[i] for i, (t, e) in enumerate(zip(tok, exp))}


def test_moe_rows_invariant_to_t_and_routing():
    E, N, K = 64, 2048, 7168
    plan = bg.bi_gemm_plan(N, K, bg.BI_DTYPE_BF16, E)
    B = inputs.bf16_gaussian((E, N, K), seed=5001, std=K ** -0.5, device=DEV)
    test_tokens = inputs.bf16_gaussian((16, K), seed=5002, device=DEV)
    test_logits_seed = 5003
    # each test token alone (T = 1): its 8 (token, expert) rows
    g = inputs.generator(test_logits_seed, DEV)
    test_logits = torch.randn(16, E, generator=g, device=DEV)
    test_experts = routing_mod.topk_experts(test_logits, 8)
    ref = {}
    for i in range(16):
        r = routing_mod.route(test_logits[i:i + 1], E, 8)
        out = pair_bits(moe_outputs(plan, B, test_tokens[i:i + 1], r), r)
        for (t, e), v in out.items():
            ref[(i, e)] = v
    for T in [64, 1024, 8192]:
        s = inputs.derived_seed(5000, T)
        tokens = inputs.bf16_gaussian((T, K), seed=s, device=DEV)
        logits = torch.randn(T, E, generator=inputs.generator(s + 1, DEV), device=DEV)
        pos = np.random.default_rng(T).choice(T, size=16, replace=False)
        tokens[torch.from_numpy(pos).to(DEV)] = test_tokens
        logits[torch.from_numpy(pos).to(DEV)] = test_logits
        r = routing_mod.route(logits, E, 8)
        out = pair_bits(moe_outputs(plan, B, tokens, r), r)
        for i, p in enumerate(pos):
            for e in test_experts[i].tolist():
                assert torch.equal(out[(int(p), e)], ref[(i, e)]), f"T={T} token {i} expert {e}"


@pytest.mark.parametrize("pattern", ["all_one_expert", "segments_127_128_129", "singletons"])
def test_moe_adversarial_routings(pattern):
    E, N, K = 8, 256, 512
    plan = bg.bi_gemm_plan(N, K, bg.BI_DTYPE_BF16, E)
    B = inputs.bf16_gaussian((E, N, K), seed=5101, device=DEV)
    tokens = inputs.bf16_gaussian((400, K), seed=5102, device=DEV)
    if pattern == "all_one_expert":
        experts = np.full(400, 3)
    elif pattern == "segments_127_128_129":
        experts = np.repeat([0, 1, 2, 5], [127, 128, 129, 16])
    else:
        experts = np.concatenate([np.arange(8), np.full(392, 7)])
    experts = np.sort(experts)
    r = routing_mod.routing_from_assignment(experts, E)
    C = moe_outputs(plan, B, tokens, r)
    # every row equals the same token computed alone with its expert (a one-row call)
    for i in np.random.default_rng(1).choice(400, 40, replace=False):
        e = int(experts[i])
        one = routing_mod.routing_from_assignment(np.array([e]), E)
        C1 = moe_outputs(plan, B, tokens[i:i + 1], one)
        assert torch.equal(C1[0], C[i]), f"{pattern}: row {i}"
    # and the same as a dense call with that expert's weights, where the two plans share a tile
    if pattern == "all_one_expert":
        f = Dense(B[3].contiguous())
        dense_info = bg.bi_gemm_plan_describe(f.plan)
        grouped_info = bg.bi_gemm_plan_describe(plan)
        same = {k: v for k, v in dense_info.items() if k != "num_experts"} == \
            {k: v for k, v in grouped_info.items() if k not in ("num_experts", "smem_bytes")} | \
            {"smem_bytes": dense_info["smem_bytes"]}
        if same:
            assert torch.equal(f(tokens).view(torch.int16), C)


@pytest.mark.parametrize("kind", ["cancel", "spikes"])
def test_moe_wide_form_agrees_bitwise_on_adversarial_inputs(kind):
    # 8448 rows over the 64 experts (>= 128 per expert on average) take the grouped wide form:
    # 2 x 2 tiles of the 128 x 128 plan on a CTA pair, one 256 x 256 cta_group::2 instruction
    # per K step.  A row alone takes the plan's own 128 x 128 form.
    E, N, K, R = 64, 2048, 7168, 8448
    plan = bg.bi_gemm_plan(N, K, bg.BI_DTYPE_BF16, E)
    info = bg.bi_gemm_plan_describe(plan)
    assert (info["block_m"], info["block_n"]) == (128, 128)
    B = adversarial_bf16((E, N, K), kind, 5201, device=DEV)
    tokens = adversarial_bf16((R, K), kind, 5202, device=DEV)
    experts = np.sort(np.random.default_rng(5203).integers(0, E, R))
    r = routing_mod.routing_from_assignment(experts, E)
    C = moe_outputs(plan, B, tokens, r)
    for i in np.random.default_rng(5204).choice(R, 24, replace=False):
        e = int(experts[i])
        one = routing_mod.routing_from_assignment(np.array([e]), E)
        C1 = moe_outputs(plan, B, tokens[i:i + 1], one)
        assert torch.equal(C1[0], C[i]), f"{kind}: row {i}"
