"""The Python binding's argument checks, on CPU tensors: the library sees only pointers, so the
binding must refuse any tensor whose shape, dtype, contiguity or device differs from what the call
reads or writes -- before the library is called.  With every check passed, a CPU tensor is then
refused as not being on a GPU."""
import pytest
import torch

from draft_block_causal_b200 import domino

B, L, d, Hs, r, V = 2, 3, 16, 8, 8, 40


def _weights(dtype=torch.bfloat16, **override):
    shapes = {"embed": (V, d), "W_ih": (3 * Hs, d), "W_hh": (3 * Hs, Hs), "b_ih": (3 * Hs,), "b_hh": (3 * Hs,),
              "W1": (r, d + Hs), "W2": (V, r)}
    shapes.update(override)
    return domino.HeadWeights(**{k: torch.zeros(v, dtype=dtype) for k, v in shapes.items()})


def _inputs(dtype=torch.bfloat16):
    return (torch.zeros(B, L, V, dtype=dtype), torch.zeros(B, L, d, dtype=dtype), torch.zeros(B, Hs))


def test_well_formed_cpu_arguments_pass_every_check_and_stop_at_the_device():
    w = _weights()
    lb, h, S0 = _inputs()
    with pytest.raises(ValueError, match="CUDA"):
        domino.draft_greedy(w, lb, h, S0, logits_out=True, states_out=True)
    with pytest.raises(ValueError, match="CUDA"):
        domino.teacher_forced(w, lb, h, S0, torch.zeros(B, L, dtype=torch.int32), states_out=True)


@pytest.mark.parametrize("name,shape", [("W1", (r, d)), ("W_ih", (3 * Hs, d + 1)), ("b_hh", (Hs,)),
                                        ("W_hh", (2 * Hs, Hs))])
def test_weight_shapes_must_agree(name, shape):
    # checked when the weights are put together, and again when one of them is replaced
    with pytest.raises(ValueError, match=f"weight {name} has shape"):
        _weights(**{name: shape})
    w = _weights()
    before = getattr(w, name)
    with pytest.raises(ValueError, match=f"weight {name} has shape"):
        setattr(w, name, torch.zeros(shape, dtype=torch.bfloat16))
    assert getattr(w, name) is before  # the rejected tensor is not kept


def test_weights_share_one_storage_type():
    w = _weights()
    with pytest.raises(ValueError, match="weight b_ih has dtype"):
        w.b_ih = w.b_ih.float()
    w = _weights()
    with pytest.raises(ValueError, match="embed_proj has dtype"):
        w.embed_proj = torch.zeros(V, 3 * Hs, dtype=torch.bfloat16)
    w.embed_proj = torch.zeros(V, 3 * Hs)  # the right table is accepted


def test_head_inputs_are_checked():
    w = _weights()
    lb, h, S0 = _inputs()
    cases = [
        (dict(base_logits=lb.float()), "base_logits has dtype"),
        (dict(base_logits=lb[:, :, : V - 8]), "base_logits has shape"),
        (dict(hidden=torch.zeros(B, L, d + 8, dtype=torch.bfloat16)), "hidden has shape"),
        (dict(hidden=torch.zeros(B, d, L, dtype=torch.bfloat16).transpose(1, 2)), "hidden must be contiguous"),
        (dict(S0=S0.double()), "S0 has dtype"),
        (dict(S0=torch.zeros(B + 1, Hs)), "S0 has shape"),
    ]
    for bad, msg in cases:
        args = dict(base_logits=lb, hidden=h, S0=S0)
        args.update(bad)
        with pytest.raises(ValueError, match=msg):
            domino.draft_greedy(w, args["base_logits"], args["hidden"], args["S0"])


def test_outputs_status_and_workspace_are_checked():
    w = _weights()
    lb, h, S0 = _inputs()
    with pytest.raises(ValueError, match="tokens_out has dtype"):
        domino.draft_greedy(w, lb, h, S0, tokens_out=torch.zeros(B, L, dtype=torch.int64))
    with pytest.raises(ValueError, match="logits_out has shape"):
        domino.draft_greedy(w, lb, h, S0, logits_out=torch.zeros(B, L, V - 8))
    with pytest.raises(ValueError, match="states_out has dtype"):
        domino.draft_greedy(w, lb, h, S0, states_out=torch.zeros(B, L, Hs, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="status"):
        domino.draft_greedy(w, lb, h, S0, status=torch.zeros(1, dtype=torch.int64))
    with pytest.raises(ValueError, match="workspace"):
        domino.draft_greedy(w, lb, h, S0, workspace=torch.zeros(64, dtype=torch.float32))
    with pytest.raises(ValueError, match="tokens_out has shape"):
        domino.draft_greedy_noalloc(w, lb, h, S0, tokens_out=torch.zeros(B, L + 1, dtype=torch.int32))


def test_teacher_forcing_arguments_are_checked():
    w = _weights()
    lb, h, S0 = _inputs()
    y = torch.zeros(B, L, dtype=torch.int32)
    with pytest.raises(ValueError, match="tokens has dtype"):
        domino.teacher_forced(w, lb, h, S0, y.long())
    with pytest.raises(ValueError, match="tokens has shape"):
        domino.teacher_forced(w, lb, h, S0, y[:, :-1])
    with pytest.raises(ValueError, match="logits_out has dtype"):
        domino.teacher_forced(w, lb, h, S0, y, logits_dtype=torch.float16)
    with pytest.raises(ValueError, match="states_out has shape"):
        domino.teacher_forced(w, lb, h, S0, y, states_out=torch.zeros(B, L, Hs + 1))


def test_accept_length_arguments_are_checked():
    T = torch.zeros(B, L, V)
    t = torch.zeros(B, L, dtype=torch.int32)
    with pytest.raises(ValueError, match="target_logits has dtype"):
        domino.accept_len(t, T.double())
    with pytest.raises(ValueError, match="draft_tokens has shape"):
        domino.accept_len(t[:1], T)
    with pytest.raises(ValueError, match="accept_out has dtype"):
        domino.accept_len(t, T, accept_out=torch.zeros(B, dtype=torch.int64))


def test_debug_gemm_operands_are_checked():
    A = torch.zeros(128, 64, dtype=torch.bfloat16)
    Bm = torch.zeros(16, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="A has shape"):
        domino.debug_gemm(A, Bm)  # K = 128 but A has 64 columns and no wrap
    with pytest.raises(ValueError, match="B has dtype"):
        domino.debug_gemm(A, Bm.float(), a_kwrap=64)
