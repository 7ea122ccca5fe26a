"""The bounds-checked build (libmoe_checked.so, compiled with -DMOE_CHECKS) on the GPU.

Each case runs in a child process that loads the checked library (MOE_LIB=checked):
  - a small layer computes the same result as the float64 oracle, with no check firing;
  - a corrupted map or table, injected from the host the way a caller's bug would pass
    it, is caught: the kernel records MOE_ERR_BAD_INDEX in the registered word, skips the
    access, and the guard bands around its output stay untouched:
      tok2row out of range (permute and combine), send2row (staged permute), expert_off
      and n_e describing rows past the routed block (grouped FFN, bf16 and block-scaled
      MX), row2tok out of range (the FC2 gate).
Nothing traps: every fault is turned into a status before any access.
"""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent(r'''
    import sys, numpy as np, torch
    sys.path.insert(0, sys.argv[1])
    import dispatch_combine_grouped_b200 as moe
    from moe_inputs import small_config, make_inputs
    from oracle import moe_oracle as O
    from tests.gpu_cases import assert_close_fro
    assert moe.checks_enabled(), "not the checked library"
    word = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.checks_register(word)
    BAD = 5
    G = 4096  # guard elements on each side

    def guarded(shape, dtype):
        n = int(np.prod(shape))
        buf = torch.full((n + 2 * G,), 77, dtype=dtype, device="cuda")
        return buf, buf[G:G + n].view(*shape)

    def guards_ok(buf):
        return bool((buf[:G] == 77).all()) and bool((buf[-G:] == 77).all())

    def fired():
        torch.cuda.synchronize()
        v = int(word.item())
        word.zero_()
        return v

    cfg = small_config("chk", cfg_id=70, N=257, d=200, E=8, S=1, k=2, I=136, P=2)
    inp = make_inputs(cfg, device="cuda")
    case = sys.argv[2]
    if case == "clean":
        for c in (cfg, small_config("chk_pairs", cfg_id=79, N=700, d=4096, E=8, S=1, k=2, I=200, P=4)):
            inp = make_inputs(c, device="cuda")
            y = moe.layer_forward(c, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], inp["w13"], inp["w2"])
            logits, ids, _ = moe.route(c, inp["x"], inp["w_gate"], inp["bias"])
            assert fired() == 0
            r = O.moe_layer(c, inp["x"], inp["w_gate"], inp["bias"], inp["w13"], inp["w2"],
                            select_keys=logits.cpu().numpy())
            assert_close_fro(y, r["y"], what=c.name)
    else:
        logits, ids, w = moe.route(cfg, inp["x"], inp["w_gate"], inp["bias"])
        lay = moe.dispatch_layout(cfg, ids)
        A = cfg.N * cfg.k
        xp = moe.permute(cfg, lay, inp["x"])
        h, out = moe.grouped_ffn(cfg, lay, xp, inp["x"], inp["w13"], inp["w2"], topk_w=w)
        assert fired() == 0
        if case == "permute":
            lay["tok2row"][5] = A + 1000
            buf, dst = guarded((A, cfg.d), torch.bfloat16)
            moe.permute(cfg, lay, inp["x"], out=dst)
            assert fired() == BAD and guards_ok(buf)
        elif case == "staged":
            lay["send2row"][3] = A + 7
            moe.permute_staged(cfg, lay, inp["x"])
            assert fired() == BAD
        elif case == "combine":
            lay["tok2row"][9] = 10 * A
            buf, y = guarded((cfg.N, cfg.d), torch.bfloat16)
            moe.combine(cfg, lay, out, y=y)
            assert fired() == BAD and guards_ok(buf)
        elif case == "ffn_groups":
            lay["expert_off"][2] = A - 3          # expert 2's rows would run past the routed rows
            hb, hh = guarded((A + cfg.N, cfg.I), torch.bfloat16)
            ob, oo = guarded((A + cfg.N, cfg.d), torch.bfloat16)
            moe.grouped_ffn(cfg, lay, xp, inp["x"], inp["w13"], inp["w2"], topk_w=w, h=hh, out=oo)
            assert fired() == BAD and guards_ok(hb) and guards_ok(ob)
        elif case == "mx_groups":  # the block-scaled kernel checks its group table the same way
            c = small_config("chk_mx", cfg_id=130, N=200, d=512, E=8, S=1, k=2, I=256, P=2)
            inp = make_inputs(c, device="cuda")
            logits, ids, w = moe.route(c, inp["x"], inp["w_gate"], inp["bias"])
            lay = moe.dispatch_layout(c, ids)
            A = c.N * c.k
            x_q, x_sf = moe.quantize_mx(inp["x"])
            w13_q, w13_sf = moe.quantize_mx(inp["w13"])
            w2_q, w2_sf = moe.quantize_mx(inp["w2"])
            xp, xp_sf = moe.permute_mx(c, lay, x_q, x_sf)
            moe.grouped_ffn_mx(c, lay, xp, xp_sf, x_q, x_sf, w13_q, w13_sf, w2_q, w2_sf, topk_w=w)
            assert fired() == 0
            lay["expert_off"][2] = A - 3
            hb, hh = guarded((A + c.N, c.I), torch.bfloat16)
            ob, oo = guarded((A + c.N, c.d), torch.bfloat16)
            moe.grouped_ffn_mx(c, lay, xp, xp_sf, x_q, x_sf, w13_q, w13_sf, w2_q, w2_sf, topk_w=w, h=hh, out=oo)
            assert fired() == BAD and guards_ok(hb) and guards_ok(ob)
        elif case == "gate":
            lay["row2tok"][0] = -5
            ob, oo = guarded((A + cfg.N, cfg.d), torch.bfloat16)
            moe.grouped_ffn(cfg, lay, xp, inp["x"], inp["w13"], inp["w2"], topk_w=w, h=h, out=oo)
            assert fired() == BAD and guards_ok(ob)
        else:
            raise SystemExit("unknown case " + case)
    print("CHECKED_OK", case)
''')


@pytest.fixture(scope="module")
def checked_lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location("_moe_build", os.path.join(ROOT, "dispatch_combine_grouped_b200",
                                                                             "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    return b.build(checked=True)


@pytest.mark.parametrize("case", ["clean", "permute", "staged", "combine", "ffn_groups", "mx_groups", "gate"])
def test_checked_build(checked_lib, case):
    env = dict(os.environ, MOE_LIB="checked")
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT, case], capture_output=True, text=True, env=env,
                       timeout=600, cwd=ROOT)
    assert r.returncode == 0 and f"CHECKED_OK {case}" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
