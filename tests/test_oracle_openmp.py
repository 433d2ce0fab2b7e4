"""The oracle's OpenMP build (used only for the benchmark's all-cores CPU timing)
gives the same bits as the plain single-threaded build the pins check, on every
function it parallelises."""
import os

import numpy as np

import oracle
import workloads


def _chain(inputs):
    r = oracle.run_chain(inputs)
    wl = inputs["workload"]
    # the int8 round trip in combine and the smooth-scaled permute as well
    r["out_q8"] = oracle.combine_fwd(
        r["y"], inputs["topk_idx"], inputs["topk_weights"], r["assist"],
        num_experts=wl.num_experts, a_capacity=wl.a_capacity, dtype=wl.dtype,
        zero_expert_num=wl.zero_expert_num, copy_expert_num=wl.copy_expert_num,
        const_expert_num=wl.const_expert_num, mask=inputs["mask"], shared=inputs["shared"],
        ori_x=inputs["ori_x"], alpha1=inputs["alpha1"], alpha2=inputs["alpha2"],
        const_v=inputs["v"], comm_quant_mode=2)
    sm = workloads.smooth_scales(wl)
    r["smooth_q"], r["smooth_s"] = oracle.dispatch_permute_quant_smooth(
        inputs["x"], inputs["topk_idx"], sm, r["assist"], wl.a_capacity, wl.dtype)
    return r


def test_all_cores_build_matches_the_pinned_build():
    for base in (workloads.BY_NAME["dsv3_bs4096_h7168_k8_e256"].scaled(bs=300, h=512),
                 workloads.BY_NAME["mixtral_bs16384_h4096_k2_e8"].scaled(bs=700, h=264),
                 workloads.BY_NAME["special_int8_bs8192_h2048_k8_n70"].scaled(bs=400, h=256,
                                                                            backward=True)):
        inputs = workloads.generate(base)
        want = _chain(inputs)
        with oracle.all_cores():
            got = _chain(inputs)
            threads = oracle.num_threads()
        assert oracle.num_threads() == 1
        if (os.cpu_count() or 1) > 1:
            assert threads > 1
        for key, v in want.items():
            if isinstance(v, np.ndarray):
                assert np.array_equal(got[key].view(np.uint8), v.view(np.uint8)), key
            else:
                assert got[key] == v, key
