"""Plant plausible mistakes in copies of the oracle and show that a pin fails.

Each mutant is the oracle function's own source with one edit (a dropped term, a
wrong sign, a wrong axis or index, a relaxed comparison), compiled into a private
namespace; the real oracle is never modified.  Every mutant must make at least one
of the pin checks in pins.py fail, otherwise the pins would not be able to tell the
oracle from a broken one.
"""
import inspect
import textwrap

import pytest

import pins
from oracle import attention, policy


def mutate(module, name, old, new, extra=None):
    src = textwrap.dedent(inspect.getsource(getattr(module, name)))
    assert src.count(old) >= 1, (name, old)
    src = src.replace(old, new, 1)
    ns = dict(vars(module))
    if extra:
        ns.update(extra)
    exec(compile(src, f"<mutant {name}>", "exec"), ns)
    return ns[name]


def caught(fn, *args):
    try:
        fn(*args)
    except (AssertionError, ValueError, FloatingPointError, IndexError, ZeroDivisionError):
        return True
    return False


ATTEND_MUTANTS = [
    ("dropped scale", "s = scale * (q @ k.T)", "s = (q @ k.T)"),
    ("softmax over the query axis", "mx = s.max(axis=1, keepdims=True)", "mx = s.max(axis=0, keepdims=True)"),
    ("normaliser summed over queries", "z = e.sum(axis=1)", "z = e.sum(axis=0)"),
    ("L without the max", "l = mx[:, 0] + np.log(z)", "l = np.log(z)"),
    ("wrong sign in the exponent", "e = np.exp(s - mx)", "e = np.exp(mx - s)"),
    ("unnormalised output", "a = (e @ v) / z[:, None]", "a = (e @ v)"),
]

MERGE_MUTANTS = [
    ("weights swapped", "a = (w_out[..., None] * a_out + w_in[..., None] * a_in)",
     "a = (w_in[..., None] * a_out + w_out[..., None] * a_in)"),
    ("L_full drops the log term", "l = np.where(empty, -np.inf, m_safe + np.log(den_safe))",
     "l = np.where(empty, -np.inf, m_safe)"),
    ("denominator drops a term", "den = w_out + w_in", "den = w_out + 0 * w_in + (w_in > 2)"),
    ("min instead of max", "m = np.maximum(l_out, l_in)", "m = np.minimum(l_out, l_in)"),
    ("both-empty merge gives L = 0", "l = np.where(empty, -np.inf, m_safe + np.log(den_safe))",
     "l = np.where(empty, 0.0, m_safe + np.log(den_safe))"),
]

DECIDE_MUTANTS = [
    ("tau: <= instead of <", "reuse &= (m < int(tau))[:, None]", "reuse &= (m <= int(tau))[:, None]"),
    ("gamma: >= instead of >", "reuse &= np.asarray(cos) > np.float64(gamma)",
     "reuse &= np.asarray(cos) >= np.float64(gamma)"),
    ("gates OR-ed", "reuse &= np.asarray(cos) > np.float64(gamma)",
     "reuse |= np.asarray(cos) > np.float64(gamma)"),
    ("invalid cache ignored", "return ~(reuse & valid)", "return ~reuse"),
    ("force reuse ignored", "if flags & FORCE_REUSE:", "if flags & 0:"),
]

CUMULATIVE_MUTANTS = [
    ("cumulative: <= instead of <", "reuse &= m < int(tau)", "reuse &= m <= int(tau)"),
    ("cumulative: this step's updates left out", "m = np.asarray(m_acc, dtype=np.int64) + np.asarray(n_updated, dtype=np.int64)[:, None]",
     "m = np.asarray(m_acc, dtype=np.int64) + 0 * np.asarray(n_updated, dtype=np.int64)[:, None]"),
]

NEXT_M_MUTANTS = [
    ("count not reset on recompute", "return np.where(recompute, 0, grown)", "return grown"),
    ("count reset on reuse", "return np.where(recompute, 0, grown)", "return np.where(recompute, grown, 0)"),
    ("updates dropped from the count", "grown = np.asarray(m_acc, dtype=np.int64) + np.asarray(n_updated, dtype=np.int64)[:, None]",
     "grown = np.asarray(m_acc, dtype=np.int64)"),
]

COSINE_MUTANTS = [
    ("no square root", "den = np.sqrt(np.dot(x, x) * np.dot(y, y))", "den = np.dot(x, x) * np.dot(y, y)"),
    ("cache addressed by packed row", "y = q_ref[crow[r0:r1], h].reshape(-1)", "y = q_ref[r0:r1, h].reshape(-1)"),
]

PROBLEM_MUTANTS = [
    ("GQA mapping h % H_kv", "hs = [h for h in head_list if h // g == hk]",
     "hs = [h for h in head_list if h % Hk == hk]"),
    ("keys of every sequence", "k0, k1 = _key_range(problem, which, b)",
     "k0, k1 = 0, int(k_bits.shape[0])"),
]


@pytest.mark.parametrize("label,old,new", ATTEND_MUTANTS, ids=[m[0] for m in ATTEND_MUTANTS])
def test_attend_mutants_caught(label, old, new):
    bad = mutate(attention, "attend", old, new)
    assert (caught(pins.check_golden_attend, bad) or caught(pins.check_brute_force, bad)
            or caught(pins.check_closed_forms, bad)), label


@pytest.mark.parametrize("label,old,new", MERGE_MUTANTS, ids=[m[0] for m in MERGE_MUTANTS])
def test_merge_mutants_caught(label, old, new):
    bad = mutate(attention, "merge", old, new)
    assert (caught(pins.check_golden_merge, bad)
            or caught(pins.check_fresh_cache_identity, attention.attend, bad)
            or caught(pins.check_merge_order_independent, attention.attend, bad)), label


@pytest.mark.parametrize("label,old,new", DECIDE_MUTANTS, ids=[m[0] for m in DECIDE_MUTANTS])
def test_decide_mutants_caught(label, old, new):
    bad = mutate(policy, "decide", old, new)
    assert caught(pins.check_golden_gates, bad), label


@pytest.mark.parametrize("label,old,new", CUMULATIVE_MUTANTS, ids=[m[0] for m in CUMULATIVE_MUTANTS])
def test_cumulative_mutants_caught(label, old, new):
    bad = mutate(policy, "decide", old, new)
    assert caught(pins.check_cumulative_gate, bad, policy.next_m_acc), label


@pytest.mark.parametrize("label,old,new", NEXT_M_MUTANTS, ids=[m[0] for m in NEXT_M_MUTANTS])
def test_next_m_mutants_caught(label, old, new):
    bad = mutate(policy, "next_m_acc", old, new)
    assert caught(pins.check_cumulative_gate, policy.decide, bad), label


@pytest.mark.parametrize("label,old,new", COSINE_MUTANTS, ids=[m[0] for m in COSINE_MUTANTS])
def test_cosine_mutants_caught(label, old, new):
    bad = mutate(policy, "head_cosine", old, new)
    assert caught(pins.check_cosine, bad), label


@pytest.mark.parametrize("label,old,new", PROBLEM_MUTANTS, ids=[m[0] for m in PROBLEM_MUTANTS])
def test_problem_mutants_caught(label, old, new):
    bad = mutate(attention, "attend_problem", old, new)
    assert caught(pins.check_problem_vs_brute, bad, attention.merge), label


def test_unmutated_oracle_passes_every_pin():
    pins.check_golden_attend(attention.attend)
    pins.check_brute_force(attention.attend)
    pins.check_closed_forms(attention.attend)
    pins.check_golden_merge(attention.merge)
    pins.check_fresh_cache_identity(attention.attend, attention.merge)
    pins.check_merge_order_independent(attention.attend, attention.merge)
    pins.check_golden_gates(policy.decide)
    pins.check_cosine(policy.head_cosine)
    pins.check_problem_vs_brute(attention.attend_problem, attention.merge)
    pins.check_cumulative_gate(policy.decide, policy.next_m_acc)
    pins.check_branch_hooks(policy.cache_copy_seq, policy.cache_invalidate_seqs)
    pins.check_policy_replay(policy.run_policy)
    pins.check_bf16_widening(attention.bf16_to_f64)
    from oracle import sparse, transition
    pins.check_block_transition(transition.grow_prefix, transition.finish_block, transition.next_block_workload,
                                policy.run_policy, attention.attend)
    pins.check_sparse_workload(sparse.sparse_workload, policy.run_policy, attention.attend_full)


SPARSE_MUTANTS = [
    ("selected keys also left in the residual", "keep[sel] = False", "keep[sel] = keep[sel]"),
    ("selected keys dropped", "ext_k.append(np.concatenate([k_in[i0:i1], k_out[o0:o1][sel]]))",
     "ext_k.append(np.concatenate([k_in[i0:i1], k_out[o0:o1][sel][:0]]))"),
    ("selection placed before the block", "ext_k.append(np.concatenate([k_in[i0:i1], k_out[o0:o1][sel]]))",
     "ext_k.append(np.concatenate([k_out[o0:o1][sel], k_in[i0:i1]]))"),
    ("values gathered from the keys", "res_v.append(v_out[o0:o1][keep])", "res_v.append(k_out[o0:o1][keep])"),
]


@pytest.mark.parametrize("label,old,new", SPARSE_MUTANTS, ids=[m[0] for m in SPARSE_MUTANTS])
def test_sparse_mutants_caught(label, old, new):
    from oracle import sparse
    bad = mutate(sparse, "rearrange", old, new)
    assert caught(pins.check_sparse_partition, bad, attention.attend_problem, attention.attend_full,
                  attention.merge), label


BRANCH_MUTANTS = [
    ("copy: source and destination swapped", "cache.a_out[d0:d0 + n] = cache.a_out[s0:s0 + n]",
     "cache.a_out[s0:s0 + n] = cache.a_out[d0:d0 + n]"),
    ("copy: one position short", "n = min(s1 - s0, d1 - d0)", "n = min(s1 - s0, d1 - d0) - 1"),
    ("copy: a longer destination marked valid", "cache.valid[dst] = cache.valid[src] & (d1 - d0 <= s1 - s0)",
     "cache.valid[dst] = cache.valid[src]"),
    ("copy: queries not copied", "cache.q_ref[d0:d0 + n] = cache.q_ref[s0:s0 + n]", "pass"),
    ("copy: count not copied", "cache.m_acc[dst] = cache.m_acc[src]", "pass"),
]

REFRESH_MUTANTS = [
    ("refresh: mask ignored", "cache.valid[m] = False", "cache.valid[:] = False"),
    ("refresh: count kept", "cache.m_acc[m] = 0", "cache.m_acc[m] = cache.m_acc[m]"),
]


@pytest.mark.parametrize("label,old,new", BRANCH_MUTANTS, ids=[m[0] for m in BRANCH_MUTANTS])
def test_branch_copy_mutants_caught(label, old, new):
    bad = mutate(policy, "cache_copy_seq", old, new)
    assert caught(pins.check_branch_hooks, bad, policy.cache_invalidate_seqs), label


@pytest.mark.parametrize("label,old,new", REFRESH_MUTANTS, ids=[m[0] for m in REFRESH_MUTANTS])
def test_refresh_mutants_caught(label, old, new):
    bad = mutate(policy, "cache_invalidate_seqs", old, new)
    assert caught(pins.check_branch_hooks, policy.cache_copy_seq, bad), label


POLICY_MUTANTS = [
    ("queries of a recompute not kept", "cache.q_ref[crow[rs_all], h] = q[rs_all, h]", "pass"),
    ("cache written at the packed row", "cache.a_out[crow[rs], h] = a", "cache.a_out[rs, h] = a"),
    ("a recompute never marks the entry valid", "cache.valid[b, h] = True", "pass"),
    ("cumulative count not advanced", "cache.m_acc = next_m_acc(flags, cache.m_acc, st.n_updated, rec)", "pass"),
    ("prefix of kv-head 0 for every head", "kk = bf16_to_f64(workload.k_out[o0:o1, hk])",
     "kk = bf16_to_f64(workload.k_out[o0:o1, 0])"),
]


@pytest.mark.parametrize("label,old,new", POLICY_MUTANTS, ids=[m[0] for m in POLICY_MUTANTS])
def test_policy_mutants_caught(label, old, new):
    bad = mutate(policy, "run_policy", old, new)
    assert caught(pins.check_policy_replay, bad), label


WIDEN_MUTANTS = [
    ("every value scaled by 1 + 2^-7", ".view(np.float32).astype(np.float64)",
     ".view(np.float32).astype(np.float64) * (1 + 2.0 ** -7)"),
    ("bits shifted by 15", "(b.astype(np.uint32) << 16)", "(b.astype(np.uint32) << 15)"),
    ("widened through float16", "(b.astype(np.uint32) << 16).view(np.float32)",
     "b.view(np.float16).astype(np.float32)"),
    ("low fraction bit dropped", "b = np.ascontiguousarray(bits, dtype=np.uint16)",
     "b = np.ascontiguousarray(bits, dtype=np.uint16) & np.uint16(0xFFFE)"),
]


@pytest.mark.parametrize("label,old,new", WIDEN_MUTANTS, ids=[m[0] for m in WIDEN_MUTANTS])
def test_widen_mutants_caught(label, old, new):
    bad = mutate(attention, "bf16_to_f64", old, new)
    assert caught(pins.check_bf16_widening, bad), label


SPARSE_WORKLOAD_MUTANTS = [
    ("the first step's block on every step",
     "rearrange(st.problem, workload.k_out, workload.v_out, st.k_in, st.v_in,",
     "rearrange(st.problem, workload.k_out, workload.v_out, workload.steps[0].k_in, workload.steps[0].v_in,"),
    ("the original prefix kept as the residual", "problem=p0, k_out=k_res, v_out=v_res,",
     "problem=p0, k_out=workload.k_out, v_out=workload.v_out,"),
    ("the step's queries replaced by step 0's", "steps.append(dataclasses.replace(st, k_in=k_ext, v_in=v_ext, problem=p2s))",
     "steps.append(dataclasses.replace(st, q=workload.steps[0].q if workload.steps[0].q.shape == st.q.shape else st.q, "
     "k_in=k_ext, v_in=v_ext, problem=p2s))"),
]


@pytest.mark.parametrize("label,old,new", SPARSE_WORKLOAD_MUTANTS, ids=[m[0] for m in SPARSE_WORKLOAD_MUTANTS])
def test_sparse_workload_mutants_caught(label, old, new):
    from oracle import sparse
    bad = mutate(sparse, "sparse_workload", old, new)
    assert caught(pins.check_sparse_workload, bad, policy.run_policy, attention.attend_full), label


GROW_MUTANTS = [
    ("block placed before the prefix", "ks.append(np.concatenate([k_out[o0:o1], k_in[i0:i1]]))",
     "ks.append(np.concatenate([k_in[i0:i1], k_out[o0:o1]]))"),
    ("values of the block taken from its keys", "vs.append(np.concatenate([v_out[o0:o1], v_in[i0:i1]]))",
     "vs.append(np.concatenate([v_out[o0:o1], k_in[i0:i1]]))"),
    ("block lengths left out of the new offsets", "lens.append((o1 - o0) + (i1 - i0))", "lens.append(o1 - o0)"),
    ("blocks of the next sequence", "i0, i1 = int(cu_i[b]), int(cu_i[b + 1])",
     "i0, i1 = int(cu_i[(b + 1) % problem.num_seqs]), int(cu_i[(b + 1) % problem.num_seqs + 1])"),
]

FINISH_MUTANTS = [
    ("the block's first step instead of its last", "last = workload.steps[-1]", "last = workload.steps[0]"),
]


@pytest.mark.parametrize("label,old,new", GROW_MUTANTS, ids=[m[0] for m in GROW_MUTANTS])
def test_grow_prefix_mutants_caught(label, old, new):
    from oracle import transition
    bad = mutate(transition, "grow_prefix", old, new)
    bad_finish = mutate(transition, "finish_block", "last = workload.steps[-1]", "last = workload.steps[-1]",
                        extra={"grow_prefix": bad})
    bad_next = mutate(transition, "next_block_workload", "cu, k, v = finish_block(finished)",
                      "cu, k, v = finish_block(finished)", extra={"finish_block": bad_finish})
    assert caught(pins.check_block_transition, bad, bad_finish, bad_next, policy.run_policy, attention.attend), label


@pytest.mark.parametrize("label,old,new", FINISH_MUTANTS, ids=[m[0] for m in FINISH_MUTANTS])
def test_finish_block_mutants_caught(label, old, new):
    from oracle import transition
    bad = mutate(transition, "finish_block", old, new)
    bad_next = mutate(transition, "next_block_workload", "cu, k, v = finish_block(finished)",
                      "cu, k, v = finish_block(finished)", extra={"finish_block": bad})
    assert caught(pins.check_block_transition, transition.grow_prefix, bad, bad_next, policy.run_policy,
                  attention.attend), label
