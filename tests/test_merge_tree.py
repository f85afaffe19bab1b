"""The split-K merge order (host logic, no GPU).

For the decode classes whose split count the tuner may change (up to 8 query rows per
kv-head), a CTA holds an aligned power-of-two run of merge-tree leaves and builds that
node of the tree with a binary counter (mq_decode_common.cuh, tree_step: carries while a
leaf closes a right child, the right edge at the CTA's last leaf); merge_kernel
(mq_decode.cu) combines the CTA partials over a binary tree over the CTA index, passing
a left child through where the right one starts past the last CTA.  This module restates
both on symbolic values (a leaf is its index, a merge is the pair (left, right)) and
checks that every power-of-two split count yields the one fixed binary tree over the
leaves: node (k, i) = (node (k-1, 2i), node (k-1, 2i+1)), or its left child when the
right one starts past the last leaf.  Equal trees mean the same floating-point operations
in the same order, so the output bytes cannot depend on the split count.
"""


def fixed_tree(n):
    H = 0
    while (1 << H) < n:
        H += 1

    def node(k, i):
        if k == 0:
            return i
        right = (2 * i + 1) << (k - 1)
        return (node(k - 1, 2 * i), node(k - 1, 2 * i + 1)) if right < n else node(k - 1, 2 * i)
    return node(H, 0)


def tree_step(li, l0, last, occ, kmax):
    mask, t, idx = 0, 0, li
    while t < kmax and (idx & 1) and ((idx - 1) << t) >= l0:
        mask |= 1 << t
        idx >>= 1
        t += 1
    if last:
        mask |= occ & ~mask
    return mask, t, not last


def cta_node(l0, l1, kmax):
    """The node a CTA builds from leaves [l0, l1)."""
    occ, slots = 0, {}
    for li in range(l0, l1):
        mask, level, push = tree_step(li, l0, li == l1 - 1, occ, kmax)
        cur = li
        for t in range(kmax):
            if (mask >> t) & 1:
                cur = (slots.pop(t), cur)
        if push:
            slots[level] = cur
            occ = (occ & ~mask) | (1 << level)
        else:
            assert not slots, "pending children left behind"
            return cur


def merge_over_ctas(parts):
    n = len(parts)
    H = 0
    while (1 << H) < n:
        H += 1
    nodes = list(parts)
    for lv in range(1, H + 1):
        nodes = [(nodes[2 * u], nodes[2 * u + 1]) if 2 * u + 1 < len(nodes) else nodes[2 * u]
                 for u in range((len(nodes) + 1) // 2)]
    return nodes[0]


def test_every_power_of_two_split_gives_the_fixed_tree():
    kmax = 8
    for n in list(range(1, 80)) + [127, 128, 129, 200, 255, 256]:
        padded = 1
        while padded < n:
            padded *= 2
        want = fixed_tree(n)
        for splits in (1, 2, 4, 8, 16, 32, 64):
            if splits > padded:
                continue
            lpc = padded // splits
            parts = [cta_node(l0, min(l0 + lpc, n), kmax) for l0 in range(0, n, lpc)]
            got = parts[0] if len(parts) == 1 else merge_over_ctas(parts)
            assert got == want, (n, splits)


def test_one_leaf_per_cta_keeps_the_sequential_tree_over_ctas():
    # the wider classes: a CTA's range is one leaf (kmax 0), the merge is over the CTAs
    for n_ctas in range(1, 65):
        parts = [cta_node(s, s + 1, 0) for s in range(n_ctas)]
        assert parts == list(range(n_ctas))
        assert merge_over_ctas(parts) == fixed_tree(n_ctas)
