"""The fused decode kernel names each launch by a tag that its CTAs derive on their own: every
CTA adds 1 to a 64-bit launch counter as it starts and takes tag = (value its add returned) //
gridDim.x + 1, kept in 32 bits. Values cross CTAs as 64-bit words tag << 32 | FP32 bits, and a
reader accepts a word once it carries its own launch's tag. This models the protocol on the
host, with CTA start orders drawn at random, and checks what the kernel relies on: all CTAs of
a launch derive the same tag, whatever order their adds land in; consecutive launches never
share a tag (also across the 32-bit wrap); no tag is 0, the value of zeroed words, also after
the host zeroes the counter; and a reader never accepts a word left by an earlier launch."""
import numpy as np

N_CTA = 148


def run_launches(counter: int, n_launches: int, rng, n=N_CTA):
    """Tags each CTA of each launch derives, and the counter afterwards."""
    tags = []
    for _ in range(n_launches):
        derived = np.empty(n, dtype=np.int64)
        for cta in rng.permutation(n):          # the order the CTAs' adds land in
            old = counter
            counter += 1
            derived[cta] = (old // n + 1) & 0xFFFFFFFF
        tags.append(derived)
    return tags, counter


def test_one_tag_per_launch_consecutive_launches_differ():
    rng = np.random.default_rng(7)
    tags, counter = run_launches(0, 50, rng)
    assert counter == 50 * N_CTA
    per_launch = [int(t[0]) for t in tags]
    for t in tags:
        assert np.all(t == t[0])
    assert per_launch == list(range(1, 51))
    assert 0 not in per_launch


def test_reset_restarts_at_one_and_zeroed_words_never_match():
    rng = np.random.default_rng(8)
    _, counter = run_launches(0, 7, rng)
    counter = 0                                  # the host zeroes counter and words together
    tags, _ = run_launches(counter, 3, rng)
    assert [int(t[0]) for t in tags] == [1, 2, 3]
    zero_word = 0
    assert all((zero_word >> 32) != int(t[0]) for t in tags)


def test_thirty_two_bit_wrap_keeps_consecutive_tags_apart():
    rng = np.random.default_rng(9)
    start = ((1 << 32) - 2) * N_CTA              # two launches before the 32-bit tag wraps
    tags, _ = run_launches(start, 4, rng)
    per_launch = [int(t[0]) for t in tags]
    for t in tags:
        assert np.all(t == t[0])
    assert per_launch == [(1 << 32) - 1, 0, 1, 2]
    assert all(a != b for a, b in zip(per_launch, per_launch[1:]))


def test_reader_accepts_only_its_own_launch_words():
    """Words written by launches with different token counts: a launch reads only words it
    writes itself, and before its write lands the word still carries an older tag."""
    rng = np.random.default_rng(10)
    words = np.zeros(8 * 128, dtype=np.uint64)   # [token, expert] logit words
    counter = 0
    for T in (8, 1, 3, 8, 2, 1, 8):
        tags, counter = run_launches(counter, 1, rng)
        tag = int(tags[0][0])
        mine = np.arange(T * 128)
        # before the writers store: no word this launch reads carries its tag
        assert np.all((words[mine] >> np.uint64(32)) != np.uint64(tag))
        vals = rng.standard_normal(T * 128).astype(np.float32)
        words[mine] = (np.uint64(tag) << np.uint64(32)) | vals.view(np.uint32).astype(np.uint64)
        got = words[mine]
        assert np.all((got >> np.uint64(32)) == np.uint64(tag))
        back = (got & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)
        assert np.array_equal(back.view(np.uint32), vals.view(np.uint32))
