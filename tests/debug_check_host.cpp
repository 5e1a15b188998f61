// Host program for tests/test_debug_check.py: runs the debug build's
// check-recording function on the host, where the error word is ordinary
// memory, and prints what the word holds after each step.
#include <cstdio>

#include "debug_check.cuh"

int main()
{
    int word[4] = {0, 0, 0, 0};
    const bool in = csa::record_check(word, csa::kChkListPos, 2559, 2560);
    std::printf("in_bounds %d word %d %d %d %d\n", in ? 1 : 0, word[0], word[1], word[2], word[3]);
    const bool out = csa::record_check(word, csa::kChkListPos, 2560, 2560);
    std::printf("past_end %d word %d %d %d %d\n", out ? 1 : 0, word[0], word[1], word[2], word[3]);
    const bool neg = csa::record_check(word, csa::kChkTmemEpi, -1, 512);
    std::printf("negative %d word %d %d %d %d\n", neg ? 1 : 0, word[0], word[1], word[2], word[3]);
    return 0;
}
