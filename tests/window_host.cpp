// Host build of the mask builder's window predicate (csrc/window.cuh), for the CPU tests:
// enumerates the window of every query tile of a T x Hs x Ws grid as a [NT, NT] byte
// matrix. The tests compare it with the oracle's own enumeration.
#include "window.cuh"

extern "C" int window_tiles(int T, int Hs, int Ws, int kind, int r, unsigned char* out) {
  const int nT = (T + 3) / 4, nY = (Hs + 3) / 4, nX = (Ws + 3) / 4;
  const int NT = nT * nY * nX;
  for (int i = 0; i < NT; ++i) {
    const uint32_t ci = bsa::pack_coord(i / (nY * nX), (i / nX) % nY, i % nX);
    for (int j = 0; j < NT; ++j) {
      const uint32_t cj = bsa::pack_coord(j / (nY * nX), (j / nX) % nY, j % nX);
      out[(long long)i * NT + j] = bsa::in_window(ci, cj, kind, r) ? 1 : 0;
    }
  }
  return NT;
}

// Support slots of key tile j for slot r of query tile i, one 64-bit mask.
extern "C" unsigned long long support_slots(int T, int Hs, int Ws, int i, int r, int j, int rho) {
  const int nY = (Hs + 3) / 4, nX = (Ws + 3) / 4;
  const int qt = 4 * (i / (nY * nX)) + (r >> 4), qy = 4 * ((i / nX) % nY) + ((r >> 2) & 3),
            qx = 4 * (i % nX) + (r & 3);
  return bsa::token_support_slots(qt, qy, qx, j / (nY * nX), (j / nX) % nY, j % nX, rho);
}

// [NT, NT] bytes: 1 where every valid token of key tile j lies in the support of every
// valid token of query tile i.
extern "C" int all_inside(int T, int Hs, int Ws, int rho, unsigned char* out) {
  const int nT = (T + 3) / 4, nY = (Hs + 3) / 4, nX = (Ws + 3) / 4;
  const int NT = nT * nY * nX;
  for (int i = 0; i < NT; ++i) {
    const uint32_t ci = bsa::pack_coord(i / (nY * nX), (i / nX) % nY, i % nX);
    for (int j = 0; j < NT; ++j) {
      const uint32_t cj = bsa::pack_coord(j / (nY * nX), (j / nX) % nY, j % nX);
      out[(long long)i * NT + j] = bsa::token_tiles_all_inside(ci, cj, T, Hs, Ws, rho) ? 1 : 0;
    }
  }
  return NT;
}
