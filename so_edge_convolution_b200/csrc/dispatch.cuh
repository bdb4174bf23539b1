// dispatch.cuh -- compile-time instances of the per-edge kernels by shape.
#pragma once

// Common shapes get kernels with lmax fixed at compile time (LC), the rest
// the generic ones (LC = -1).
#define DISPATCH_LM(L_, mm, ...)                                        \
  if ((L_) == 4 && (mm) == 2) {                                         \
    constexpr int MM = 2, LC = 4;                                       \
    __VA_ARGS__;                                                        \
  } else if ((L_) == 6 && (mm) == 2) {                                  \
    constexpr int MM = 2, LC = 6;                                       \
    __VA_ARGS__;                                                        \
  } else if ((L_) == 2 && (mm) == 2) {                                  \
    constexpr int MM = 2, LC = 2;                                       \
    __VA_ARGS__;                                                        \
  } else {                                                              \
    constexpr int LC = -1;                                              \
    DISPATCH_MM(mm, __VA_ARGS__);                                       \
  }

#define DISPATCH_MM(mm, ...)                  \
  switch (mm) {                               \
    case 0: { constexpr int MM = 0; __VA_ARGS__; } break; \
    case 1: { constexpr int MM = 1; __VA_ARGS__; } break; \
    case 2: { constexpr int MM = 2; __VA_ARGS__; } break; \
    case 3: { constexpr int MM = 3; __VA_ARGS__; } break; \
    case 4: { constexpr int MM = 4; __VA_ARGS__; } break; \
    case 5: { constexpr int MM = 5; __VA_ARGS__; } break; \
    default: { constexpr int MM = 6; __VA_ARGS__; } break; \
  }
