#pragma once
#include "warp_emu.h"
